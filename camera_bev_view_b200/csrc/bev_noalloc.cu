// bev_noalloc.cu -- feature-gradient entry point that allocates nothing and
// needs no workspace from the caller.
//
// Some callers cannot hand the library a scratch buffer: a plugin inside an
// inference or training engine that plans all device memory itself and gives
// its plugins no allocator, a deployment that forbids device allocation once
// it has started (fixed memory budgets, certified stacks), or a real-time loop
// where cudaMalloc / cudaFree would stall the device and break the latency
// budget.  For them, bev_sample_backward_noalloc runs the normal backward with
// its fp32 channels-last accumulation buffer placed in a fixed-size array in
// the library's own device memory.
//
// The array is a file-scope __device__ variable, so every GPU that loads this
// library holds BEV_NOALLOC_SCRATCH_BYTES for it until the process exits.  On
// the host its name is only a stand-in, never a device address: the first call
// in each CUDA context asks the runtime for the real address with
// cudaGetSymbolAddress (that context current) and caches it, keyed by the
// device and by the context's unique id, so an address from a context that
// was destroyed (cudaDeviceReset) or from another context on the same device
// is never reused.  Every
// call shares the one array and leaves its contents behind; the backward clears
// the part it uses before accumulating, so stale contents never leak into a
// result.  Two calls whose work overlaps on the GPU (different streams, or
// different host threads) race on the array and must be serialised by the
// caller.
#include <cuda.h>  // driver API types; its two functions are fetched at run time

#include <mutex>

#include "bev_kernels.cuh"
#include "bevsample.h"

#define BEV_API extern "C" __attribute__((visibility("default")))

namespace {

static __device__ __align__(256) unsigned char g_backward_scratch[BEV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

struct CachedAddress {
    unsigned long long ctx_id;  // unique id of the context the address belongs to
    void* ptr;
};

std::mutex g_mu;
CachedAddress g_cache[kMaxDevices];

// Unique id of the current context (cuCtxGetId: ids are never reused within
// a process); false when the driver does not provide it.
bool current_context_id(unsigned long long* id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(f);
        cudaGetLastError();
    });
    CUcontext ctx = nullptr;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_backward_scratch in the current context of `dev`.
// Cached per (device, context id); without a context id it is looked up on
// every call.  nullptr if the runtime cannot provide it.
void* scratch_address(int dev) {
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    unsigned long long id = 0;
    const bool have_id = current_context_id(&id);
    std::lock_guard<std::mutex> lock(g_mu);
    if (have_id && g_cache[dev].ptr && g_cache[dev].ctx_id == id) return g_cache[dev].ptr;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_backward_scratch) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (have_id) g_cache[dev] = CachedAddress{id, p};
    return p;
}

}  // namespace

BEV_API int bev_sample_backward_noalloc(const float* dout, int B, int N, int C, int Hf, int Wf,
                                        const float* intrinsics, const float* ego2cam, int img_h,
                                        int img_w, const bev_grid_t* grid, float* dfeatures,
                                        bev_stream_t stream) {
    if (!dout || !intrinsics || !ego2cam || !dfeatures || !grid) return BEV_ERR_INVALID_ARG;
    const size_t need = bev_workspace_size(BEV_F32, BEV_NCHW, B, N, C, Hf, Wf, 1);
    if (need == (size_t)-1) return BEV_ERR_INVALID_ARG;
    if (need > (size_t)BEV_NOALLOC_SCRATCH_BYTES) return BEV_ERR_UNSUPPORTED;
    int dev;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return BEV_ERR_CUDA;
    }
    void* scratch = scratch_address(dev);
    if (!scratch) return BEV_ERR_CUDA;
    return bev_sample_backward(dout, B, N, C, Hf, Wf, intrinsics, ego2cam, img_h, img_w, grid, dfeatures,
                               scratch, (size_t)BEV_NOALLOC_SCRATCH_BYTES, stream);
}
