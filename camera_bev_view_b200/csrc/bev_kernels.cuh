// bev_kernels.cuh -- launch parameters shared by the host layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "bev_geometry.cuh"

namespace bev {

// BEV tile owned by one CTA: kTileI rows (ego x) by kTileJ columns (ego y),
// worked on by kThreads threads (bev_tile.cuh).
constexpr int kTileI = 8;
constexpr int kTileJ = 8;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
static_assert(kTileJ % 4 == 0, "tile rows are stored as 16-byte vectors");

// Feature-pyramid levels.  Every level shares the voxel's projection,
// validity and count; level l samples its own map at its own scale.  The
// single-level operator is a table of one level.
constexpr int kMaxLevels = 4;

struct LevelTable {
    int n;                            // levels, 1 .. kMaxLevels
    int Hf[kMaxLevels], Wf[kMaxLevels];
    float sW[kMaxLevels], sH[kMaxLevels];  // (float)W_l / img_w, (float)H_l / img_h, host IEEE divide
    float* grad[kMaxLevels];          // fp32 channels-last gradient buffer of level l
};

struct SampleArgs {
    const float* K;         // [B,N,3,3]
    const float* E;         // [B,N,4,4]
    const float* dout;      // [B,C,X,Y]
    GeoParams g;            // grid and image (level sizes come from lv)
    int B, N, C;
    int cpl;                // channels per lane: a channel slice is 32 * cpl channels
    int cpad;               // channels per texel in the channels-last buffers (padded)
    int out_vec;            // dout is 16-byte aligned and Y % 4 == 0
    int tiles_i, tiles_j;   // tiles along X and Y
    LevelTable lv;          // feature levels
};

// Preferred shared-memory carveout for `ctas` CTAs of `smem` bytes each:
// the smallest shared-memory configuration of the SM (KB) that holds them,
// as a percentage of the 228 KB maximum; the rest of the array is L1.
inline int carveout_percent(size_t smem, int ctas) {
    const int sizes_kb[] = {0, 8, 16, 32, 64, 100, 132, 164, 196, 228};
    const size_t need = (size_t)ctas * (smem + 1024);
    for (int kb : sizes_kb)
        if ((size_t)kb * 1024 >= need) return (100 * kb + 227) / 228;
    return 100;
}

// A kernel's dynamic shared-memory limit and carveout preference, set once
// per device and size rather than on every launch (cudaFuncSetAttribute is a
// driver call that costs microseconds of host time).  `cache` is one static
// array per kernel; carveout < 0 leaves the preference alone.
constexpr int kAttrDevices = 64;

template <typename Kernel>
inline cudaError_t set_smem_attributes(Kernel* k, size_t smem, int carveout,
                                       std::atomic<long long> (&cache)[kAttrDevices]) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const long long key = (((long long)carveout + 1) << 32) | (long long)smem;
    const bool cached = dev >= 0 && dev < kAttrDevices;
    if (cached && cache[dev].load(std::memory_order_relaxed) == key) return cudaSuccess;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess && carveout >= 0)
        e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, carveout);
    if (e == cudaSuccess && cached) cache[dev].store(key, std::memory_order_relaxed);
    return e;
}

}  // namespace bev

// Launchers (defined next to their kernels).  The feature gradient: `slices`
// channel slices of 32 * a.cpl channels each.
cudaError_t bev_launch_backward(const bev::SampleArgs& a, int slices, cudaStream_t stream);
// The forward (bev_rows.cuh): `slices` channel slices, L lanes per cell (in
// the arguments) and V 16-byte chunks per lane.
namespace bev {
namespace row {
struct SampleArgs;
}
}  // namespace bev
cudaError_t bev_launch_forward_rows(const bev::row::SampleArgs& a, bool bf16, int V, int slices, cudaStream_t stream);
cudaError_t bev_launch_forward_rows_ms(const bev::row::SampleArgs& a, bool bf16, int V, int slices,
                                       cudaStream_t stream);
#ifdef BEV_BOUNDS_CHECK
// Checked build: read and clear the device error word of a dense kernel's
// translation unit (call after the launch's stream has drained).
unsigned bev_launch_forward_rows_check_take();
unsigned bev_launch_forward_rows_ms_check_take();
unsigned bev_backward_check_take();
#endif
cudaError_t bev_launch_to_channels_last(const void* src, int layout, int esize, int BN, int C,
                                        int HW, int Cp, void* dst, cudaStream_t stream);
cudaError_t bev_launch_to_nchw(const float* src, int BN, int C, int HW, int Cp, float* dst,
                               cudaStream_t stream);
