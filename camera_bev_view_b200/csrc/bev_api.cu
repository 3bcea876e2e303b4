// bev_api.cu -- host side of the C ABI declared in include/bevsample.h.
//
// Validates every argument before anything is enqueued, picks the launch
// shape (channel slices, lanes per cell) and enqueues the kernels on the
// caller's stream.  No allocation, no synchronisation, no global state.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "bev_deform.cuh"
#include "bev_lss.cuh"
#include "bev_kernels.cuh"
#include "bev_rows.cuh"
#include "bevsample.h"

#define BEV_API extern "C" __attribute__((visibility("default")))

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool dims_ok(int B, int N, int C, int Hf, int Wf) {
    if (B < 1 || N < 1 || C < 1 || Hf < 1 || Wf < 1) return false;
    if (N > BEV_MAX_CAMERAS || Hf > BEV_MAX_DIM || Wf > BEV_MAX_DIM) return false;
    if ((long long)B * N > 65535) return false;  // grid limits of the layout kernels
    if (C > (1 << 20)) return false;
    return true;
}

bool grid_ok(const bev_grid_t* g) {
    if (!g) return false;
    if (g->X < 1 || g->Y < 1 || g->Z < 1) return false;
    if (g->X > BEV_MAX_DIM || g->Y > BEV_MAX_DIM || g->Z > BEV_MAX_Z) return false;
    const float v[6] = {g->xmin, g->ymin, g->zmin, g->dx, g->dy, g->dz};
    for (float f : v)
        if (!isfinite(f)) return false;
    return g->dx > 0.0f && g->dy > 0.0f && g->dz > 0.0f;
}

// A pointer the kernels may dereference: device or managed memory of `dev`.
int device_ptr(const void* p, int dev) {
    if (!p) return BEV_ERR_INVALID_ARG;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return BEV_ERR_INVALID_ARG;
    }
    if (at.type == cudaMemoryTypeManaged) return BEV_OK;
    if (at.type != cudaMemoryTypeDevice || at.device != dev) return BEV_ERR_INVALID_ARG;
    return BEV_OK;
}

int current_device(int* dev) {
    if (cudaGetDevice(dev) != cudaSuccess) {
        cudaGetLastError();
        return BEV_ERR_CUDA;
    }
    return BEV_OK;
}

int chan_per_chunk(int dtype) { return dtype == BEV_BF16 ? 8 : 4; }
int elem_size(int dtype) { return dtype == BEV_BF16 ? 2 : 4; }
int round_up(int v, int m) { return (v + m - 1) / m * m; }

// Does the forward need a repacked channels-last copy of the features?
bool needs_repack(int dtype, int layout, int C) {
    return layout == BEV_NCHW || (C % chan_per_chunk(dtype)) != 0;
}

size_t forward_ws(int dtype, int layout, int B, int N, int C, int Hf, int Wf) {
    if (!needs_repack(dtype, layout, C)) return 0;
    const size_t Cp = (size_t)round_up(C, chan_per_chunk(dtype));
    return align_up((size_t)B * N * Hf * Wf * Cp * elem_size(dtype));
}

size_t backward_ws(int B, int N, int C, int Hf, int Wf) {
    return align_up((size_t)B * N * Hf * Wf * (size_t)round_up(C, 4) * sizeof(float));
}

bev::GeoParams geo(const bev_grid_t* g, int Hf, int Wf, int img_h, int img_w) {
    bev::GeoParams p;
    p.xmin = g->xmin;
    p.ymin = g->ymin;
    p.zmin = g->zmin;
    p.dx = g->dx;
    p.dy = g->dy;
    p.dz = g->dz;
    p.img_w = (float)img_w;
    p.img_h = (float)img_h;
    p.sW = (float)Wf / (float)img_w;
    p.sH = (float)Hf / (float)img_h;
    p.X = g->X;
    p.Y = g->Y;
    p.Z = g->Z;
    p.Hf = Hf;
    p.Wf = Wf;
    return p;
}

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return BEV_OK;
    cudaGetLastError();
    return BEV_ERR_CUDA;
}

// Status of a dense launch.  In the bounds-checked build the stream is
// drained and the kernel's device error word read back (by `take`): a check
// that failed on the device gives BEV_ERR_INTERNAL.
#ifdef BEV_BOUNDS_CHECK
using CheckTake = unsigned (*)();
#define BEV_TAKE(f) (f)
#else
using CheckTake = void*;
#define BEV_TAKE(f) nullptr
#endif

int dense_status(cudaError_t launch, cudaStream_t s, CheckTake take) {
    const int st = cuda_status(launch);
#ifdef BEV_BOUNDS_CHECK
    if (st != BEV_OK) return st;
    if (cudaStreamSynchronize(s) != cudaSuccess) return cuda_status(cudaErrorUnknown);
    return take() ? BEV_ERR_INTERNAL : BEV_OK;
#else
    (void)s;
    (void)take;
    return st;
#endif
}

// Lanes per cell L and 16-byte chunks per lane V (<= 8) for a slice of qs
// chunks (qs <= 32).  An exact fit with at most five chunks a lane comes
// first, eight lanes per cell before four, 16 and 32: each load instruction
// of eight lanes covers whole 128-byte lines of four cells, and no lane
// idles (80 fp32 channels take four lanes of five chunks, which measured 10%
// faster than eight lanes of three with a sixth of the slots idle).  Without
// an exact fit, eight lanes are kept unless they would leave more than a
// fifth of the slots idle.
void pick_lanes(int qs, int* L, int* V) {
    const int exact[4] = {8, 4, 16, 32};
    for (int k = 0; k < 4; ++k) {
        const int l = exact[k], v = qs / l;
        if (v >= 1 && v <= 5 && l * v == qs) {
            *L = l;
            *V = v;
            return;
        }
    }
    const int order[4] = {8, 16, 32, 4};
    for (int k = 0; k < 4; ++k) {
        const int l = order[k], v = (qs + l - 1) / l;
        if (v <= 8 && 5 * (l * v - qs) <= l * v) {
            *L = l;
            *V = v;
            return;
        }
    }
    int best_l = 4, best_v = (qs + 3) / 4, best_waste = 1 << 30;
    for (int k = 0; k < 4; ++k) {
        const int l = order[k], v = (qs + l - 1) / l;
        if (v > 8) continue;
        if (l * v - qs < best_waste) {
            best_waste = l * v - qs;
            best_l = l;
            best_v = v;
        }
    }
    *L = best_l;
    *V = best_v;
}


// Launch shape of the row forward for Cp channels in chunks of cpc: channel
// slices of up to kSliceMax channels, lanes per cell and chunks per lane;
// returns the chunks per lane V (0 when the slices exceed the grid limit).
int row_layout(bev::row::SampleArgs& a, int Cp, int cpc, const bev_grid_t* grid, int* slices) {
    a.Qtot = Cp / cpc;
    a.chan_per_chunk = cpc;
    const int max_chunks = bev::row::kSliceMax / cpc;
    *slices = (a.Qtot + max_chunks - 1) / max_chunks;
    if (*slices > 65535) return 0;
    a.slice_chunks = (a.Qtot + *slices - 1) / *slices;
    int V;
    pick_lanes(a.slice_chunks, &a.L, &V);
    a.tile_j = bev::row::kTileJ;
    a.tiles_i = (grid->X + bev::row::kTileI - 1) / bev::row::kTileI;
    a.tiles_j = (grid->Y + bev::row::kTileJ - 1) / bev::row::kTileJ;
    a.out_vec = (grid->Y % 4) == 0;
    return V;
}

// Channel slices of the dense kernels: each lane of a warp owns cpl
// consecutive channels, so a CTA covers 32 * cpl channels of the Cp padded
// channels per texel (4-, 8- or 16-byte loads per lane).  Fills a.cpl and
// a.cpad and returns the number of slices.
int channel_slices(bev::SampleArgs& a, bool bf16, int Cp) {
    a.cpl = bf16 ? (Cp <= 64 ? 2 : 4) : (Cp <= 32 ? 1 : Cp <= 64 ? 2 : 4);
    a.cpad = Cp;
    return (Cp + 32 * a.cpl - 1) / (32 * a.cpl);
}

// 8x8 tiles of the grid.
void tile_grid(bev::SampleArgs& a, const bev_grid_t* grid) {
    a.tiles_i = (grid->X + bev::kTileI - 1) / bev::kTileI;
    a.tiles_j = (grid->Y + bev::kTileJ - 1) / bev::kTileJ;
}

// A single-level table: the level is the feature map itself.
void single_level(bev::SampleArgs& a, int Hf, int Wf, int img_h, int img_w) {
    a.lv.n = 1;
    a.lv.Hf[0] = Hf;
    a.lv.Wf[0] = Wf;
    a.lv.sW[0] = (float)Wf / (float)img_w;
    a.lv.sH[0] = (float)Hf / (float)img_h;
}

}  // namespace

BEV_API int bev_bounds_checked(void) {
#ifdef BEV_BOUNDS_CHECK
    return 1;
#else
    return 0;
#endif
}

BEV_API const char* bev_status_string(int status) {
    switch (status) {
        case BEV_OK: return "ok";
        case BEV_ERR_INVALID_ARG: return "invalid argument";
        case BEV_ERR_UNSUPPORTED: return "unsupported request";
        case BEV_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
        case BEV_ERR_CUDA: return "CUDA runtime error";
        case BEV_ERR_INTERNAL: return "internal consistency check failed";
        default: return "unknown status";
    }
}

BEV_API int bev_grid_spec(const float range[6], const float res[3], bev_grid_t* out) {
    if (!range || !res || !out) return BEV_ERR_INVALID_ARG;
    int counts[3];
    float cell[3];
    for (int a = 0; a < 3; ++a) {
        const float lo = range[2 * a], hi = range[2 * a + 1], r = res[a];
        if (!isfinite(lo) || !isfinite(hi) || !isfinite(r) || !(hi > lo) || !(r > 0.0f))
            return BEV_ERR_INVALID_ARG;
        const float extent = hi - lo;
        const double q = (double)extent / (double)r;
        const double k = nearbyint(q);
        const int limit = a == 2 ? BEV_MAX_Z : BEV_MAX_DIM;
        if (fabs(q - k) > 1e-4 || k < 1.0 || k > (double)limit) return BEV_ERR_INVALID_ARG;
        counts[a] = (int)k;
        cell[a] = extent / (float)counts[a];
    }
    out->X = counts[0];
    out->Y = counts[1];
    out->Z = counts[2];
    out->xmin = range[0];
    out->xmax = range[1];
    out->ymin = range[2];
    out->ymax = range[3];
    out->zmin = range[4];
    out->zmax = range[5];
    out->dx = cell[0];
    out->dy = cell[1];
    out->dz = cell[2];
    return BEV_OK;
}

BEV_API size_t bev_workspace_size(int dtype, int layout, int B, int N, int C, int Hf, int Wf,
                                  int for_backward) {
    if (!dims_ok(B, N, C, Hf, Wf)) return (size_t)-1;
    if (for_backward) return backward_ws(B, N, C, Hf, Wf);
    if ((dtype != BEV_F32 && dtype != BEV_BF16) || (layout != BEV_NCHW && layout != BEV_NHWC))
        return (size_t)-1;
    return forward_ws(dtype, layout, B, N, C, Hf, Wf);
}

BEV_API int bev_sample_forward(const void* features, int dtype, int layout, int B, int N, int C, int Hf,
                               int Wf, const float* intrinsics, const float* ego2cam, int img_h,
                               int img_w, const bev_grid_t* grid, float* out, uint8_t* valid_count,
                               void* workspace, size_t workspace_bytes, bev_stream_t stream) {
    // host-only checks first: nothing below touches CUDA until these pass
    if (!features || !intrinsics || !ego2cam || !out || !grid) return BEV_ERR_INVALID_ARG;
    if (!dims_ok(B, N, C, Hf, Wf) || !grid_ok(grid)) return BEV_ERR_INVALID_ARG;
    if (img_h < 1 || img_w < 1 || img_h > BEV_MAX_DIM || img_w > BEV_MAX_DIM) return BEV_ERR_INVALID_ARG;
    if (dtype != BEV_F32 && dtype != BEV_BF16) return BEV_ERR_UNSUPPORTED;
    if (layout != BEV_NCHW && layout != BEV_NHWC) return BEV_ERR_UNSUPPORTED;
    const bool repack = needs_repack(dtype, layout, C);
    const size_t ws_need = forward_ws(dtype, layout, B, N, C, Hf, Wf);
    if (ws_need > 0 && (!workspace || workspace_bytes < ws_need || ((uintptr_t)workspace % kAlign) != 0))
        return BEV_ERR_WORKSPACE;
    if (!repack && ((uintptr_t)features % 16) != 0) return BEV_ERR_INVALID_ARG;

    int dev;
    int st = current_device(&dev);
    if (st != BEV_OK) return st;
    const void* ptrs[5] = {features, intrinsics, ego2cam, out, valid_count};
    for (int k = 0; k < 5; ++k) {
        if (k == 4 && !valid_count) continue;
        if ((st = device_ptr(ptrs[k], dev)) != BEV_OK) return st;
    }
    if (ws_need > 0 && (st = device_ptr(workspace, dev)) != BEV_OK) return BEV_ERR_WORKSPACE;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int cpc = chan_per_chunk(dtype);
    const int Cp = round_up(C, cpc);
    const void* feat = features;
    if (repack) {
        st = cuda_status(bev_launch_to_channels_last(features, layout, elem_size(dtype), B * N, C,
                                                     Hf * Wf, Cp, workspace, s));
        if (st != BEV_OK) return st;
        feat = workspace;
    }
    bev::row::SampleArgs a;
    memset(&a, 0, sizeof(a));
    a.feat = feat;
    a.K = intrinsics;
    a.E = ego2cam;
    a.out = out;
    a.count = valid_count;
    a.g = geo(grid, Hf, Wf, img_h, img_w);
    a.B = B;
    a.N = N;
    a.C = C;
    int slices;
    const int V = row_layout(a, Cp, cpc, grid, &slices);
    if (V == 0) return BEV_ERR_UNSUPPORTED;
    a.out_vec = a.out_vec && ((uintptr_t)out % 16) == 0;
    return dense_status(bev_launch_forward_rows(a, dtype == BEV_BF16, V, slices, s), s,
                        BEV_TAKE(bev_launch_forward_rows_check_take));
}

BEV_API int bev_sample_backward(const float* dout, int B, int N, int C, int Hf, int Wf,
                                const float* intrinsics, const float* ego2cam, int img_h, int img_w,
                                const bev_grid_t* grid, float* dfeatures, void* workspace,
                                size_t workspace_bytes, bev_stream_t stream) {
    if (!dout || !intrinsics || !ego2cam || !dfeatures || !grid) return BEV_ERR_INVALID_ARG;
    if (!dims_ok(B, N, C, Hf, Wf) || !grid_ok(grid)) return BEV_ERR_INVALID_ARG;
    if (img_h < 1 || img_w < 1 || img_h > BEV_MAX_DIM || img_w > BEV_MAX_DIM) return BEV_ERR_INVALID_ARG;
    const size_t ws_need = backward_ws(B, N, C, Hf, Wf);
    if (!workspace || workspace_bytes < ws_need || ((uintptr_t)workspace % kAlign) != 0)
        return BEV_ERR_WORKSPACE;

    int dev;
    int st = current_device(&dev);
    if (st != BEV_OK) return st;
    const void* ptrs[4] = {dout, intrinsics, ego2cam, dfeatures};
    for (int k = 0; k < 4; ++k)
        if ((st = device_ptr(ptrs[k], dev)) != BEV_OK) return st;
    if (device_ptr(workspace, dev) != BEV_OK) return BEV_ERR_WORKSPACE;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int Cp = round_up(C, 4);
    if ((st = cuda_status(cudaMemsetAsync(workspace, 0, ws_need, s))) != BEV_OK) return st;
    bev::SampleArgs a;
    memset(&a, 0, sizeof(a));
    a.K = intrinsics;
    a.E = ego2cam;
    a.dout = dout;
    a.g = geo(grid, Hf, Wf, img_h, img_w);
    a.B = B;
    a.N = N;
    a.C = C;
    single_level(a, Hf, Wf, img_h, img_w);
    a.lv.grad[0] = static_cast<float*>(workspace);
    a.out_vec = ((uintptr_t)dout % 16) == 0 && (grid->Y % 4) == 0;
    const int slices = channel_slices(a, false, Cp);
    tile_grid(a, grid);
    if ((st = dense_status(bev_launch_backward(a, slices, s), s, BEV_TAKE(bev_backward_check_take))) != BEV_OK)
        return st;
    return cuda_status(bev_launch_to_nchw(static_cast<const float*>(workspace), B * N, C, Hf * Wf, Cp,
                                          dfeatures, s));
}

BEV_API int bev_features_to_channels_last(const void* features, int dtype, int B, int N, int C, int Hf,
                                          int Wf, void* out, bev_stream_t stream) {
    if (!features || !out) return BEV_ERR_INVALID_ARG;
    if (!dims_ok(B, N, C, Hf, Wf)) return BEV_ERR_INVALID_ARG;
    if (dtype != BEV_F32 && dtype != BEV_BF16) return BEV_ERR_UNSUPPORTED;
    int dev;
    int st = current_device(&dev);
    if (st != BEV_OK) return st;
    if ((st = device_ptr(features, dev)) != BEV_OK) return st;
    if ((st = device_ptr(out, dev)) != BEV_OK) return st;
    return cuda_status(bev_launch_to_channels_last(features, BEV_NCHW, elem_size(dtype), B * N, C, Hf * Wf,
                                                   C, out, reinterpret_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------------------
// Multi-scale dense Sampling-VT
// ---------------------------------------------------------------------------

namespace {

static_assert(bev::kMaxLevels == BEV_MAX_LEVELS, "level table size");

bool levels_ok(int nlevels, const int* Hf, const int* Wf, int B, int N, int C) {
    if (nlevels < 1 || nlevels > BEV_MAX_LEVELS || !Hf || !Wf) return false;
    for (int l = 0; l < nlevels; ++l)
        if (!dims_ok(B, N, C, Hf[l], Wf[l])) return false;
    return true;
}

// Byte offset of level l's region in the workspace (each region 256-byte
// aligned) and the total: forward = the channels-last copies, backward = the
// fp32 channels-last gradient buffers.
size_t ms_ws(int dtype, int layout, int B, int N, int C, int nlevels, const int* Hf, const int* Wf,
             int for_backward, size_t* offsets) {
    size_t total = 0;
    for (int l = 0; l < nlevels; ++l) {
        if (offsets) offsets[l] = total;
        total += for_backward ? backward_ws(B, N, C, Hf[l], Wf[l]) : forward_ws(dtype, layout, B, N, C, Hf[l], Wf[l]);
    }
    return total;
}

template <class Table>
Table level_table(int nlevels, const int* Hf, const int* Wf, int img_h, int img_w) {
    Table t;
    memset(&t, 0, sizeof(t));
    t.n = nlevels;
    for (int l = 0; l < nlevels; ++l) {
        t.Hf[l] = Hf[l];
        t.Wf[l] = Wf[l];
        t.sW[l] = (float)Wf[l] / (float)img_w;
        t.sH[l] = (float)Hf[l] / (float)img_h;
    }
    return t;
}

}  // namespace

BEV_API size_t bev_multiscale_workspace_size(int dtype, int layout, int B, int N, int C, int nlevels,
                                             const int* Hf, const int* Wf, int for_backward) {
    if (!levels_ok(nlevels, Hf, Wf, B, N, C)) return (size_t)-1;
    if (!for_backward &&
        ((dtype != BEV_F32 && dtype != BEV_BF16) || (layout != BEV_NCHW && layout != BEV_NHWC)))
        return (size_t)-1;
    return ms_ws(dtype, layout, B, N, C, nlevels, Hf, Wf, for_backward, nullptr);
}

BEV_API int bev_sample_forward_multiscale(const void* const* features, int nlevels, const int* Hf, const int* Wf,
                                          int dtype, int layout, int B, int N, int C, const float* intrinsics,
                                          const float* ego2cam, int img_h, int img_w, const bev_grid_t* grid,
                                          float* out, uint8_t* valid_count, void* workspace,
                                          size_t workspace_bytes, bev_stream_t stream) {
    if (!features || !intrinsics || !ego2cam || !out || !grid) return BEV_ERR_INVALID_ARG;
    if (!levels_ok(nlevels, Hf, Wf, B, N, C) || !grid_ok(grid)) return BEV_ERR_INVALID_ARG;
    for (int l = 0; l < nlevels; ++l)
        if (!features[l]) return BEV_ERR_INVALID_ARG;
    if (img_h < 1 || img_w < 1 || img_h > BEV_MAX_DIM || img_w > BEV_MAX_DIM) return BEV_ERR_INVALID_ARG;
    if (dtype != BEV_F32 && dtype != BEV_BF16) return BEV_ERR_UNSUPPORTED;
    if (layout != BEV_NCHW && layout != BEV_NHWC) return BEV_ERR_UNSUPPORTED;
    const bool repack = needs_repack(dtype, layout, C);
    size_t off[BEV_MAX_LEVELS];
    const size_t ws_need = ms_ws(dtype, layout, B, N, C, nlevels, Hf, Wf, 0, off);
    if (ws_need > 0 && (!workspace || workspace_bytes < ws_need || ((uintptr_t)workspace % kAlign) != 0))
        return BEV_ERR_WORKSPACE;
    for (int l = 0; l < nlevels; ++l)
        if (!repack && ((uintptr_t)features[l] % 16) != 0) return BEV_ERR_INVALID_ARG;

    int dev;
    int st = current_device(&dev);
    if (st != BEV_OK) return st;
    const void* ptrs[4] = {intrinsics, ego2cam, out, valid_count};
    for (int k = 0; k < 4; ++k) {
        if (k == 3 && !valid_count) continue;
        if ((st = device_ptr(ptrs[k], dev)) != BEV_OK) return st;
    }
    for (int l = 0; l < nlevels; ++l)
        if ((st = device_ptr(features[l], dev)) != BEV_OK) return st;
    if (ws_need > 0 && (st = device_ptr(workspace, dev)) != BEV_OK) return BEV_ERR_WORKSPACE;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int cpc = chan_per_chunk(dtype);
    const int Cp = round_up(C, cpc);
    const void* base[BEV_MAX_LEVELS];
    for (int l = 0; l < nlevels; ++l) {
        base[l] = features[l];
        if (repack) {
            void* dst = static_cast<unsigned char*>(workspace) + off[l];
            st = cuda_status(bev_launch_to_channels_last(features[l], layout, elem_size(dtype), B * N, C,
                                                         Hf[l] * Wf[l], Cp, dst, s));
            if (st != BEV_OK) return st;
            base[l] = dst;
        }
    }
    bev::row::SampleArgs a;
    memset(&a, 0, sizeof(a));
    a.feat = base[0];
    a.K = intrinsics;
    a.E = ego2cam;
    a.out = out;
    a.count = valid_count;
    a.g = geo(grid, Hf[0], Wf[0], img_h, img_w);
    a.lv = level_table<bev::row::LevelTable>(nlevels, Hf, Wf, img_h, img_w);
    for (int l = 0; l < nlevels; ++l) a.lv.feat[l] = base[l];
    a.B = B;
    a.N = N;
    a.C = C;
    int slices;
    const int V = row_layout(a, Cp, cpc, grid, &slices);
    if (V == 0) return BEV_ERR_UNSUPPORTED;
    a.out_vec = a.out_vec && ((uintptr_t)out % 16) == 0;
    return dense_status(bev_launch_forward_rows_ms(a, dtype == BEV_BF16, V, slices, s), s,
                        BEV_TAKE(bev_launch_forward_rows_ms_check_take));
}

BEV_API int bev_sample_backward_multiscale(const float* dout, int nlevels, const int* Hf, const int* Wf, int B,
                                           int N, int C, const float* intrinsics, const float* ego2cam, int img_h,
                                           int img_w, const bev_grid_t* grid, float* const* dfeatures,
                                           void* workspace, size_t workspace_bytes, bev_stream_t stream) {
    if (!dout || !intrinsics || !ego2cam || !dfeatures || !grid) return BEV_ERR_INVALID_ARG;
    if (!levels_ok(nlevels, Hf, Wf, B, N, C) || !grid_ok(grid)) return BEV_ERR_INVALID_ARG;
    for (int l = 0; l < nlevels; ++l)
        if (!dfeatures[l]) return BEV_ERR_INVALID_ARG;
    if (img_h < 1 || img_w < 1 || img_h > BEV_MAX_DIM || img_w > BEV_MAX_DIM) return BEV_ERR_INVALID_ARG;
    size_t off[BEV_MAX_LEVELS];
    const size_t ws_need = ms_ws(BEV_F32, BEV_NCHW, B, N, C, nlevels, Hf, Wf, 1, off);
    if (!workspace || workspace_bytes < ws_need || ((uintptr_t)workspace % kAlign) != 0)
        return BEV_ERR_WORKSPACE;

    int dev;
    int st = current_device(&dev);
    if (st != BEV_OK) return st;
    const void* ptrs[3] = {dout, intrinsics, ego2cam};
    for (int k = 0; k < 3; ++k)
        if ((st = device_ptr(ptrs[k], dev)) != BEV_OK) return st;
    for (int l = 0; l < nlevels; ++l)
        if ((st = device_ptr(dfeatures[l], dev)) != BEV_OK) return st;
    if (device_ptr(workspace, dev) != BEV_OK) return BEV_ERR_WORKSPACE;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int Cp = round_up(C, 4);
    if ((st = cuda_status(cudaMemsetAsync(workspace, 0, ws_need, s))) != BEV_OK) return st;
    float* base[BEV_MAX_LEVELS];
    for (int l = 0; l < nlevels; ++l) base[l] = reinterpret_cast<float*>(static_cast<unsigned char*>(workspace) + off[l]);
    bev::SampleArgs a;
    memset(&a, 0, sizeof(a));
    a.K = intrinsics;
    a.E = ego2cam;
    a.dout = dout;
    a.g = geo(grid, Hf[0], Wf[0], img_h, img_w);
    a.lv = level_table<bev::LevelTable>(nlevels, Hf, Wf, img_h, img_w);
    for (int l = 0; l < nlevels; ++l) a.lv.grad[l] = base[l];
    a.out_vec = ((uintptr_t)dout % 16) == 0 && (grid->Y % 4) == 0;
    a.B = B;
    a.N = N;
    a.C = C;
    const int slices = channel_slices(a, false, Cp);
    tile_grid(a, grid);
    if ((st = dense_status(bev_launch_backward(a, slices, s), s, BEV_TAKE(bev_backward_check_take))) != BEV_OK)
        return st;
    for (int l = 0; l < nlevels; ++l) {
        st = cuda_status(bev_launch_to_nchw(base[l], B * N, C, Hf[l] * Wf[l], Cp,
                                            dfeatures[l], s));
        if (st != BEV_OK) return st;
    }
    return BEV_OK;
}

// ---------------------------------------------------------------------------
// Deformable aggregation
// ---------------------------------------------------------------------------

namespace {

constexpr int kDeformMaxChunks = 128;  // 32 lanes x 4 chunks of 16 bytes

bool deform_dims_ok(int B, int N, int C, int Hf, int Wf, int Q, int Kp) {
    if (!dims_ok(B, N, C, Hf, Wf)) return false;
    if (Q < 1 || Q > (1 << 26) || Kp < 1 || Kp > BEV_DEFORM_MAX_KEYPOINTS) return false;
    return true;
}

// Channels-last fp32 gradient buffer of the backward: chunk channels per texel.
size_t deform_grad_bytes(int dtype, int B, int N, int C, int Hf, int Wf) {
    return (size_t)B * N * Hf * Wf * round_up(C, chan_per_chunk(dtype)) * sizeof(float);
}

size_t deform_ws(int dtype, int layout, int B, int N, int C, int Hf, int Wf, int for_backward) {
    const size_t rep = forward_ws(dtype, layout, B, N, C, Hf, Wf);
    if (!for_backward) return rep;
    return align_up(rep) + align_up(deform_grad_bytes(dtype, B, N, C, Hf, Wf));
}

bev::GeoParams deform_geo(int Hf, int Wf, int img_h, int img_w) {
    bev::GeoParams p;
    memset(&p, 0, sizeof(p));
    p.img_w = (float)img_w;
    p.img_h = (float)img_h;
    p.sW = (float)Wf / (float)img_w;
    p.sH = (float)Hf / (float)img_h;
    p.Hf = Hf;
    p.Wf = Wf;
    return p;
}

// Shared checks and set-up of both deformable calls: validates, repacks the
// features to channels-last when needed and fills the launch arguments.
int deform_prepare(const void* features, int dtype, int layout, int B, int N, int C, int Hf, int Wf,
                   const float* K, const float* E, int img_h, int img_w, const float* anchors,
                   const float* offsets, const float* weights, int Q, int Kp, void* workspace,
                   size_t workspace_bytes, int for_backward, const void* const* extra, int n_extra,
                   cudaStream_t s, bev::DeformArgs* a, int* V, int* dev_out) {
    if (!features || !K || !E || !anchors || !offsets || !weights) return BEV_ERR_INVALID_ARG;
    for (int k = 0; k < n_extra; ++k)
        if (!extra[k]) return BEV_ERR_INVALID_ARG;
    if (!deform_dims_ok(B, N, C, Hf, Wf, Q, Kp)) return BEV_ERR_INVALID_ARG;
    if (img_h < 1 || img_w < 1 || img_h > BEV_MAX_DIM || img_w > BEV_MAX_DIM) return BEV_ERR_INVALID_ARG;
    if (dtype != BEV_F32 && dtype != BEV_BF16) return BEV_ERR_UNSUPPORTED;
    if (layout != BEV_NCHW && layout != BEV_NHWC) return BEV_ERR_UNSUPPORTED;
    const int cpc = chan_per_chunk(dtype);
    const int Qtot = round_up(C, cpc) / cpc;
    if (Qtot > kDeformMaxChunks) return BEV_ERR_UNSUPPORTED;
    const bool repack = needs_repack(dtype, layout, C);
    const size_t ws_need = deform_ws(dtype, layout, B, N, C, Hf, Wf, for_backward);
    if (ws_need > 0 && (!workspace || workspace_bytes < ws_need || ((uintptr_t)workspace % kAlign) != 0))
        return BEV_ERR_WORKSPACE;
    if (!repack && ((uintptr_t)features % 16) != 0) return BEV_ERR_INVALID_ARG;

    int dev;
    int st = current_device(&dev);
    if (st != BEV_OK) return st;
    const void* ptrs[6] = {features, K, E, anchors, offsets, weights};
    for (int k = 0; k < 6; ++k)
        if ((st = device_ptr(ptrs[k], dev)) != BEV_OK) return st;
    for (int k = 0; k < n_extra; ++k)
        if ((st = device_ptr(extra[k], dev)) != BEV_OK) return st;
    if (ws_need > 0 && (st = device_ptr(workspace, dev)) != BEV_OK) return BEV_ERR_WORKSPACE;

    const void* feat = features;
    if (repack) {
        st = cuda_status(bev_launch_to_channels_last(features, layout, elem_size(dtype), B * N, C, Hf * Wf,
                                                     Qtot * cpc, workspace, s));
        if (st != BEV_OK) return st;
        feat = workspace;
    }
    memset(a, 0, sizeof(*a));
    a->feat = feat;
    a->K = K;
    a->E = E;
    a->anchors = anchors;
    a->offsets = offsets;
    a->weights = weights;
    a->g = deform_geo(Hf, Wf, img_h, img_w);
    a->B = B;
    a->N = N;
    a->C = C;
    a->Q = Q;
    a->Kp = Kp;
    a->Qtot = Qtot;
    a->chan_per_chunk = cpc;
    *V = (Qtot + 31) / 32;
    *dev_out = dev;
    return BEV_OK;
}

}  // namespace

BEV_API size_t bev_deform_workspace_size(int dtype, int layout, int B, int N, int C, int Hf, int Wf,
                                         int for_backward) {
    if (!dims_ok(B, N, C, Hf, Wf)) return (size_t)-1;
    if ((dtype != BEV_F32 && dtype != BEV_BF16) || (layout != BEV_NCHW && layout != BEV_NHWC))
        return (size_t)-1;
    return deform_ws(dtype, layout, B, N, C, Hf, Wf, for_backward);
}

BEV_API int bev_deform_forward(const void* features, int dtype, int layout, int B, int N, int C, int Hf, int Wf,
                               const float* intrinsics, const float* ego2cam, int img_h, int img_w,
                               const float* anchors, const float* offsets, const float* weights, int Q, int Kp,
                               float* out, void* workspace, size_t workspace_bytes, bev_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const void* extra[1] = {out};
    bev::DeformArgs a;
    int V, dev;
    int st = deform_prepare(features, dtype, layout, B, N, C, Hf, Wf, intrinsics, ego2cam, img_h, img_w, anchors,
                            offsets, weights, Q, Kp, workspace, workspace_bytes, 0, extra, 1, s, &a, &V, &dev);
    if (st != BEV_OK) return st;
    a.out = out;
    return cuda_status(bev_launch_deform_forward(a, dtype == BEV_BF16, V, s));
}

BEV_API int bev_deform_backward(const void* features, int dtype, int layout, int B, int N, int C, int Hf, int Wf,
                                const float* intrinsics, const float* ego2cam, int img_h, int img_w,
                                const float* anchors, const float* offsets, const float* weights, int Q, int Kp,
                                const float* dout, float* dfeatures, float* dweights, float* doffsets,
                                void* workspace, size_t workspace_bytes, bev_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const void* extra[4] = {dout, dfeatures, dweights, doffsets};
    bev::DeformArgs a;
    int V, dev;
    int st = deform_prepare(features, dtype, layout, B, N, C, Hf, Wf, intrinsics, ego2cam, img_h, img_w, anchors,
                            offsets, weights, Q, Kp, workspace, workspace_bytes, 1, extra, 4, s, &a, &V, &dev);
    if (st != BEV_OK) return st;
    const size_t rep = align_up(forward_ws(dtype, layout, B, N, C, Hf, Wf));
    float* grad = reinterpret_cast<float*>(static_cast<unsigned char*>(workspace) + rep);
    const size_t gbytes = deform_grad_bytes(dtype, B, N, C, Hf, Wf);
    if ((st = cuda_status(cudaMemsetAsync(grad, 0, gbytes, s))) != BEV_OK) return st;
    a.dout = dout;
    a.dfeat = grad;
    a.dweights = dweights;
    a.doffsets = doffsets;
    if ((st = cuda_status(bev_launch_deform_backward(a, dtype == BEV_BF16, V, s))) != BEV_OK) return st;
    return cuda_status(bev_launch_to_nchw(grad, B * N, C, Hf * Wf, a.Qtot * a.chan_per_chunk, dfeatures, s));
}

// ---------------------------------------------------------------------------
// Lift-splat BEV pooling
// ---------------------------------------------------------------------------

namespace {

bool lss_dims_ok(int B, int N, int D, int C, int Hf, int Wf, int X, int Y) {
    if (!dims_ok(B, N, C, Hf, Wf)) return false;
    if (D < 1 || D > 4096 || X < 1 || Y < 1 || X > BEV_MAX_DIM || Y > BEV_MAX_DIM) return false;
    return true;
}

size_t lss_ws(int B, int C, int X, int Y, int for_backward) {
    const size_t cells = (size_t)B * X * Y * C;
    if (for_backward) return align_up(cells * sizeof(float));
    return align_up(2 * sizeof(unsigned)) + align_up(cells * sizeof(unsigned long long));
}

int lss_prepare(const float* depth, const float* feat, int B, int N, int D, int C, int Hf, int Wf, const float* K,
                const float* E, int img_h, int img_w, float dmin, float dstep, const bev_grid_t* grid,
                void* workspace, size_t workspace_bytes, int for_backward, const void* const* extra, int n_extra,
                bev::LssArgs* a) {
    if (!depth || !feat || !K || !E || !grid) return BEV_ERR_INVALID_ARG;
    for (int k = 0; k < n_extra; ++k)
        if (!extra[k]) return BEV_ERR_INVALID_ARG;
    if (!grid_ok(grid)) return BEV_ERR_INVALID_ARG;
    if (!lss_dims_ok(B, N, D, C, Hf, Wf, grid->X, grid->Y)) return BEV_ERR_INVALID_ARG;
    if (img_h < 1 || img_w < 1 || img_h > BEV_MAX_DIM || img_w > BEV_MAX_DIM) return BEV_ERR_INVALID_ARG;
    if (!isfinite(dmin) || !isfinite(dstep) || !(dstep > 0.0f)) return BEV_ERR_INVALID_ARG;
    if (C > bev::kLssMaxChannels) return BEV_ERR_UNSUPPORTED;
    const size_t ws_need = lss_ws(B, C, grid->X, grid->Y, for_backward);
    if (!workspace || workspace_bytes < ws_need || ((uintptr_t)workspace % kAlign) != 0) return BEV_ERR_WORKSPACE;
    int dev;
    int st = current_device(&dev);
    if (st != BEV_OK) return st;
    const void* ptrs[4] = {depth, feat, K, E};
    for (int k = 0; k < 4; ++k)
        if ((st = device_ptr(ptrs[k], dev)) != BEV_OK) return st;
    for (int k = 0; k < n_extra; ++k)
        if ((st = device_ptr(extra[k], dev)) != BEV_OK) return st;
    if ((st = device_ptr(workspace, dev)) != BEV_OK) return BEV_ERR_WORKSPACE;
    memset(a, 0, sizeof(*a));
    a->depth = depth;
    a->feat = feat;
    a->K = K;
    a->E = E;
    a->B = B;
    a->N = N;
    a->D = D;
    a->C = C;
    a->Hf = Hf;
    a->Wf = Wf;
    a->X = grid->X;
    a->Y = grid->Y;
    a->sWi = (float)img_w / (float)Wf;
    a->sHi = (float)img_h / (float)Hf;
    a->dmin = dmin;
    a->dstep = dstep;
    a->xmin = grid->xmin;
    a->ymin = grid->ymin;
    a->zmin = grid->zmin;
    a->zmax = grid->zmax;
    a->dx = grid->dx;
    a->dy = grid->dy;
    a->points_per_batch = (long long)N * D * Hf * Wf;
    return BEV_OK;
}

}  // namespace

BEV_API size_t bev_lss_workspace_size(int B, int N, int C, int D, int Hf, int Wf, int X, int Y, int for_backward) {
    if (!lss_dims_ok(B, N, D, C, Hf, Wf, X, Y)) return (size_t)-1;
    return lss_ws(B, C, X, Y, for_backward);
}

BEV_API int bev_lss_forward(const float* depth, const float* feat, int B, int N, int D, int C, int Hf, int Wf,
                            const float* intrinsics, const float* ego2cam, int img_h, int img_w, float dmin,
                            float dstep, const bev_grid_t* grid, float* out, void* workspace,
                            size_t workspace_bytes, bev_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const void* extra[1] = {out};
    bev::LssArgs a;
    int st = lss_prepare(depth, feat, B, N, D, C, Hf, Wf, intrinsics, ego2cam, img_h, img_w, dmin, dstep, grid,
                         workspace, workspace_bytes, 0, extra, 1, &a);
    if (st != BEV_OK) return st;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    a.maxabs = reinterpret_cast<unsigned*>(ws);
    a.acc = reinterpret_cast<unsigned long long*>(ws + align_up(2 * sizeof(unsigned)));
    a.out = out;
    if ((st = cuda_status(cudaMemsetAsync(workspace, 0, lss_ws(B, C, a.X, a.Y, 0), s))) != BEV_OK) return st;
    return cuda_status(bev_launch_lss_forward(a, s));
}

BEV_API int bev_lss_backward(const float* depth, const float* feat, const float* dout, int B, int N, int D, int C,
                             int Hf, int Wf, const float* intrinsics, const float* ego2cam, int img_h, int img_w,
                             float dmin, float dstep, const bev_grid_t* grid, float* ddepth, float* dfeat,
                             void* workspace, size_t workspace_bytes, bev_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const void* extra[3] = {dout, ddepth, dfeat};
    bev::LssArgs a;
    int st = lss_prepare(depth, feat, B, N, D, C, Hf, Wf, intrinsics, ego2cam, img_h, img_w, dmin, dstep, grid,
                         workspace, workspace_bytes, 1, extra, 3, &a);
    if (st != BEV_OK) return st;
    float* dcl = static_cast<float*>(workspace);
    st = cuda_status(bev_launch_to_channels_last(dout, BEV_NCHW, 4, B, C, a.X * a.Y, C, dcl, s));
    if (st != BEV_OK) return st;
    a.dout_cl = dcl;
    a.ddepth = ddepth;
    a.dfeat = dfeat;
    return cuda_status(bev_launch_lss_backward(a, s));
}
