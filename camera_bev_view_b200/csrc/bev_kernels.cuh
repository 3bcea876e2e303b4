// bev_kernels.cuh -- launch parameters shared by the host layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "bev_geometry.cuh"

namespace bev {

// BEV tile owned by one CTA: kTileI rows (ego x) by kTileJ columns (ego y).
// Warp w owns tile row w (kTileJ = 8 cells) and works on it on its own: after
// the CTA has staged the calibrations and culled the cameras, no CTA-wide
// barrier is needed.
constexpr int kTileI = 8;
constexpr int kTileJ = 8;
constexpr int kTile = kTileI * kTileJ;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kCellsPerWarp = kTile / kWarps;
static_assert(kCellsPerWarp == kTileJ && kWarps == kTileI, "one warp per tile row");
// Height bins a lane projects per chunk (chunk = lanes per cell * this).  The
// projections of a chunk stay in registers (two of them cached per cell
// group), and taller grids take more chunks.  The forward's accumulators
// already fill the register file: fp32 slices with eight or more lanes per
// cell take one bin per lane (two spill), bf16 slices and four-lane cells
// take two (one is slower there).  The backward, which holds dout instead,
// takes four.
template <bool BF16, int L>
constexpr int z_per_lane_fwd() { return (!BF16 && L >= 8) ? 1 : 2; }
constexpr int kZPerLaneBwd = 4;
constexpr int kZPerLaneMax = kZPerLaneBwd;
// Merged-weight entries of one warp for one (camera, height chunk): the
// patches of the cells the warp works on at once.  Each entry is an exact
// fixed-point sum split over two 32-bit words (see merge_patches).
constexpr int kWarpPatchCap = 512;
// Forward: merging the weights of one (cell group, camera) pays when the
// merged patch walk takes fewer steps (four texels of every lane's chunks)
// than the bins' corners unmerged, plus this margin for the merge itself.
// The backward always merges: there a step costs global reductions.
constexpr int kMergeStepsFwd = 0;
// Per-warp shared-memory region: the patch words, reused as the
// [channel][cell] staging tile of the warp's row (kSliceMax x kStageStride).
constexpr int kSliceMax = 128;
constexpr int kStageStride = kCellsPerWarp + 1;
constexpr int kWarpBytes = 2 * sizeof(int) * kWarpPatchCap;
static_assert((int)sizeof(float) * kSliceMax * kStageStride <= kWarpBytes + 512,
              "staging tile must fit the warp region");
// CTAs kept resident per SM; shared memory stays small (~34 KB) so that most
// of the SM's on-chip array serves as L1 for the tiles' texel windows.
constexpr int kCtasPerSm = 3;
// The backward holds dout instead of accumulators and fits more CTAs.
constexpr int kCtasPerSmBwd = 3;

// Feature-pyramid levels of the multi-scale operator.  Every level shares
// the voxel's projection, validity and count; level l samples its own map at
// its own scale.  The single-level kernels read g (Hf, Wf, sW, sH) and feat
// instead.
constexpr int kMaxLevels = 4;

struct LevelTable {
    int n;                            // levels, 1 .. kMaxLevels
    int Hf[kMaxLevels], Wf[kMaxLevels];
    float sW[kMaxLevels], sH[kMaxLevels];  // (float)W_l / img_w, (float)H_l / img_h, host IEEE divide
    const void* feat[kMaxLevels];     // forward: channels-last features of level l (16-byte chunks)
    float* grad[kMaxLevels];          // backward: fp32 channels-last gradient buffer of level l
};

struct SampleArgs {
    const void* feat;       // channels-last [B*N][Hf*Wf][Qtot chunks of 16 bytes]
    const float* K;         // [B,N,3,3]
    const float* E;         // [B,N,4,4]
    float* out;             // forward: [B,C,X,Y]
    uint8_t* count;         // forward: [B,X,Y,Z] or null
    const float* dout;      // backward: [B,C,X,Y]
    float* dfeat;           // backward: channels-last fp32 [B*N][Hf*Wf][Qtot*4]
    GeoParams g;
    int B, N, C;
    int Qtot;               // 16-byte chunks per texel in the channels-last buffer
    int chan_per_chunk;     // 4 (fp32) or 8 (bf16)
    int slice_chunks;       // chunks per CTA channel slice
    int L;                  // lanes per cell (4, 8, 16 or 32)
    int tile_j;             // cells per tile row: kTileJ (forward) or a multiple of 32 / L (backward)
    int tiles_i, tiles_j;   // tiles along X and Y
    int cam_split;          // forward: two CTAs per tile, each gathering every other camera
    LevelTable lv;          // multi-scale kernels only
};

// Bytes of dynamic shared memory of one CTA (see carve_smem).
// Byte offsets of the per-CTA shared-memory regions (one source of truth for
// the kernels' carve-up and the launch size).
struct SmemLayout {
    size_t warps, cams, act, total;
};

__host__ __device__ inline SmemLayout smem_layout(int N) {
    SmemLayout l;
    size_t b = 0;
    l.warps = b;  b += (size_t)kWarps * (kWarpBytes + 512);           // per-warp patch / staging regions
    l.cams = b;   b += sizeof(float) * ((N * kCamFloats + 3) & ~3);   // camera constants
    l.act = b;    b += sizeof(int) * 128;                             // active cameras, tile slot, flags
    l.total = b;
    return l;
}

__host__ __device__ inline size_t sample_smem_bytes(int N) { return smem_layout(N).total; }

// Preferred shared-memory carveout for `ctas` CTAs of `smem` bytes each:
// the smallest shared-memory configuration of the SM (KB) that holds them,
// as a percentage of the 228 KB maximum; the rest of the array is L1.
inline int carveout_percent(size_t smem, int ctas = kCtasPerSm) {
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

// Launchers (defined next to their kernels); L lanes per cell, V chunks per lane.
cudaError_t bev_launch_forward(const bev::SampleArgs& a, bool bf16, int V, int slices,
                               cudaStream_t stream);
cudaError_t bev_launch_backward(const bev::SampleArgs& a, int V, int slices, cudaStream_t stream);
// Multi-scale forms (a.lv describes the levels).
cudaError_t bev_launch_forward_ms(const bev::SampleArgs& a, bool bf16, int V, int slices,
                                  cudaStream_t stream);
cudaError_t bev_launch_backward_ms(const bev::SampleArgs& a, int V, int slices, cudaStream_t stream);
cudaError_t bev_launch_to_channels_last(const void* src, int layout, int esize, int BN, int C,
                                        int HW, int Cp, void* dst, cudaStream_t stream);
cudaError_t bev_launch_to_nchw(const float* src, int BN, int C, int HW, int Cp, float* dst,
                               cudaStream_t stream);
