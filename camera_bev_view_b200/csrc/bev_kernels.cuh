// bev_kernels.cuh -- launch parameters shared by the host layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "bev_geometry.cuh"

namespace bev {

// BEV tile owned by one CTA: kTileI rows (ego x) by kTileJ columns (ego y).
// Warp w owns tile row w (kTileJ = 8 cells).
constexpr int kTileI = 8;
constexpr int kTileJ = 8;
constexpr int kTile = kTileI * kTileJ;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kCellsPerWarp = kTile / kWarps;
static_assert(kCellsPerWarp == kTileJ, "one warp per tile row");
// (fx, fy) slots per height chunk: kTile * active cameras * bins.
constexpr int kItemCap = 2048;
// Merged-weight patch entries per height chunk (fp32 each).
constexpr int kPatchCap = 4096;
// Height bins per chunk at most (valid counts are packed one byte per cell).
constexpr int kZChunkMax = 32;
// Channels per CTA slice (the output staging tile holds kTile x kSliceMax floats).
constexpr int kSliceMax = 128;
constexpr int kObufStride = kTile + 1;  // padded row of the [channel][cell] staging tile
// Shared-memory copy of one camera's texel window for the tile, in 16-byte chunks.
constexpr int kStageChunks = 2048;

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
    int tiles_i, tiles_j;   // tiles along X and Y
};

// Bytes of dynamic shared memory of one CTA (see carve_smem).
__host__ __device__ inline size_t sample_smem_bytes(int N) {
    size_t b = 0;
    b += sizeof(float2) * kItemCap;                      // geometry slots
    b += sizeof(float) * kPatchCap;                      // merged weights
    b += (size_t)16 * kStageChunks;                      // texel window copy
    b += sizeof(int) * (kTile / 4) * kZChunkMax;         // valid counts, one byte per (bin, cell)
    b += sizeof(int4) * kTile * N;                       // patch box per (cell, active camera)
    b += sizeof(int4) * 32;                              // texel window per active camera
    b += sizeof(float) * ((N * kCamFloats + 3) & ~3);    // camera constants
    b += sizeof(int) * 64;                               // active camera list, flags
    b += sizeof(int) * 64;                               // scan scratch
    return b;
}

// The backward adds a [channel][cell] staging tile of its upstream gradient.
__host__ __device__ inline size_t sample_smem_bytes_bwd(int N) {
    return sample_smem_bytes(N) + sizeof(float) * kSliceMax * kObufStride;
}

}  // namespace bev

// Launchers (defined next to their kernels); L lanes per cell, V chunks per lane.
cudaError_t bev_launch_forward(const bev::SampleArgs& a, bool bf16, int V, int slices,
                               cudaStream_t stream);
cudaError_t bev_launch_backward(const bev::SampleArgs& a, int V, int slices, cudaStream_t stream);
cudaError_t bev_launch_to_channels_last(const void* src, int layout, int esize, int BN, int C,
                                        int HW, int Cp, void* dst, cudaStream_t stream);
cudaError_t bev_launch_to_nchw(const float* src, int BN, int C, int HW, int Cp, float* dst,
                               cudaStream_t stream);
