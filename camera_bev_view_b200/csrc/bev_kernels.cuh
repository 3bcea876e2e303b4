// bev_kernels.cuh -- launch parameters shared by the host layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "bev_geometry.cuh"

namespace bev {

// BEV tile owned by one CTA: kTileI rows (ego x) by kTileJ columns (ego y).
constexpr int kTileI = 8;
constexpr int kTileJ = 8;
constexpr int kTile = kTileI * kTileJ;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
// Per-(cell, camera, height-bin) geometry slots staged per z-chunk.
constexpr int kItemCap = 4096;
// Height bins per z-chunk at most (bounds the per-bin count table).
constexpr int kZChunkMax = 32;
// Channels per CTA slice (the output staging tile holds kTile x kSliceMax floats).
constexpr int kSliceMax = 128;
constexpr int kObufStride = kTile + 1;  // padded row of the [channel][cell] staging tile

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
    int L;                  // lanes per cell (power of two, divides 32)
    int tiles_j;            // tiles along Y
};

// Dynamic shared memory of one CTA.
inline size_t sample_smem_bytes(int N) {
    size_t b = 0;
    b += sizeof(float2) * kItemCap;                      // geometry slots
    b += sizeof(float) * kSliceMax * kObufStride;        // output/dout staging tile
    b += sizeof(int) * kTile * kZChunkMax;               // valid counts per (cell, bin)
    b += sizeof(float) * ((N * kCamFloats + 3) & ~3);    // camera constants
    b += sizeof(int) * 64;                               // active camera list
    return b;
}

}  // namespace bev

// Launchers (defined next to their kernels); V = chunks per lane.
cudaError_t bev_launch_forward(const bev::SampleArgs& a, bool bf16, int V, int slices,
                               cudaStream_t stream);
cudaError_t bev_launch_backward(const bev::SampleArgs& a, int V, int slices, cudaStream_t stream);
cudaError_t bev_launch_to_channels_last(const void* src, int layout, int esize, int BN, int C,
                                        int HW, int Cp, void* dst, cudaStream_t stream);
cudaError_t bev_launch_to_nchw(const float* src, int BN, int C, int HW, int Cp, float* dst,
                               cudaStream_t stream);
