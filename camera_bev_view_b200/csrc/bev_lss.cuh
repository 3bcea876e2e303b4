// bev_lss.cuh -- launch parameters of the lift-splat pooling kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace bev {

// Warps per pixel in the backward (they split its depth bins).
constexpr int kLssWarps = 4;
// Channels per call: 32 lanes x 8 channels per lane.
constexpr int kLssMaxChannels = 256;

struct LssArgs {
    const float* depth;           // [B,N,D,Hf,Wf]
    const float* feat;            // [B,N,C,Hf,Wf]
    const float* K;               // [B,N,3,3]
    const float* E;               // [B,N,4,4]
    float* out;                   // forward: [B,C,X,Y]
    unsigned long long* acc;      // forward: fixed-point sums, channels-last [B][X*Y][C]
    unsigned* maxabs;             // forward: {max|depth|, max|feat|} as float bits
    const float* dout_cl;         // backward: channels-last dout [B][X*Y][C]
    float* ddepth;                // backward: [B,N,D,Hf,Wf]
    float* dfeat;                 // backward: [B,N,C,Hf,Wf]
    int B, N, D, C, Hf, Wf, X, Y;
    float sWi, sHi;               // (float)img_w / Wf, (float)img_h / Hf (host IEEE divides)
    float dmin, dstep;
    float xmin, ymin, zmin, zmax, dx, dy;
    long long points_per_batch;   // N * D * Hf * Wf
    int bins_per_cta;             // forward: depth bins per CTA (1, 2, 4 or 8), set by the launcher
};

}  // namespace bev

cudaError_t bev_launch_lss_forward(const bev::LssArgs& a, cudaStream_t stream);
cudaError_t bev_launch_lss_backward(const bev::LssArgs& a, cudaStream_t stream);
