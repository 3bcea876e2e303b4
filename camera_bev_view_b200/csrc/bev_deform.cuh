// bev_deform.cuh -- launch parameters of the deformable-aggregation kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "bev_geometry.cuh"

namespace bev {

// Keypoints per query the kernels accept (per-warp shared-memory accumulator
// of the offset gradient).
constexpr int kDeformMaxKeypoints = 64;
// One CTA per query; its warps split the query's (camera, keypoint) pairs.
constexpr int kDeformWarps = 4;

struct DeformArgs {
    const void* feat;       // channels-last [B*N][Hf*Wf][Qtot chunks of 16 bytes]
    const float* K;         // [B,N,3,3]
    const float* E;         // [B,N,4,4]
    const float* anchors;   // [B,Q,3]
    const float* offsets;   // [B,Q,Kp,3]
    const float* weights;   // [B,Q,N,Kp]
    const float* dout;      // backward: [B,Q,C]
    float* out;             // forward: [B,Q,C]
    float* dfeat;           // backward: channels-last fp32 [B*N][Hf*Wf][Qtot * chan_per_chunk]
    float* dweights;        // backward: [B,Q,N,Kp]
    float* doffsets;        // backward: [B,Q,Kp,3]
    GeoParams g;
    int B, N, C, Q, Kp;
    int Qtot;               // 16-byte feature chunks per texel
    int chan_per_chunk;     // 4 (fp32) or 8 (bf16)
};

// Shared memory of one CTA: calibrations, then per warp either the partial
// sums of the forward (C floats) or the offset-gradient accumulator of the
// backward (Kp x 3 floats).
inline size_t deform_smem_bytes(int N, int C, int Kp) {
    const size_t per_warp = (size_t)((C > Kp * 3 ? C : Kp * 3) + 3) & ~(size_t)3;
    return sizeof(float) * (((size_t)N * kCamFloats + 3) / 4 * 4 + (size_t)kDeformWarps * per_warp);
}

}  // namespace bev

// Launchers (bev_deform.cu); V = feature chunks per lane (1..4).
cudaError_t bev_launch_deform_forward(const bev::DeformArgs& a, bool bf16, int V, cudaStream_t stream);
cudaError_t bev_launch_deform_backward(const bev::DeformArgs& a, bool bf16, int V, cudaStream_t stream);
