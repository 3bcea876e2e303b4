// bev_deform.cuh -- launch parameters of the deformable-aggregation kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "bev_geometry.cuh"

namespace bev {

// Keypoints per query the kernels accept (per-warp shared-memory accumulator
// of the offset gradient).
constexpr int kDeformMaxKeypoints = 64;
// Queries per CTA: one warp each.
constexpr int kDeformWarps = 8;

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
    int vec_out;            // forward: C % chan_per_chunk == 0 and out 16-byte aligned
};

inline size_t deform_smem_bytes(int N) {
    return sizeof(float) * ((size_t)N * kCamFloats + (size_t)kDeformWarps * kDeformMaxKeypoints * 3);
}

}  // namespace bev

// Launchers (bev_deform.cu); V = feature chunks per lane (1..4).
cudaError_t bev_launch_deform_forward(const bev::DeformArgs& a, bool bf16, int V, cudaStream_t stream);
cudaError_t bev_launch_deform_backward(const bev::DeformArgs& a, bool bf16, int V, cudaStream_t stream);
