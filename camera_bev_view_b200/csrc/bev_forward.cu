// bev_forward.cu -- single-level forward launcher (kernel in bev_forward.cuh).
#include "bev_forward.cuh"

cudaError_t bev_launch_forward(const bev::SampleArgs& a, bool bf16, int V, int slices,
                               cudaStream_t stream) {
    const dim3 grid(a.tiles_i * a.tiles_j * (a.cam_split ? 2 : 1), a.B, slices);
    const size_t smem = bev::sample_smem_bytes(a.N);
    return bf16 ? bev::launch_fwd_bf16<false>(a, V, grid, smem, stream)
                : bev::launch_fwd_f32<false>(a, V, grid, smem, stream);
}
