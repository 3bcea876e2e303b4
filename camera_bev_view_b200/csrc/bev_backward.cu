// bev_backward.cu -- single-level backward launcher (kernel in bev_backward.cuh).
#include "bev_backward.cuh"

cudaError_t bev_launch_backward(const bev::SampleArgs& a, int V, int slices, cudaStream_t stream) {
    const dim3 grid(a.tiles_i * a.tiles_j, a.B, slices);
    return bev::launch_bwd<false>(a, V, grid, bev::sample_smem_bytes(a.N), stream);
}
