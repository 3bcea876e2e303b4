// bev_forward_rows_ms.cu -- multi-scale forward launcher (kernel in bev_forward_rows.cuh).
#include "bev_forward_rows.cuh"

#ifdef BEV_BOUNDS_CHECK
unsigned bev_launch_forward_rows_ms_check_take() { return bev::row::check_take(); }
#endif

cudaError_t bev_launch_forward_rows_ms(const bev::row::SampleArgs& a, bool bf16, int V, int slices, cudaStream_t stream) {
    const dim3 grid(a.tiles_i * a.tiles_j, a.B, slices);
    const size_t smem = bev::row::sample_smem_bytes(a.N);
    return bf16 ? bev::row::launch_fwd_bf16<true>(a, V, grid, smem, stream)
                : bev::row::launch_fwd_f32<true>(a, V, grid, smem, stream);
}
