// bev_backward.cu -- gradient of the exact dense Sampling-VT with respect to
// the features (sm_100a).
//
// The forward is linear in F, so dL/dF is its adjoint (FlashBEV reading notes,
// "Method" item 4: forward and backward differ from the materialised form only
// by floating-point order):
//   dF[b, n, c, y, x] += w * dout[b, c, i, j] / cnt_k
// for every valid (cell, bin, camera) sample and every in-range bilinear corner
// (y, x) it touches.
//
// One CTA = one 8x8 BEV tile of one batch item and one channel slice, with the
// same culling and once-per-voxel geometry as the forward.  The tile's dout
// slice is staged in shared memory (coalesced along y); each lane then owns V
// chunks of 4 channels of one cell and scatters w / cnt * dout into the fp32
// channels-last gradient buffer with 16-byte vector reductions
// (red.global.add.v4.f32), one per (corner, chunk).
#include "bev_tile.cuh"

namespace bev {

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
                 "f"(d)
                 : "memory");
}

template <int V>
__global__ void __launch_bounds__(kThreads) sample_backward_kernel(const SampleArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const TileSmem s = carve_smem(smem_raw, a.N);
    const GeoParams& g = a.g;

    const int b = blockIdx.y;
    const int ti0 = (blockIdx.x / a.tiles_j) * kTileI;
    const int tj0 = (blockIdx.x % a.tiles_j) * kTileJ;
    const int chunk0 = blockIdx.z * a.slice_chunks;
    const int nchunks = min(a.slice_chunks, a.Qtot - chunk0);
    const int cs = nchunks * 4;
    const int c_base = chunk0 * 4;

    // stage dout[b, c_base + c, tile] as [c][cell]; padding channels read as 0
    for (int t = threadIdx.x; t < cs * kTile; t += kThreads) {
        const int c = t / kTile, cell = t - c * kTile;
        const int i = ti0 + cell / kTileJ, j = tj0 + cell % kTileJ;
        float v = 0.0f;
        if (c_base + c < a.C && i < g.X && j < g.Y)
            v = a.dout[(((size_t)b * a.C + c_base + c) * g.X + i) * g.Y + j];
        s.obuf[c * kObufStride + cell] = v;
    }
    setup_tile(a, s, b, ti0, tj0);
    const int nA = s.act[32];
    if (nA == 0) return;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = a.L, G = 32 / L;
    const int sub = lane / L, ql = lane - sub * L;
    const int zc = z_chunk(g.Z, nA);
    const size_t texels = (size_t)g.Hf * g.Wf;
    const int tstride = a.Qtot * 4;  // floats per texel in the gradient buffer

    for (int z0 = 0; z0 < g.Z; z0 += zc) {
        const int zlen = min(zc, g.Z - z0);
        geometry_chunk(a, s, ti0, tj0, nA, z0, zlen);
        for (int cg = warp; cg * G < kTile; cg += kWarps) {
            const int cell = cg * G + sub;
            float d[V][4];
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const int q = ql + v * L;
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    d[v][e] = q < nchunks ? s.obuf[(q * 4 + e) * kObufStride + cell] : 0.0f;
            }
            for (int aa = 0; aa < nA; ++aa) {
                const int n = s.act[aa];
                float* Gn = a.dfeat + ((size_t)b * a.N + n) * texels * tstride + (size_t)(chunk0 + ql) * 4;
                const float2* it = s.items + (cell * nA + aa) * zlen;
                const int* cn = s.cnt + cell * zlen;
                for (int zl = 0; zl < zlen; ++zl) {
                    const float2 f = it[zl];
                    if (!(f.x == f.x)) continue;
                    const float sc = __frcp_rn((float)cn[zl]);
                    const Corners c = bilinear_corners(f.x, f.y);
                    const int ys[4] = {c.y0, c.y0, c.y0 + 1, c.y0 + 1};
                    const int xs[4] = {c.x0, c.x0 + 1, c.x0, c.x0 + 1};
                    const float ws[4] = {c.w00 * sc, c.w01 * sc, c.w10 * sc, c.w11 * sc};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        if ((unsigned)ys[k] >= (unsigned)g.Hf || (unsigned)xs[k] >= (unsigned)g.Wf) continue;
                        float* p = Gn + ((size_t)ys[k] * g.Wf + xs[k]) * tstride;
#pragma unroll
                        for (int v = 0; v < V; ++v) {
                            if (ql + v * L < nchunks)
                                red_add_v4(p + v * L * 4, ws[k] * d[v][0], ws[k] * d[v][1],
                                           ws[k] * d[v][2], ws[k] * d[v][3]);
                        }
                    }
                }
            }
        }
    }
}

static cudaError_t launch_bwd_v(const SampleArgs& a, int V, dim3 grid, size_t smem, cudaStream_t st) {
    switch (V) {
#define BEV_BWD_CASE(VV)                                                                        \
    case VV: {                                                                                  \
        auto k = sample_backward_kernel<VV>;                                                    \
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,    \
                                             (int)smem);                                        \
        if (e != cudaSuccess) return e;                                                         \
        k<<<grid, kThreads, smem, st>>>(a);                                                     \
        return cudaGetLastError();                                                              \
    }
        BEV_BWD_CASE(1)
        BEV_BWD_CASE(2)
        BEV_BWD_CASE(3)
        BEV_BWD_CASE(4)
        BEV_BWD_CASE(5)
        BEV_BWD_CASE(6)
        BEV_BWD_CASE(7)
        BEV_BWD_CASE(8)
#undef BEV_BWD_CASE
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace bev

cudaError_t bev_launch_backward(const bev::SampleArgs& a, int V, int slices, cudaStream_t stream) {
    const int tiles_i = (a.g.X + bev::kTileI - 1) / bev::kTileI;
    const dim3 grid(tiles_i * a.tiles_j, a.B, slices);
    return bev::launch_bwd_v(a, V, grid, bev::sample_smem_bytes(a.N), stream);
}
