// bev_backward.cu -- gradient of the exact dense Sampling-VT with respect to
// the features (sm_100a).
//
// The forward is linear in F, so dL/dF is its adjoint (FlashBEV reading notes,
// "Method" item 4: forward and backward differ from the materialised form only
// by floating-point order):
//   dF[b, n, c, y, x] += (sum_k w_k / cnt_k) * dout[b, c, i, j]
// over every (cell, camera) and every texel (y, x) its valid samples touch.
//
// One CTA = one 8x8 BEV tile of one batch item and one channel slice, with the
// same culling, once-per-voxel geometry and merged per-(cell, camera, texel)
// weights as the forward (bev_tile.cuh).  The tile's dout slice is staged in
// shared memory (coalesced along y) and held in registers: each lane owns V
// chunks of 4 channels of one cell.  Each touched texel then receives one
// 16-byte vector reduction per chunk (red.global.add.v4.f32) into the fp32
// channels-last gradient buffer, however many height bins hit it.
#include "bev_tile.cuh"

namespace bev {

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
                 "f"(d)
                 : "memory");
}

template <int L, int V>
__device__ __forceinline__ void scatter_texel(float* p, const float (&d)[V][4], float w, int ql,
                                              int nchunks) {
#pragma unroll
    for (int v = 0; v < V; ++v)
        if (ql + v * L < nchunks)
            red_add_v4(p + v * L * 4, w * d[v][0], w * d[v][1], w * d[v][2], w * d[v][3]);
}

template <int L, int V>
__device__ __forceinline__ void scatter_patch(const float (&d)[V][4], const float* pf, const int4 pi,
                                              float* Gn, int Wf, int tstride, int ql, int nchunks) {
    const int h = pi.z >> 16, w = pi.z & 0xffff;
    const float* pw = pf + pi.w;
    float* grow = Gn + ((size_t)pi.x * Wf + pi.y) * tstride;
    for (int r = 0; r < h; ++r, grow += (size_t)Wf * tstride, pw += w) {
        for (int cc = 0; cc < w; ++cc) {
            const float wt = pw[cc];
            if (wt != 0.0f) scatter_texel<L, V>(grow + (size_t)cc * tstride, d, wt, ql, nchunks);
        }
    }
}

template <int L, int V>
__device__ __forceinline__ void scatter_direct(const float (&d)[V][4], const TileSmem& s, int cell, int aa,
                                               int zlen, float* Gn, int Hf, int Wf, int tstride, int ql,
                                               int nchunks) {
    for (int zl = 0; zl < zlen; ++zl) {
        const float2 f = s.items[item_index(cell, aa, zl, zlen)];
        if (!(f.x == f.x)) continue;
        const float cntf = (float)cell_count(s.cnt, zl, cell);
        const Corners c = bilinear_corners(f.x, f.y);
        const float ws[4] = {c.w00, c.w01, c.w10, c.w11};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int yy = c.y0 + (k >> 1), xx = c.x0 + (k & 1);
            if ((unsigned)yy >= (unsigned)Hf || (unsigned)xx >= (unsigned)Wf) continue;
            scatter_texel<L, V>(Gn + ((size_t)yy * Wf + xx) * tstride, d, __fdiv_rn(ws[k], cntf), ql, nchunks);
        }
    }
}

template <int L, int V>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) sample_backward_kernel(const SampleArgs a) {
    constexpr int G = 32 / L;
    constexpr int CG = kCellsPerWarp / G;
    static_assert(G * CG == kCellsPerWarp, "lanes per cell must be 4, 8, 16 or 32");
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const TileSmem s = carve_smem(smem_raw, a.N);
    const GeoParams& g = a.g;

    const int b = blockIdx.y;
    int ti0, tj0;
    tile_origin(a, s.act + 40, ti0, tj0);
    const int chunk0 = blockIdx.z * a.slice_chunks;
    const int nchunks = min(a.slice_chunks, a.Qtot - chunk0);
    const int c_base = chunk0 * 4;

    setup_tile(a, s, b, ti0, tj0);
    const int nA = s.act[32];
    if (nA == 0) return;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / L, ql = lane - sub * L;
    // Upstream gradient of the tile into registers, kGroupCh channels at a time
    // through the [channel][cell] staging tile (loads coalesced along y).
    float d[CG][V][4];
#pragma unroll
    for (int q = 0; q < CG; ++q)
#pragma unroll
        for (int v = 0; v < V; ++v)
#pragma unroll
            for (int e = 0; e < 4; ++e) d[q][v][e] = 0.0f;
    for (int g0 = 0; g0 < nchunks * 4; g0 += kGroupCh) {
        __syncthreads();
        for (int t = threadIdx.x; t < kGroupCh * kTile; t += kThreads) {
            const int c = t / kTile, cell = t - c * kTile;
            const int i = ti0 + cell / kTileJ, j = tj0 + cell % kTileJ;
            float v = 0.0f;
            if (g0 + c < nchunks * 4 && c_base + g0 + c < a.C && i < g.X && j < g.Y)
                v = a.dout[(((size_t)b * a.C + c_base + g0 + c) * g.X + i) * g.Y + j];
            s.obuf[c * kObufStride + cell] = v;
        }
        __syncthreads();
#pragma unroll
        for (int q = 0; q < CG; ++q) {
            const int cell = warp * kCellsPerWarp + q * G + sub;
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const int c0 = (ql + v * L) * 4 - g0;
                if (c0 >= 0 && c0 < kGroupCh) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) d[q][v][e] = s.obuf[(c0 + e) * kObufStride + cell];
                }
            }
        }
    }
    const size_t texels = (size_t)g.Hf * g.Wf;
    const int tstride = a.Qtot * 4;  // floats per texel in the gradient buffer
    float* grad = a.dfeat + (size_t)(chunk0 + ql) * 4;

    int zc = z_chunk(g.Z, nA);
    int z0 = 0;
    while (z0 < g.Z) {
        const int zlen = min(zc, g.Z - z0);
        geometry_chunk(a, s, ti0, tj0, nA, z0, zlen);
        int total = layout_patches(a, s, zlen, 0, nA);
        if (total < 0 && zlen > 1) {  // too many texels: fewer bins per chunk
            zc = (zlen + 1) / 2;
            continue;
        }
        int a0 = 0, ga = nA;
        while (a0 < nA) {
            const int a1 = min(nA, a0 + ga);
            if (a0 > 0 || a1 < nA) total = layout_patches(a, s, zlen, a0, a1);
            if (total < 0 && a1 - a0 > 1) {  // still too many: fewer cameras at once
                ga = (a1 - a0 + 1) / 2;
                continue;
            }
            if (total >= 0) fill_patches(a, s, zlen, a0, a1);
            const float* pf = s.patch;
#pragma unroll
            for (int q = 0; q < CG; ++q) {
                const int cell = warp * kCellsPerWarp + q * G + sub;
                for (int aa = a0; aa < a1; ++aa) {
                    float* Gn = grad + ((size_t)b * a.N + s.act[aa]) * texels * tstride;
                    if (total >= 0)
                        scatter_patch<L, V>(d[q], pf, s.pinfo[aa * kTile + cell], Gn, g.Wf, tstride, ql, nchunks);
                    else
                        scatter_direct<L, V>(d[q], s, cell, aa, zlen, Gn, g.Hf, g.Wf, tstride, ql, nchunks);
                }
            }
            __syncthreads();
            a0 = a1;
            total = -1;
        }
        z0 += zlen;
    }
}

template <int L, int V>
static cudaError_t launch_one(const SampleArgs& a, dim3 grid, size_t smem, cudaStream_t st) {
    auto k = sample_backward_kernel<L, V>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, carveout_percent(smem));
    if (e != cudaSuccess) return e;
    k<<<grid, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

static cudaError_t launch_bwd(const SampleArgs& a, int V, dim3 grid, size_t smem, cudaStream_t st) {
    switch (a.L * 16 + V) {
        case 32 * 16 + 1: return launch_one<32, 1>(a, grid, smem, st);
        case 16 * 16 + 1: return launch_one<16, 1>(a, grid, smem, st);
        case 16 * 16 + 2: return launch_one<16, 2>(a, grid, smem, st);
        case 8 * 16 + 1: return launch_one<8, 1>(a, grid, smem, st);
        case 8 * 16 + 2: return launch_one<8, 2>(a, grid, smem, st);
        case 8 * 16 + 3: return launch_one<8, 3>(a, grid, smem, st);
        case 8 * 16 + 4: return launch_one<8, 4>(a, grid, smem, st);
        case 4 * 16 + 1: return launch_one<4, 1>(a, grid, smem, st);
        case 4 * 16 + 2: return launch_one<4, 2>(a, grid, smem, st);
        case 4 * 16 + 3: return launch_one<4, 3>(a, grid, smem, st);
        case 4 * 16 + 4: return launch_one<4, 4>(a, grid, smem, st);
        case 4 * 16 + 5: return launch_one<4, 5>(a, grid, smem, st);
        case 4 * 16 + 6: return launch_one<4, 6>(a, grid, smem, st);
        case 4 * 16 + 7: return launch_one<4, 7>(a, grid, smem, st);
        case 4 * 16 + 8: return launch_one<4, 8>(a, grid, smem, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace bev

cudaError_t bev_launch_backward(const bev::SampleArgs& a, int V, int slices, cudaStream_t stream) {
    const dim3 grid(a.tiles_i * a.tiles_j, a.B, slices);
    return bev::launch_bwd(a, V, grid, bev::sample_smem_bytes(a.N), stream);
}
