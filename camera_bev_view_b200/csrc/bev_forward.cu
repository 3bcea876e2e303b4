// bev_forward.cu -- fused forward of the exact dense Sampling-VT (sm_100a).
//
// out[b, c, i, j] = sum_k [cnt_k > 0] (1 / cnt_k) sum_{valid n} bilinear(F[b, n, c], fx, fy)
// (FlashBEV reading notes, "Method" items 1-2: per-bin valid mean over cameras,
// then a sum over height, in one kernel with nothing intermediate in HBM).
//
// One CTA = one 8x8 BEV tile of one batch item and one channel slice.
//   1. camera constants to shared memory; cameras that cannot see the tile
//      are culled (conservative box test);
//   2. per chunk of height bins: (fx, fy) of every (cell, active camera, bin)
//      and the per-(cell, bin) valid count, computed once, in shared memory;
//   3. each warp takes G = 32 / L cells at a time; the L lanes of a cell sweep
//      the channel slice with 16-byte loads from the channels-last feature
//      buffer (V chunks per lane) and accumulate w / cnt * F in fp32 registers;
//   4. the per-cell partial sums are folded into a [channel][cell] staging tile
//      in shared memory, which is finally stored along y (the contiguous axis
//      of out) in coalesced rows.
#include "bev_tile.cuh"

namespace bev {

template <bool BF16>
struct Chunk;

template <>
struct Chunk<false> {
    static constexpr int kCh = 4;
    __device__ __forceinline__ static void fma(float (&acc)[4], const uint4& d, float w) {
        acc[0] = fmaf(w, __uint_as_float(d.x), acc[0]);
        acc[1] = fmaf(w, __uint_as_float(d.y), acc[1]);
        acc[2] = fmaf(w, __uint_as_float(d.z), acc[2]);
        acc[3] = fmaf(w, __uint_as_float(d.w), acc[3]);
    }
};

template <>
struct Chunk<true> {
    static constexpr int kCh = 8;
    // bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32 word.
    __device__ __forceinline__ static void fma(float (&acc)[8], const uint4& d, float w) {
        acc[0] = fmaf(w, __uint_as_float(d.x << 16), acc[0]);
        acc[1] = fmaf(w, __uint_as_float(d.x & 0xffff0000u), acc[1]);
        acc[2] = fmaf(w, __uint_as_float(d.y << 16), acc[2]);
        acc[3] = fmaf(w, __uint_as_float(d.y & 0xffff0000u), acc[3]);
        acc[4] = fmaf(w, __uint_as_float(d.z << 16), acc[4]);
        acc[5] = fmaf(w, __uint_as_float(d.z & 0xffff0000u), acc[5]);
        acc[6] = fmaf(w, __uint_as_float(d.w << 16), acc[6]);
        acc[7] = fmaf(w, __uint_as_float(d.w & 0xffff0000u), acc[7]);
    }
};

template <bool BF16, int V>
__global__ void __launch_bounds__(kThreads) sample_forward_kernel(const SampleArgs a) {
    using CK = Chunk<BF16>;
    constexpr int CH = CK::kCh;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const TileSmem s = carve_smem(smem_raw, a.N);
    const GeoParams& g = a.g;

    const int b = blockIdx.y;
    const int ti0 = (blockIdx.x / a.tiles_j) * kTileI;
    const int tj0 = (blockIdx.x % a.tiles_j) * kTileJ;
    const int chunk0 = blockIdx.z * a.slice_chunks;
    const int nchunks = min(a.slice_chunks, a.Qtot - chunk0);
    const int cs = nchunks * CH;

    for (int t = threadIdx.x; t < cs * kObufStride; t += kThreads) s.obuf[t] = 0.0f;
    setup_tile(a, s, b, ti0, tj0);
    const int nA = s.act[32];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = a.L, G = 32 / L;
    const int sub = lane / L, ql = lane - sub * L;
    const bool write_count = a.count != nullptr && blockIdx.z == 0;

    if (nA == 0) {
        if (write_count) store_counts(a, nullptr, b, ti0, tj0, 0, g.Z);
    } else {
        const int zc = z_chunk(g.Z, nA);
        const size_t texels = (size_t)g.Hf * g.Wf;
        for (int z0 = 0; z0 < g.Z; z0 += zc) {
            const int zlen = min(zc, g.Z - z0);
            geometry_chunk(a, s, ti0, tj0, nA, z0, zlen);
            if (write_count) store_counts(a, s.cnt, b, ti0, tj0, z0, zlen);

            for (int cg = warp; cg * G < kTile; cg += kWarps) {
                const int cell = cg * G + sub;
                float acc[V][CH];
#pragma unroll
                for (int v = 0; v < V; ++v)
#pragma unroll
                    for (int e = 0; e < CH; ++e) acc[v][e] = 0.0f;

                for (int aa = 0; aa < nA; ++aa) {
                    const int n = s.act[aa];
                    const uint4* Fn = reinterpret_cast<const uint4*>(a.feat) +
                                      ((size_t)b * a.N + n) * texels * a.Qtot + chunk0 + ql;
                    const float2* it = s.items + (cell * nA + aa) * zlen;
                    const int* cn = s.cnt + cell * zlen;
                    for (int zl = 0; zl < zlen; ++zl) {
                        const float2 f = it[zl];
                        if (!(f.x == f.x)) continue;  // camera not valid for this voxel
                        const float sc = __frcp_rn((float)cn[zl]);
                        const Corners c = bilinear_corners(f.x, f.y);
                        const bool x0in = (unsigned)c.x0 < (unsigned)g.Wf;
                        const bool x1in = (unsigned)(c.x0 + 1) < (unsigned)g.Wf;
                        const bool y0in = (unsigned)c.y0 < (unsigned)g.Hf;
                        const bool y1in = (unsigned)(c.y0 + 1) < (unsigned)g.Hf;
                        const uint4* p00 = Fn + ((long long)c.y0 * g.Wf + c.x0) * a.Qtot;
                        const size_t row = (size_t)g.Wf * a.Qtot;
#pragma unroll
                        for (int v = 0; v < V; ++v) {
                            if (ql + v * L < nchunks) {
                                const int o = v * L;
                                if (y0in && x0in) CK::fma(acc[v], __ldg(p00 + o), c.w00 * sc);
                                if (y0in && x1in) CK::fma(acc[v], __ldg(p00 + a.Qtot + o), c.w01 * sc);
                                if (y1in && x0in) CK::fma(acc[v], __ldg(p00 + row + o), c.w10 * sc);
                                if (y1in && x1in)
                                    CK::fma(acc[v], __ldg(p00 + row + a.Qtot + o), c.w11 * sc);
                            }
                        }
                    }
                }
                // fold into the staging tile; each (channel, cell) has exactly one owner lane
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    const int q = ql + v * L;
                    if (q < nchunks) {
#pragma unroll
                        for (int e = 0; e < CH; ++e) s.obuf[(q * CH + e) * kObufStride + cell] += acc[v][e];
                    }
                }
            }
        }
    }
    __syncthreads();
    const int c_base = chunk0 * CH;
    const int c_real = max(0, min(cs, a.C - c_base));
    for (int t = threadIdx.x; t < c_real * kTile; t += kThreads) {
        const int c = t / kTile, cell = t - c * kTile;
        const int i = ti0 + cell / kTileJ, j = tj0 + cell % kTileJ;
        if (i < g.X && j < g.Y)
            a.out[(((size_t)b * a.C + c_base + c) * g.X + i) * g.Y + j] = s.obuf[c * kObufStride + cell];
    }
}

template <bool BF16>
static cudaError_t launch_fwd_v(const SampleArgs& a, int V, dim3 grid, size_t smem, cudaStream_t st) {
    switch (V) {
#define BEV_FWD_CASE(VV)                                                                        \
    case VV: {                                                                                  \
        auto k = sample_forward_kernel<BF16, VV>;                                               \
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,    \
                                             (int)smem);                                        \
        if (e != cudaSuccess) return e;                                                         \
        k<<<grid, kThreads, smem, st>>>(a);                                                     \
        return cudaGetLastError();                                                              \
    }
        BEV_FWD_CASE(1)
        BEV_FWD_CASE(2)
        BEV_FWD_CASE(3)
        BEV_FWD_CASE(4)
        BEV_FWD_CASE(5)
        BEV_FWD_CASE(6)
        BEV_FWD_CASE(7)
        BEV_FWD_CASE(8)
#undef BEV_FWD_CASE
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace bev

cudaError_t bev_launch_forward(const bev::SampleArgs& a, bool bf16, int V, int slices,
                               cudaStream_t stream) {
    const int tiles_i = (a.g.X + bev::kTileI - 1) / bev::kTileI;
    const dim3 grid(tiles_i * a.tiles_j, a.B, slices);
    const size_t smem = bev::sample_smem_bytes(a.N);
    return bf16 ? bev::launch_fwd_v<true>(a, V, grid, smem, stream)
                : bev::launch_fwd_v<false>(a, V, grid, smem, stream);
}
