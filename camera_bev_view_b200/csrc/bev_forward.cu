// bev_forward.cu -- fused forward of the exact dense Sampling-VT (sm_100a).
//
// out[b, c, i, j] = sum_k [cnt_k > 0] (1 / cnt_k) sum_{valid n} sum_l bilinear(F_l[b, n, c], fx_l, fy_l)
// (FlashBEV reading notes, "Method" items 1-2: per-bin valid mean over
// cameras, then a sum over height, in one kernel with nothing intermediate in
// HBM; with one level l this is the single-level operator, with several it is
// the multi-scale fused form of "Takeaway" 4).
//
// One CTA = one 8x8 BEV tile of one batch item and one channel slice of 32 *
// CPL channels (the tile machinery of bev_tile.cuh).  Each lane owns CPL
// consecutive channels.  A warp sweeps one group of cells at a time: per
// texel of the group's union box it loads the lane's channels once (a
// 4-32-byte load from the channels-last features, through L1) and the
// group's merged weights once (one shared-memory vector load, broadcast), and
// accumulates every member cell in fp32 registers with packed FMAs.  The
// group's sums are added into the CTA's [cell][channel] output tile; after
// the last camera the tile is stored along y, the contiguous axis of out.
#include "bev_tile.cuh"

namespace bev {

// Sweep of one group's union box, two rows by two columns per step.
template <bool BF16, int CPL, int G>
__device__ __forceinline__ void gather_group(float (&acc)[G][CPL], const Group& gp, const float* wf,
                                             const unsigned char* fl, size_t rowb, int tb, bool on) {
    constexpr int S = G == 1 ? 1 : G == 2 ? 2 : G <= 4 ? 4 : 8;
    const int h = gp.h, w = gp.w;
    const float* wb = wf + gp.off;
    const unsigned char* fb = fl + (size_t)gp.y0 * rowb + (size_t)gp.x0 * tb;
    for (int c0 = 0; c0 < w; c0 += 2) {
        const bool c1 = c0 + 1 < w;
        const unsigned char* p = fb + (size_t)c0 * tb;
        const float* q = wb + c0 * S;
        for (int r0 = 0; r0 < h; r0 += 2, p += 2 * rowb, q += 2 * w * S) {
            const bool r1 = r0 + 1 < h;
            const bool in[4] = {true, c1, r1, r1 && c1};
            LaneVec<BF16, CPL> d[4];
            float wt[4][S];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (in[u]) {
                    load_weights<S>(wt[u], q + ((u >> 1) * w + (u & 1)) * S);
                } else {
#pragma unroll
                    for (int k = 0; k < S; ++k) wt[u][k] = 0.0f;
                }
                if (in[u] && on)
                    d[u].load(p + (u >> 1) * rowb + (u & 1) * tb);
                else
                    d[u].zero();
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float v[CPL];
#pragma unroll
                for (int c = 0; c < CPL; ++c) v[c] = d[u].get(c);
#pragma unroll
                for (int gg = 0; gg < G; ++gg) fma_lane<CPL>(acc[gg], wt[u][gg], v);
            }
        }
    }
}

// Add a lane's channels of one cell into the output tile.
template <int CPL>
__device__ __forceinline__ void add_to_tile(float* t, const float (&v)[CPL]) {
    if constexpr (CPL == 4) {
        float4 o = *reinterpret_cast<float4*>(t);
        o.x += v[0]; o.y += v[1]; o.z += v[2]; o.w += v[3];
        *reinterpret_cast<float4*>(t) = o;
    } else if constexpr (CPL == 2) {
        float2 o = *reinterpret_cast<float2*>(t);
        o.x += v[0]; o.y += v[1];
        *reinterpret_cast<float2*>(t) = o;
    } else {
        t[0] += v[0];
    }
}

template <bool BF16, int CPL, int G>
__device__ __forceinline__ void forward_group(const TileSm& s, const Group& gp, const unsigned char* fl, size_t rowb,
                                              int tb, bool on, int lane) {
    float acc[G][CPL];
#pragma unroll
    for (int gg = 0; gg < G; ++gg)
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[gg][c] = 0.0f;
    gather_group<BF16, CPL, G>(acc, gp, s.wf, fl, rowb, tb, on);
    if (on) {
#pragma unroll
        for (int gg = 0; gg < G; ++gg) add_to_tile<CPL>(s.tile + gp.cell[gg] * s.tile_stride + lane * CPL, acc[gg]);
    }
}

// A group too large to merge: each member cell's valid bins, corner by
// corner, with weight w / cnt.
template <bool BF16, int CPL>
__device__ __noinline__ void forward_direct(const TileSm& s, int gi, int zc, int Hl, int Wl, float sW,
                                            float sH, const unsigned char* fl, size_t rowb, int tb, bool on,
                                            int lane) {
    const Group& gp = s.grp[gi];
    for (int m = 0; m < gp.n; ++m) {
        const int cell = gp.cell[m];
        float acc[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[c] = 0.0f;
        for (int zz = 0; zz < zc; ++zz) {
            const float2 uv = s.uv[cell * kZc + zz];
            if (isnan(uv.x)) continue;
            float fx, fy;
            level_position(uv, sW, sH, fx, fy);
            const Corners c = bilinear_corners(fx, fy);
            const float rc = s.rc[cell * kZc + zz];
            const float ws[4] = {c.w00, c.w01, c.w10, c.w11};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int yy = c.y0 + (k >> 1), xx = c.x0 + (k & 1);
                if ((unsigned)yy >= (unsigned)Hl || (unsigned)xx >= (unsigned)Wl) continue;
                LaneVec<BF16, CPL> d;
                if (on)
                    d.load(fl + (size_t)yy * rowb + (size_t)xx * tb);
                else
                    d.zero();
                float v[CPL];
#pragma unroll
                for (int q = 0; q < CPL; ++q) v[q] = d.get(q);
                fma_lane<CPL>(acc, __fmul_rn(ws[k], rc), v);
            }
        }
        if (on) add_to_tile<CPL>(s.tile + cell * s.tile_stride + lane * CPL, acc);
    }
}

// Warps take the groups of round r in turn until none is left.
template <bool BF16, int CPL>
__device__ __forceinline__ void sweep_forward(const TileSm& s, int r, int zc, int Hl, int Wl, float sW, float sH,
                                              const unsigned char* fl, size_t rowb, int tb, bool on, int lane) {
    const int rend = s.ctl[kCtlRstart + r + 1];
    for (;;) {
        int gi = 0;
        if (lane == 0) gi = atomicAdd(&s.ctl[kCtlNext], 1);
        gi = __shfl_sync(0xffffffffu, gi, 0);
        if (gi >= rend) break;
        const Group gp = s.grp[gi];
        if (gp.direct) {
            forward_direct<BF16, CPL>(s, gi, zc, Hl, Wl, sW, sH, fl, rowb, tb, on, lane);
            continue;
        }
        switch (gp.n) {
            case 1: forward_group<BF16, CPL, 1>(s, gp, fl, rowb, tb, on, lane); break;
            case 2: forward_group<BF16, CPL, 2>(s, gp, fl, rowb, tb, on, lane); break;
            case 3: forward_group<BF16, CPL, 3>(s, gp, fl, rowb, tb, on, lane); break;
            case 4: forward_group<BF16, CPL, 4>(s, gp, fl, rowb, tb, on, lane); break;
            case 5: forward_group<BF16, CPL, 5>(s, gp, fl, rowb, tb, on, lane); break;
            case 6: forward_group<BF16, CPL, 6>(s, gp, fl, rowb, tb, on, lane); break;
            case 7: forward_group<BF16, CPL, 7>(s, gp, fl, rowb, tb, on, lane); break;
            default: forward_group<BF16, CPL, 8>(s, gp, fl, rowb, tb, on, lane); break;
        }
    }
}

// The level table is indexed at run time: __grid_constant__ lets the body
// read it in place from the parameter space.
template <bool BF16, int CPL>
__global__ void __launch_bounds__(kThreads, kTileCtas) sample_forward_kernel(const __grid_constant__ SampleArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const TileSm s = carve_tile(smem_raw, a.N, CPL);
    const GeoParams& g = a.g;
    const int b = blockIdx.y;
    const int c_base = blockIdx.z * 32 * CPL;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int esize = BF16 ? 2 : 4;

    for (int e = threadIdx.x; e < kEntries; e += kThreads) s.wq[e] = 0ull;
    for (int e = threadIdx.x; e < kCells * s.tile_stride; e += kThreads) s.tile[e] = 0.0f;
    int ti0, tj0;
    locate_tile(a, s, b, ti0, tj0);
    cull_cameras(a, s, ti0, tj0);
    const int nA = s.ctl[kCtlNA];
    const bool on = c_base + lane * CPL < a.cpad;
    const bool write_count = a.count != nullptr && blockIdx.z == 0;
    const int tb = a.texel_bytes;

    for (int z0 = 0; z0 < g.Z; z0 += kZc) {
        const int zc = min(kZc, g.Z - z0);
        count_pass(a, s, b, ti0, tj0, z0, zc, write_count);
        __syncthreads();
        for (int aa = 0; aa < nA; ++aa) {
            project_pass(a, s, ti0, tj0, z0, zc, aa);
            __syncthreads();
            const int cam = s.ctl[kCtlActive + aa];
            for (int l = 0; l < a.lv.n; ++l) {
                const int Hl = a.lv.Hf[l], Wl = a.lv.Wf[l];
                const float sW = a.lv.sW[l], sH = a.lv.sH[l];
                box_pass(s, zc, Hl, Wl, sW, sH);
                __syncthreads();
                if (warp == 0) form_groups(s);
                __syncthreads();
                const int nr = s.ctl[kCtlRounds];
                const size_t rowb = (size_t)Wl * tb;
                const unsigned char* fl = static_cast<const unsigned char*>(a.lv.feat[l]) +
                                          ((size_t)b * a.N + cam) * Hl * rowb + (size_t)(c_base + lane * CPL) * esize;
                for (int r = 0; r < nr; ++r) {
                    merge_pass(s, zc, Hl, Wl, sW, sH, r);
                    __syncthreads();
                    convert_pass(s, r);
                    if (threadIdx.x == 0) s.ctl[kCtlNext] = s.ctl[kCtlRstart + r];
                    __syncthreads();
                    sweep_forward<BF16, CPL>(s, r, zc, Hl, Wl, sW, sH, fl, rowb, tb, on, lane);
                }
                __syncthreads();
            }
        }
    }
    __syncthreads();

    // Store: each thread takes (channel, tile row) pairs and writes the row's
    // 8 cells along y (two 16-byte stores where out allows).
    const int nch = min(32 * CPL, a.C - c_base);
    for (int idx = threadIdx.x; idx < nch * kTileI; idx += kThreads) {
        const int ci = idx / nch, c = idx - ci * nch;
        const int i = ti0 + ci;
        if (i >= g.X) continue;
        const float* tp = s.tile + ci * kTileJ * s.tile_stride + c;
        float v[kTileJ];
#pragma unroll
        for (int cj = 0; cj < kTileJ; ++cj) v[cj] = tp[cj * s.tile_stride];
        float* op = a.out + (((size_t)b * a.C + c_base + c) * g.X + i) * g.Y + tj0;
        if (a.out_vec && tj0 + kTileJ <= g.Y) {
            *reinterpret_cast<float4*>(op) = make_float4(v[0], v[1], v[2], v[3]);
            *reinterpret_cast<float4*>(op + 4) = make_float4(v[4], v[5], v[6], v[7]);
        } else {
#pragma unroll
            for (int cj = 0; cj < kTileJ; ++cj)
                if (tj0 + cj < g.Y) op[cj] = v[cj];
        }
    }
}

template <bool BF16, int CPL>
static cudaError_t launch(const SampleArgs& a, dim3 grid, cudaStream_t st) {
    const size_t smem = tile_layout(a.N, CPL).total;
    static std::atomic<long long> attrs[kAttrDevices];
    const cudaError_t e = set_smem_attributes(sample_forward_kernel<BF16, CPL>, smem,
                                              carveout_percent(smem, kTileCtas), attrs);
    if (e != cudaSuccess) return e;
    sample_forward_kernel<BF16, CPL><<<grid, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace bev

cudaError_t bev_launch_forward(const bev::SampleArgs& a, bool bf16, int slices, cudaStream_t stream) {
    const dim3 grid(a.tiles_i * a.tiles_j, a.B, slices);
    if (bf16) {
        switch (a.cpl) {
            case 2: return bev::launch<true, 2>(a, grid, stream);
            case 4: return bev::launch<true, 4>(a, grid, stream);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (a.cpl) {
        case 1: return bev::launch<false, 1>(a, grid, stream);
        case 2: return bev::launch<false, 2>(a, grid, stream);
        case 4: return bev::launch<false, 4>(a, grid, stream);
        default: return cudaErrorInvalidValue;
    }
}
