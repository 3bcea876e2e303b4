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

// Sweep of one group's union box, two rows by two columns per step; weights
// [texel][member] with S per texel.  An even box needs no edge predicates;
// lanes past the slice's channels load channel 0 (harmless, never stored).
template <bool BF16, int CPL, int G, bool EVEN>
__device__ __forceinline__ void gather_walk(float (&acc)[G][CPL], const Members& m, const float* wb,
                                            const unsigned char* fl, size_t rowb, int tb) {
    constexpr int S = G == 1 ? 1 : G == 2 ? 2 : G <= 4 ? 4 : 8;
    const int h = m.h, w = m.w;
    const unsigned char* fb = fl + (size_t)m.y0 * rowb + (size_t)m.x0 * tb;
    for (int c0 = 0; c0 < w; c0 += 2) {
        const bool c1 = EVEN || c0 + 1 < w;
        const unsigned char* p = fb + (size_t)c0 * tb;
        const float* q = wb + c0 * S;
        if constexpr (EVEN && G * CPL <= 0) {
            // two rows by two columns per step; the next step's texels are
            // loaded before this step's FMAs, so two steps of loads are in
            // flight per warp (where the accumulators leave room for them)
            LaneVec<BF16, CPL> d[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) d[u].load(p + (u >> 1) * rowb + (u & 1) * tb);
            for (int r0 = 0; r0 < h; r0 += 2, p += 2 * rowb, q += 2 * w * S) {
                LaneVec<BF16, CPL> nx[4];
                if (r0 + 2 < h) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) nx[u].load(p + (2 + (u >> 1)) * rowb + (u & 1) * tb);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    float wt[S];
                    load_weights<S>(wt, q + ((u >> 1) * w + (u & 1)) * S);
                    float v[CPL];
#pragma unroll
                    for (int c = 0; c < CPL; ++c) v[c] = d[u].get(c);
#pragma unroll
                    for (int gg = 0; gg < G; ++gg) fma_lane<CPL>(acc[gg], wt[gg], v);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) d[u] = nx[u];
            }
        } else {
            for (int r0 = 0; r0 < h; r0 += 2, p += 2 * rowb, q += 2 * w * S) {
                const bool r1 = EVEN || r0 + 1 < h;
                const bool in[4] = {true, c1, r1, r1 && c1};
                LaneVec<BF16, CPL> d[4];
                float wt[4][S];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (in[u]) {
                        load_weights<S>(wt[u], q + ((u >> 1) * w + (u & 1)) * S);
                        d[u].load(p + (u >> 1) * rowb + (u & 1) * tb);
                    } else {
#pragma unroll
                        for (int k = 0; k < S; ++k) wt[u][k] = 0.0f;
                        d[u].zero();
                    }
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
}

template <bool BF16, int CPL, int G>
__device__ __forceinline__ void gather_members(float (&acc)[G][CPL], const Members& m, const float* wb,
                                               const unsigned char* fl, size_t rowb, int tb) {
    if (m.even)
        gather_walk<BF16, CPL, G, true>(acc, m, wb, fl, rowb, tb);
    else
        gather_walk<BF16, CPL, G, false>(acc, m, wb, fl, rowb, tb);
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
__device__ __forceinline__ void forward_group(const TileSm& s, const Members& m, const float* wb,
                                              const unsigned char* fl, size_t rowb, int tb, bool on, int lane) {
    float acc[G][CPL];
#pragma unroll
    for (int gg = 0; gg < G; ++gg)
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[gg][c] = 0.0f;
    gather_members<BF16, CPL, G>(acc, m, wb, fl, rowb, tb);
    if (on) {
#pragma unroll
        for (int gg = 0; gg < G; ++gg) add_to_tile<CPL>(s.tile + m.cell[gg] * s.tile_stride + lane * CPL, acc[gg]);
    }
}

// Merge the members' weights in the warp's region, sweep, clear the region.
template <bool BF16, int CPL>
__device__ __forceinline__ void forward_members(const TileSm& s, const Members& m, const GroupItems& it, int zc,
                                                int Hl, int Wl, float sW, float sH, const unsigned char* fl,
                                                size_t rowb, int tb, bool on, int lane, unsigned* wh, unsigned* wl) {
    merge_members(s, m, it, zc, Hl, Wl, sW, sH, wh, wl);
    const float* wb = reinterpret_cast<const float*>(wh);
    switch (m.n) {
        case 1: forward_group<BF16, CPL, 1>(s, m, wb, fl, rowb, tb, on, lane); break;
        case 2: forward_group<BF16, CPL, 2>(s, m, wb, fl, rowb, tb, on, lane); break;
        case 3: forward_group<BF16, CPL, 3>(s, m, wb, fl, rowb, tb, on, lane); break;
        case 4: forward_group<BF16, CPL, 4>(s, m, wb, fl, rowb, tb, on, lane); break;
        case 5: forward_group<BF16, CPL, 5>(s, m, wb, fl, rowb, tb, on, lane); break;
        case 6: forward_group<BF16, CPL, 6>(s, m, wb, fl, rowb, tb, on, lane); break;
        case 7: forward_group<BF16, CPL, 7>(s, m, wb, fl, rowb, tb, on, lane); break;
        default: forward_group<BF16, CPL, 8>(s, m, wb, fl, rowb, tb, on, lane); break;
    }
    clear_members(m, wh);
}

// A cell whose box does not fit a warp's region: its valid bins (lanes
// 0 .. zc-1 of `one`, a one-cell projection), corner by corner, with weight
// w / cnt.
template <bool BF16, int CPL>
__device__ __forceinline__ void forward_direct(const TileSm& s, const GroupItems& one, int cell, int zc, int Hl,
                                               int Wl, float sW, float sH, const unsigned char* fl, size_t rowb,
                                               int tb, bool on, int lane) {
    float acc[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[c] = 0.0f;
    for (int zz = 0; zz < zc; ++zz) {
        const float2 uv = make_float2(__shfl_sync(0xffffffffu, one.uv[0].x, zz), __shfl_sync(0xffffffffu, one.uv[0].y, zz));
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
            d.load(fl + (size_t)yy * rowb + (size_t)xx * tb);
            float v[CPL];
#pragma unroll
            for (int q = 0; q < CPL; ++q) v[q] = d.get(q);
            fma_lane<CPL>(acc, __fmul_rn(ws[k], rc), v);
        }
    }
    if (on) add_to_tile<CPL>(s.tile + cell * s.tile_stride + lane * CPL, acc);
}

// Warps take camera slot aa's groups in turn (largest first) until none is
// left; each group is projected once and swept on every level.
template <bool BF16, int CPL>
__device__ __forceinline__ void sweep_forward(const SampleArgs& a, const TileSm& s, int aa, int b, int ti0, int tj0,
                                              int z0, int zc, int lane_c, bool on, int lane, int warp) {
    constexpr int esize = BF16 ? 2 : 4;
    unsigned* wh = s.wqh + warp * kWarpEntries;
    unsigned* wl = s.wql + warp * kWarpEntries;
    const int ng = s.ctl[kCtlGroups];
    const int cam = s.ctl[kCtlActive + aa];
    const int tb = a.texel_bytes;
    for (;;) {
        int k = 0;
        if (lane == 0) k = atomicAdd(&s.ctl[kCtlNext], 1);
        k = __shfl_sync(0xffffffffu, k, 0);
        if (k >= ng) break;
        const Group& gp = s.grp[s.ctl[kCtlOrder + k]];
        if (!checked(gp.n >= 1 && gp.n <= kGmax, kCheckGroups)) continue;
        const GroupItems it = project_members(a, s, gp.cell, gp.n, cam, ti0, tj0, z0, zc);
        for (int l = 0; l < a.lv.n; ++l) {
            const int Hl = a.lv.Hf[l], Wl = a.lv.Wf[l];
            const float sW = a.lv.sW[l], sH = a.lv.sH[l];
            const size_t rowb = (size_t)Wl * tb;
            const unsigned char* fl = static_cast<const unsigned char*>(a.lv.feat[l]) +
                                      ((size_t)b * a.N + cam) * Hl * rowb + (size_t)lane_c * esize;
            const Members m = members_box(it, gp.cell, gp.n, Hl, Wl, sW, sH);
            if (!box_inside(m, Hl, Wl)) continue;
            if (m.entries <= kWarpEntries) {
                forward_members<BF16, CPL>(s, m, it, zc, Hl, Wl, sW, sH, fl, rowb, tb, on, lane, wh, wl);
                continue;
            }
            for (int q = 0; q < gp.n; ++q) {  // too large together: cell by cell
                const GroupItems one = project_members(a, s, gp.cell + q, 1, cam, ti0, tj0, z0, zc);
                const Members m1 = members_box(one, gp.cell + q, 1, Hl, Wl, sW, sH);
                if (!box_inside(m1, Hl, Wl)) continue;
                if (m1.entries <= kWarpEntries)
                    forward_members<BF16, CPL>(s, m1, one, zc, Hl, Wl, sW, sH, fl, rowb, tb, on, lane, wh, wl);
                else
                    forward_direct<BF16, CPL>(s, one, gp.cell[q], zc, Hl, Wl, sW, sH, fl, rowb, tb, on, lane);
            }
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

    for (int e = 4 * threadIdx.x; e < kWarps * kWarpEntries; e += 4 * kThreads) {
        *reinterpret_cast<uint4*>(s.wqh + e) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(s.wql + e) = make_uint4(0u, 0u, 0u, 0u);
    }
    for (int e = 4 * threadIdx.x; e < kCells * s.tile_stride; e += 4 * kThreads)
        *reinterpret_cast<float4*>(s.tile + e) = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    int ti0, tj0;
    locate_tile(a, s, b, ti0, tj0);
    cull_cameras(a, s, ti0, tj0);
    const int nA = s.ctl[kCtlNA];
    const bool on = c_base + lane * CPL < a.cpad;
    const int lane_c = on ? c_base + lane * CPL : c_base;  // lanes past the channels read channel c_base
    const bool write_count = a.count != nullptr && blockIdx.z == 0;

    for (int z0 = 0; z0 < g.Z; z0 += kZc) {
        const int zc = min(kZc, g.Z - z0);
        count_pass(a, s, b, ti0, tj0, z0, zc, write_count);
        __syncthreads();
        for (int aa = 0; aa < nA; ++aa) {
            if (warp == 0) form_groups(s, s.xlo + aa * kCells);
            __syncthreads();
            sweep_forward<BF16, CPL>(a, s, aa, b, ti0, tj0, z0, zc, lane_c, on, lane, warp);
            __syncthreads();
        }
    }
    __syncthreads();

    // Store: the row of 8 cells of one (channel, tile row) is 32 bytes along
    // y; two neighbouring lanes take its two 16-byte halves, so that each
    // warp store instruction writes whole 32-byte sectors.
    constexpr int SL = 32 * CPL;        // channels of a slice (a power of two)
    constexpr int HALVES = kTileJ / 4;  // 16-byte pieces of a tile row
    const int nch = min(SL, a.C - c_base);
    for (int idx = threadIdx.x; idx < SL * kTileI * HALVES; idx += kThreads) {
        const int hv = idx % HALVES, c = (idx / HALVES) & (SL - 1), ci = idx / (HALVES * SL);
        const int i = ti0 + ci, j = tj0 + 4 * hv;
        if (c >= nch || i >= g.X) continue;
        const float* tp = s.tile + (ci * kTileJ + 4 * hv) * s.tile_stride + c;
        const float v0 = tp[0], v1 = tp[s.tile_stride], v2 = tp[2 * s.tile_stride], v3 = tp[3 * s.tile_stride];
        float* op = a.out + (((size_t)b * a.C + c_base + c) * g.X + i) * g.Y + j;
        if (!checked(b < a.B && c_base + c < a.C, kCheckStore)) continue;
        if (a.out_vec && j + 4 <= g.Y) {
            *reinterpret_cast<float4*>(op) = make_float4(v0, v1, v2, v3);
        } else {
            const float v[4] = {v0, v1, v2, v3};
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (j + q < g.Y) op[q] = v[q];
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

#ifdef BEV_BOUNDS_CHECK
unsigned bev_forward_check_take() { return bev::check_take(); }
#endif

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
