// bev_backward.cu -- gradient of the exact dense Sampling-VT with respect to
// the features (sm_100a).
//
// The forward is linear in F, so dL/dF is its adjoint (FlashBEV reading notes,
// "Method" item 4: forward and backward differ from the materialised form only
// by floating-point order):
//   dF_l[b, n, c, y, x] += (sum_k w_k / cnt_k) * dout[b, c, i, j]
// over every (cell, camera) and every texel (y, x) of level l its valid
// samples touch.
//
// One CTA = one 8x8 BEV tile of one batch item and one channel slice of 32 *
// CPL channels, with the tile machinery of bev_tile.cuh.  The tile's dout is
// staged once in shared memory ([cell][channel], read coalesced along y).  A
// warp sweeps one group of cells at a time: the members' dout sit in
// registers, and each texel of the group's union box receives
// sum_g w_g * dout_g over the members with one vector reduction
// (red.global.add.v{1,2,4}.f32) per lane into the fp32 channels-last gradient
// buffer -- one reduction for the whole group, where a per-cell scatter would
// send one per member cell.  Texels where every member's weight is zero (holes
// of the union box) send none.
#include "bev_tile.cuh"

namespace bev {

template <int CPL>
__device__ __forceinline__ void red_add(float* p, const float (&v)[CPL]) {
    if constexpr (CPL == 4)
        asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v[0]), "f"(v[1]), "f"(v[2]),
                     "f"(v[3])
                     : "memory");
    else if constexpr (CPL == 2)
        asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(v[0]), "f"(v[1]) : "memory");
    else
        asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v[0]) : "memory");
}

template <int CPL>
__device__ __forceinline__ void load_tile(float (&v)[CPL], const float* t) {
    if constexpr (CPL == 4) {
        const float4 o = *reinterpret_cast<const float4*>(t);
        v[0] = o.x; v[1] = o.y; v[2] = o.z; v[3] = o.w;
    } else if constexpr (CPL == 2) {
        const float2 o = *reinterpret_cast<const float2*>(t);
        v[0] = o.x; v[1] = o.y;
    } else {
        v[0] = t[0];
    }
}

// Scatter of one group over its union box, two rows by two columns per
// step; weights [texel][member] with S per texel.
template <int CPL, int G>
__device__ __forceinline__ void backward_group(const TileSm& s, const Members& m, const float* wb, float* gl,
                                               size_t rowf, int tf, bool on, int lane) {
    constexpr int S = G == 1 ? 1 : G == 2 ? 2 : G <= 4 ? 4 : 8;
    float d[G][CPL];
#pragma unroll
    for (int gg = 0; gg < G; ++gg) load_tile<CPL>(d[gg], s.tile + m.cell[gg] * s.tile_stride + lane * CPL);
    const int h = m.h, w = m.w;
    float* fb = gl + (size_t)m.y0 * rowf + (size_t)m.x0 * tf;
    for (int c0 = 0; c0 < w; c0 += 2) {
        const bool c1 = m.even || c0 + 1 < w;
        float* p = fb + (size_t)c0 * tf;
        const float* q = wb + c0 * S;
        for (int r0 = 0; r0 < h; r0 += 2, p += 2 * rowf, q += 2 * w * S) {
            const bool r1 = m.even || r0 + 1 < h;
            const bool in[4] = {true, c1, r1, r1 && c1};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (!in[u]) continue;
                float wt[S];
                load_weights<S>(wt, q + ((u >> 1) * w + (u & 1)) * S);
                bool any = false;
#pragma unroll
                for (int gg = 0; gg < G; ++gg) any |= wt[gg] != 0.0f;
                if (!any || !on) continue;
                float v[CPL];
#pragma unroll
                for (int c = 0; c < CPL; ++c) v[c] = __fmul_rn(wt[0], d[0][c]);
#pragma unroll
                for (int gg = 1; gg < G; ++gg)
#pragma unroll
                    for (int c = 0; c < CPL; ++c) v[c] = __fmaf_rn(wt[gg], d[gg][c], v[c]);
                red_add<CPL>(p + (u >> 1) * rowf + (u & 1) * tf, v);
            }
        }
    }
}

// Merge the members' weights in the warp's region, scatter, clear the region.
template <int CPL>
__device__ __forceinline__ void backward_members(const TileSm& s, const Members& m, const GroupItems& it, int zc,
                                                 int Hl, int Wl, float sW, float sH, float* gl, size_t rowf, int tf,
                                                 bool on, int lane, unsigned* wh, unsigned* wl) {
    merge_members(s, m, it, zc, Hl, Wl, sW, sH, wh, wl);
    const float* wb = reinterpret_cast<const float*>(wh);
    switch (m.n) {
        case 1: backward_group<CPL, 1>(s, m, wb, gl, rowf, tf, on, lane); break;
        case 2: backward_group<CPL, 2>(s, m, wb, gl, rowf, tf, on, lane); break;
        case 3: backward_group<CPL, 3>(s, m, wb, gl, rowf, tf, on, lane); break;
        case 4: backward_group<CPL, 4>(s, m, wb, gl, rowf, tf, on, lane); break;
        case 5: backward_group<CPL, 5>(s, m, wb, gl, rowf, tf, on, lane); break;
        case 6: backward_group<CPL, 6>(s, m, wb, gl, rowf, tf, on, lane); break;
        case 7: backward_group<CPL, 7>(s, m, wb, gl, rowf, tf, on, lane); break;
        default: backward_group<CPL, 8>(s, m, wb, gl, rowf, tf, on, lane); break;
    }
    clear_members(m, wh);
}

// A cell whose box does not fit a warp's region: its valid bins (lanes
// 0 .. zc-1 of `one`, a one-cell projection), corner by corner, with weight
// w / cnt.
template <int CPL>
__device__ __forceinline__ void backward_direct(const TileSm& s, const GroupItems& one, int cell, int zc, int Hl,
                                                int Wl, float sW, float sH, float* gl, size_t rowf, int tf, bool on,
                                                int lane) {
    float d[CPL];
    load_tile<CPL>(d, s.tile + cell * s.tile_stride + lane * CPL);
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
            const float wk = __fmul_rn(ws[k], rc);
            if (wk == 0.0f || !on) continue;
            float v[CPL];
#pragma unroll
            for (int q = 0; q < CPL; ++q) v[q] = __fmul_rn(wk, d[q]);
            red_add<CPL>(gl + (size_t)yy * rowf + (size_t)xx * tf, v);
        }
    }
}

// Warps take camera slot aa's groups in turn (largest first) until none is
// left; each group is projected once and scattered on every level.
template <int CPL>
__device__ __forceinline__ void sweep_backward(const SampleArgs& a, const TileSm& s, int aa, int b, int ti0, int tj0,
                                               int z0, int zc, int c_base, bool on, int lane, int warp) {
    unsigned* wh = s.wqh + warp * kWarpEntries;
    unsigned* wl = s.wql + warp * kWarpEntries;
    const int ng = s.ctl[kCtlGroups];
    const int cam = s.ctl[kCtlActive + aa];
    const int tf = a.cpad;  // floats per texel of the gradient buffers
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
            const size_t rowf = (size_t)Wl * tf;
            float* gl = a.lv.grad[l] + ((size_t)b * a.N + cam) * Hl * rowf + c_base + lane * CPL;
            const Members m = members_box(it, gp.cell, gp.n, Hl, Wl, sW, sH);
            if (m.h <= 0 || m.w <= 0) continue;  // no member has a valid voxel on this level
            if (!box_inside(m, Hl, Wl)) continue;
            if (m.entries <= kWarpEntries) {
                backward_members<CPL>(s, m, it, zc, Hl, Wl, sW, sH, gl, rowf, tf, on, lane, wh, wl);
                continue;
            }
            for (int q = 0; q < gp.n; ++q) {  // too large together: cell by cell
                const GroupItems one = project_members(a, s, gp.cell + q, 1, cam, ti0, tj0, z0, zc);
                const Members m1 = members_box(one, gp.cell + q, 1, Hl, Wl, sW, sH);
                if (!box_inside(m1, Hl, Wl)) continue;
                if (m1.entries <= kWarpEntries)
                    backward_members<CPL>(s, m1, one, zc, Hl, Wl, sW, sH, gl, rowf, tf, on, lane, wh, wl);
                else
                    backward_direct<CPL>(s, one, gp.cell[q], zc, Hl, Wl, sW, sH, gl, rowf, tf, on, lane);
            }
        }
    }
}

template <int CPL>
__global__ void __launch_bounds__(kThreads, kTileCtas) sample_backward_kernel(const __grid_constant__ SampleArgs a) {
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
    int ti0, tj0;
    locate_tile(a, s, b, ti0, tj0);
    cull_cameras(a, s, ti0, tj0);
    const int nA = s.ctl[kCtlNA];
    if (nA == 0) return;  // no camera sees the tile: nothing to add

    // dout of the tile: thread (channel, tile row) reads the row's 8 cells
    // along y (two 16-byte loads where dout allows); absent cells and
    // channels are 0.  The loads are issued here and land in shared memory
    // after the count pass, which hides their latency.
    constexpr int SL = 32 * CPL;  // channels of a slice (a power of two)
    constexpr int kIt = (SL * kTileI + kThreads - 1) / kThreads;
    const int nch = min(SL, a.C - c_base);
    float dv[kIt][kTileJ];
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int idx = threadIdx.x + it * kThreads;
        const int c = idx & (SL - 1), i = ti0 + idx / SL;
#pragma unroll
        for (int cj = 0; cj < kTileJ; ++cj) dv[it][cj] = 0.0f;
        if (idx < SL * kTileI && c < nch && i < g.X && checked(b < a.B && c_base + c < a.C, kCheckStore)) {
            const float* dp = a.dout + (((size_t)b * a.C + c_base + c) * g.X + i) * g.Y + tj0;
            if (a.out_vec && tj0 + kTileJ <= g.Y) {
#pragma unroll
                for (int q = 0; q < kTileJ / 4; ++q) {
                    const float4 u4 = __ldg(reinterpret_cast<const float4*>(dp) + q);
                    dv[it][4 * q] = u4.x; dv[it][4 * q + 1] = u4.y; dv[it][4 * q + 2] = u4.z; dv[it][4 * q + 3] = u4.w;
                }
            } else {
#pragma unroll
                for (int cj = 0; cj < kTileJ; ++cj)
                    if (tj0 + cj < g.Y) dv[it][cj] = __ldg(dp + cj);
            }
        }
    }
    const bool on = c_base + lane * CPL < a.cpad;

    for (int z0 = 0; z0 < g.Z; z0 += kZc) {
        const int zc = min(kZc, g.Z - z0);
        if (nA == 1)
            single_camera_pass(a, s, ti0, tj0, z0, zc);
        else
            count_pass(a, s, ti0, tj0, z0, zc);
        if (z0 == 0) {
#pragma unroll
            for (int it = 0; it < kIt; ++it) {
                const int idx = threadIdx.x + it * kThreads;
                if (idx >= SL * kTileI) break;
                float* tp = s.tile + (idx / SL) * kTileJ * s.tile_stride + (idx & (SL - 1));
#pragma unroll
                for (int cj = 0; cj < kTileJ; ++cj) tp[cj * s.tile_stride] = dv[it][cj];
            }
        }
        __syncthreads();
        for (int aa = 0; aa < nA; ++aa) {
            if (warp == 0) form_groups(s, s.xlo + aa * kCells);
            __syncthreads();
            sweep_backward<CPL>(a, s, aa, b, ti0, tj0, z0, zc, c_base, on, lane, warp);
            __syncthreads();
        }
    }
}

template <int CPL>
static cudaError_t launch(const SampleArgs& a, dim3 grid, cudaStream_t st) {
    const size_t smem = tile_layout(a.N, CPL).total;
    static std::atomic<long long> attrs[kAttrDevices];
    const cudaError_t e =
        set_smem_attributes(sample_backward_kernel<CPL>, smem, carveout_percent(smem, kTileCtas), attrs);
    if (e != cudaSuccess) return e;
    sample_backward_kernel<CPL><<<grid, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace bev

#ifdef BEV_BOUNDS_CHECK
unsigned bev_backward_check_take() { return bev::check_take(); }
#endif

cudaError_t bev_launch_backward(const bev::SampleArgs& a, int slices, cudaStream_t stream) {
    const dim3 grid(a.tiles_i * a.tiles_j, a.B, slices);
    switch (a.cpl) {
        case 1: return bev::launch<1>(a, grid, stream);
        case 2: return bev::launch<2>(a, grid, stream);
        case 4: return bev::launch<4>(a, grid, stream);
        default: return cudaErrorInvalidValue;
    }
}
