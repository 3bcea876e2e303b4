// bev_backward.cuh -- gradient of the exact dense Sampling-VT with respect to
// the features (sm_100a): kernel body and launch tables, instantiated by
// bev_backward.cu (one feature level) and bev_backward_ms.cu (several
// pyramid levels, each with its own gradient buffer).
//
// The forward is linear in F, so dL/dF is its adjoint (FlashBEV reading notes,
// "Method" item 4: forward and backward differ from the materialised form only
// by floating-point order):
//   dF[b, n, c, y, x] += (sum_k w_k / cnt_k) * dout[b, c, i, j]
// over every (cell, camera) and every texel (y, x) its valid samples touch.
//
// One CTA = one tile of 8 BEV rows of one batch item and one channel slice,
// with the same culling, once-per-voxel geometry and merged per-(cell,
// camera, texel) weights as the forward (bev_warp.cuh).  Each lane holds
// dout of V chunks of 4 channels of its cell in registers; each touched
// texel then receives one 16-byte vector reduction per chunk
// (red.global.add.v4.f32) into the fp32 channels-last gradient buffer,
// however many height bins hit it.  The tile width is chosen per launch:
// narrower tiles when the grid gives few tiles, so that the launch does not
// end on a short second wave of heavy tiles.
#pragma once

#include "bev_warp.cuh"

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

// Merged path: walk the cell's patch two rows by two columns per step, as
// the forward does; the trip counts are the warp's largest patch and other
// cells are predicated off past their own.  Texels with weight 0 get no
// reduction.
template <int L, int V>
__device__ __forceinline__ void scatter_patch(const float (&d)[V][4], const float* pf, const Patch& pt, float* Gn,
                                              int Wf, int tstride, int ql, int nchunks) {
    const int h = pt.h, w = pt.w;
    const int hmax = __reduce_max_sync(0xffffffffu, h);
    const int wmax = __reduce_max_sync(0xffffffffu, w);
    const size_t rstride = (size_t)Wf * tstride;
    bool lane_ok[V];
#pragma unroll
    for (int v = 0; v < V; ++v) lane_ok[v] = ql + v * L < nchunks;
    for (int c0 = 0; c0 < wmax; c0 += 2) {
        const bool c0in = c0 < w, c1in = c0 + 1 < w;
        const float* pw = pf + pt.off + c0;
        float* rp = Gn + ((size_t)pt.y0 * Wf + pt.x0 + c0) * tstride;
        for (int r0 = 0; r0 < hmax; r0 += 2, pw += 2 * w, rp += 2 * rstride) {
            const bool r0in = r0 < h, r1in = r0 + 1 < h;
            const bool in[4] = {r0in && c0in, r0in && c1in, r1in && c0in, r1in && c1in};
            const float wt[4] = {in[0] ? pw[0] : 0.0f, in[1] ? pw[1] : 0.0f, in[2] ? pw[w] : 0.0f,
                                 in[3] ? pw[w + 1] : 0.0f};
            float* pp[4] = {rp, rp + tstride, rp + rstride, rp + rstride + tstride};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (wt[u] == 0.0f) continue;
#pragma unroll
                for (int v = 0; v < V; ++v)
                    if (lane_ok[v])
                        red_add_v4(pp[u] + v * L * 4, wt[u] * d[v][0], wt[u] * d[v][1], wt[u] * d[v][2],
                                   wt[u] * d[v][3]);
            }
        }
    }
}

// Fallback for cells whose patches did not fit: each valid bin's four
// corners, broadcast from the lane that projected it.  Called by the whole
// warp.
template <int L, int V, int ZN>
__device__ __forceinline__ void scatter_direct(const float (&d)[V][4], const Items<ZN>& it,
                                               const float (&rc)[ZN], int zn, bool mine, int sub,
                                               float* Gn, int Hf, int Wf, int tstride, int ql, int nchunks) {
#pragma unroll
    for (int t = 0; t < ZN; ++t) {
        if (t >= zn) break;
        for (int zz = 0; zz < L; ++zz) {
            const int src = sub * L + zz;
            const float fx = __shfl_sync(0xffffffffu, it.fx[t], src);
            const float fy = __shfl_sync(0xffffffffu, it.fy[t], src);
            const bool ok = (__shfl_sync(0xffffffffu, it.ok, src) >> t) & 1u;
            const float r = __shfl_sync(0xffffffffu, rc[t], src);
            if (!(mine && ok)) continue;
            const Corners c = bilinear_corners(fx, fy);
            const float ws[4] = {c.w00, c.w01, c.w10, c.w11};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int yy = c.y0 + (k >> 1), xx = c.x0 + (k & 1);
                if ((unsigned)yy >= (unsigned)Hf || (unsigned)xx >= (unsigned)Wf) continue;
                scatter_texel<L, V>(Gn + ((size_t)yy * Wf + xx) * tstride, d, ws[k] * r, ql, nchunks);
            }
        }
    }
}

// One camera's (or one pyramid level's) scatter for the warp's current
// cells: always merged -- a merged texel costs one reduction per chunk
// instead of one per bin that touches it.
template <int L, int V, int ZN>
__device__ __forceinline__ void scatter_camera(const float (&d)[V][4], const Items<ZN>& it, const float (&rc)[ZN],
                                               int zn, int sub, int ql, float* Gn, int Hf, int Wf, int tstride,
                                               int nchunks, int* region) {
    Patch pt = patch_box<L, ZN>(it, zn, Hf, Wf);
    merge_patches<L, ZN>(pt, it, rc, zn, sub, ql, Hf, Wf, region);
    scatter_patch<L, V>(d, reinterpret_cast<const float*>(region), pt, Gn, Wf, tstride, ql, nchunks);
    if (__any_sync(0xffffffffu, pt.overflow))
        scatter_direct<L, V, ZN>(d, it, rc, zn, pt.overflow, sub, Gn, Hf, Wf, tstride, ql, nchunks);
    __syncwarp();  // the region is rebuilt for the next camera
}

// Kernel body.  MS: multi-scale -- each camera's projections are taken to
// every level of a.lv, each level scattering into its own gradient buffer.
template <int L, int V, bool MS>
__device__ __forceinline__ void backward_body(const SampleArgs& a) {
    constexpr int G = 32 / L;
    static_assert(G * L == 32, "lanes per cell must divide the warp");
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const CtaSmem s = carve_smem(smem_raw, a.N);
    const GeoParams& g = a.g;

    const int b = blockIdx.y;
    int ti0, tj0;
    tile_origin(a, s, b, s.act + 40, ti0, tj0);
    const int chunk0 = blockIdx.z * a.slice_chunks;
    const int nchunks = min(a.slice_chunks, a.Qtot - chunk0);
    const int c_base = chunk0 * 4;
    setup_tile(a, s, ti0, tj0);
    const int nA = s.act[32];
    if (nA == 0) return;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / L, ql = lane - sub * L;
    int* region = reinterpret_cast<int*>(s.warps + (size_t)warp * (kWarpBytes + 512));
    const int i = ti0 + warp;
    const size_t texels = (size_t)g.Hf * g.Wf;
    const int tstride = a.Qtot * 4;  // floats per texel in the gradient buffer
    // single level: this lane's chunks of batch item b (camera 0)
    float* grad = MS ? nullptr : a.dfeat + (size_t)(chunk0 + ql) * 4 + (size_t)b * a.N * texels * tstride;
    const float x = voxel_centre(g.xmin, i, g.dx);
    constexpr int ZN = kZPerLaneBwd;
    const int zn = min(ZN, (g.Z + L - 1) / L);
    const size_t cstride = (size_t)g.X * g.Y;

    // G cells at a time along the warp's row of tile_j cells
    for (int j1 = tj0; j1 < tj0 + a.tile_j; j1 += G) {
        const int j = j1 + sub;
        const bool in_grid = i < g.X && j < g.Y;
        const float y = voxel_centre(g.ymin, j, g.dy);
        // dout of this lane's cell and channel chunks (for one channel the G
        // cells of the group are consecutive along y)
        float d[V][4];
        const float* dp = a.dout + ((size_t)b * a.C + c_base) * cstride + (size_t)i * g.Y + j;
#pragma unroll
        for (int v = 0; v < V; ++v) {
            const int c0 = (ql + v * L) * 4;
#pragma unroll
            for (int e = 0; e < 4; ++e)
                d[v][e] = (in_grid && ql + v * L < nchunks && c_base + c0 + e < a.C) ? dp[(c0 + e) * cstride] : 0.0f;
        }
        for (int z0 = 0; z0 < g.Z; z0 += L * zn) {
            // valid cameras per bin of this lane, over all active cameras; the
            // projections of the first two cameras are kept for the merge pass
            int cnt[ZN] = {};
            Items<ZN> keep0, keep1;
            for (int aa = 0; aa < nA; ++aa) {
                const Items<ZN> it = project_items<L, ZN, MS>(s.cams + s.act[aa] * kCamFloats, x, y, in_grid, z0, zn, ql, g);
                if (aa == 0) keep0 = it;
                if (aa == 1) keep1 = it;
#pragma unroll
                for (int t = 0; t < ZN; ++t) cnt[t] += (it.ok >> t) & 1u;
            }
            float rc[ZN];
#pragma unroll
            for (int t = 0; t < ZN; ++t) rc[t] = cnt[t] > 0 ? __frcp_rn((float)cnt[t]) : 0.0f;
            for (int aa = 0; aa < nA; ++aa) {
                const Items<ZN> it = aa == 0 ? keep0
                                   : aa == 1 ? keep1
                                             : project_items<L, ZN, MS>(s.cams + s.act[aa] * kCamFloats, x, y, in_grid, z0, zn, ql, g);
                const int cam = s.act[aa];
                if constexpr (!MS) {
                    scatter_camera<L, V, ZN>(d, it, rc, zn, sub, ql, grad + (size_t)cam * texels * tstride, g.Hf, g.Wf,
                                             tstride, nchunks, region);
                } else {
                    for (int l = 0; l < a.lv.n; ++l) {
                        const int Hl = a.lv.Hf[l], Wl = a.lv.Wf[l];
                        float* Gn = a.lv.grad[l] + (size_t)(chunk0 + ql) * 4 +
                                    ((size_t)b * a.N + cam) * ((size_t)Hl * Wl) * tstride;
                        scatter_camera<L, V, ZN>(d, at_level(it, a.lv.sW[l], a.lv.sH[l]), rc, zn, sub, ql, Gn, Hl, Wl,
                                                 tstride, nchunks, region);
                    }
                }
            }
        }
    }
}

template <int L, int V>
__global__ void __launch_bounds__(kThreads, kCtasPerSmBwd) sample_backward_kernel(const SampleArgs a) {
    backward_body<L, V, false>(a);
}

// The level table is indexed at run time: __grid_constant__ lets the body
// read it in place from the parameter space.
template <int L, int V>
__global__ void __launch_bounds__(kThreads, kCtasPerSmBwd) sample_backward_ms_kernel(const __grid_constant__ SampleArgs a) {
    backward_body<L, V, true>(a);
}

template <bool MS, int L, int V>
static cudaError_t launch_one(const SampleArgs& a, dim3 grid, size_t smem, cudaStream_t st) {
    void (*k)(const SampleArgs);
    if constexpr (MS)
        k = sample_backward_ms_kernel<L, V>;
    else
        k = sample_backward_kernel<L, V>;
    static std::atomic<long long> attrs[kAttrDevices];
    const cudaError_t e = set_smem_attributes(k, smem, carveout_percent(smem, kCtasPerSmBwd), attrs);
    if (e != cudaSuccess) return e;
    k<<<grid, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <bool MS>
static cudaError_t launch_bwd(const SampleArgs& a, int V, dim3 grid, size_t smem, cudaStream_t st) {
    switch (a.L * 16 + V) {
        case 32 * 16 + 1: return launch_one<MS, 32, 1>(a, grid, smem, st);
        case 16 * 16 + 1: return launch_one<MS, 16, 1>(a, grid, smem, st);
        case 16 * 16 + 2: return launch_one<MS, 16, 2>(a, grid, smem, st);
        case 8 * 16 + 1: return launch_one<MS, 8, 1>(a, grid, smem, st);
        case 8 * 16 + 2: return launch_one<MS, 8, 2>(a, grid, smem, st);
        case 8 * 16 + 3: return launch_one<MS, 8, 3>(a, grid, smem, st);
        case 8 * 16 + 4: return launch_one<MS, 8, 4>(a, grid, smem, st);
        case 4 * 16 + 1: return launch_one<MS, 4, 1>(a, grid, smem, st);
        case 4 * 16 + 2: return launch_one<MS, 4, 2>(a, grid, smem, st);
        case 4 * 16 + 3: return launch_one<MS, 4, 3>(a, grid, smem, st);
        case 4 * 16 + 4: return launch_one<MS, 4, 4>(a, grid, smem, st);
        case 4 * 16 + 5: return launch_one<MS, 4, 5>(a, grid, smem, st);
        case 4 * 16 + 6: return launch_one<MS, 4, 6>(a, grid, smem, st);
        case 4 * 16 + 7: return launch_one<MS, 4, 7>(a, grid, smem, st);
        case 4 * 16 + 8: return launch_one<MS, 4, 8>(a, grid, smem, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace bev
