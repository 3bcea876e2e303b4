// bev_forward_rows.cuh -- fused forward of the exact dense Sampling-VT
// (sm_100a): kernel body and launch tables, instantiated by
// bev_forward_rows.cu (one feature level) and bev_forward_rows_ms.cu (several
// pyramid levels).
//
// out[b, c, i, j] = sum_k [cnt_k > 0] (1 / cnt_k) sum_{valid n} bilinear(F[b, n, c], fx, fy)
// (FlashBEV reading notes, "Method" items 1-2: per-bin valid mean over cameras,
// then a sum over height, in one kernel with nothing intermediate in HBM).
//
// One CTA = one 8x8 BEV tile of one batch item and one channel slice; warp w
// owns tile row w (bev_rows.cuh: cameras culled per tile, every (cell, camera,
// bin) voxel projected once, the weights w / cnt of all bins merged per
// (cell, camera, texel)).  The channel loop then visits each touched texel of
// a (cell, camera) once: the L lanes of a cell read its channel vector with
// 16-byte loads (V chunks per lane) from the channels-last feature buffer and
// accumulate in fp32 registers, which persist across height chunks.  The warp
// finally stores its row along y, the contiguous axis of out, through a
// [channel][cell] staging tile in its own shared-memory region.
//
// Multi-scale form (FlashBEV reading notes, "Takeaway" 4: multi-scale fused
// view transformation): the cell's projections and counts are computed once
// per camera and taken to every pyramid level (u * W_l / W_img - 0.5), whose
// samples add into the same accumulators, so the output is written once.
#pragma once

#include "bev_rows.cuh"

namespace bev {
namespace row {


// Channel chunks of 16 bytes: 4 fp32 or 8 bf16 channels, accumulated in fp32
// pairs with the packed fp32x2 FMA of sm_100 (each half is an IEEE fma.rn).
template <bool BF16>
struct Chunk;

template <>
struct Chunk<false> {
    static constexpr int kPairs = 2;
    __device__ __forceinline__ static void fma(float2 (&acc)[2], const uint4& d, float w) {
        const float2 ww = make_float2(w, w);
        acc[0] = __ffma2_rn(ww, make_float2(__uint_as_float(d.x), __uint_as_float(d.y)), acc[0]);
        acc[1] = __ffma2_rn(ww, make_float2(__uint_as_float(d.z), __uint_as_float(d.w)), acc[1]);
    }
};

template <>
struct Chunk<true> {
    static constexpr int kPairs = 4;
    // bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32 word.
    __device__ __forceinline__ static void fma(float2 (&acc)[4], const uint4& d, float w) {
        const float2 ww = make_float2(w, w);
        acc[0] = __ffma2_rn(ww, make_float2(__uint_as_float(d.x << 16), __uint_as_float(d.x & 0xffff0000u)), acc[0]);
        acc[1] = __ffma2_rn(ww, make_float2(__uint_as_float(d.y << 16), __uint_as_float(d.y & 0xffff0000u)), acc[1]);
        acc[2] = __ffma2_rn(ww, make_float2(__uint_as_float(d.z << 16), __uint_as_float(d.z & 0xffff0000u)), acc[2]);
        acc[3] = __ffma2_rn(ww, make_float2(__uint_as_float(d.w << 16), __uint_as_float(d.w & 0xffff0000u)), acc[3]);
    }
};

template <bool BF16, int V>
using Acc = float2[V][Chunk<BF16>::kPairs];

// Merged path: walk the cell's patch two rows by two columns per step
// (patches are mostly two texels wide: a vertical column of voxels projects
// to a near-vertical line).  The trip counts are the warp's largest patch;
// the other cells of the warp are predicated off past their own.
template <bool BF16, int L, int V>
__device__ __forceinline__ void gather_patch(Acc<BF16, V>& acc, const float* pf, const Patch& pt,
                                             const uint4* Fn, int Wf, int Qtot, int ql, int nchunks) {
    const int h = pt.h, w = pt.w;
    const int hmax = __reduce_max_sync(0xffffffffu, h);
    const int wmax = __reduce_max_sync(0xffffffffu, w);
    const size_t rstride = (size_t)Wf * Qtot;
    bool lane_ok[V];
#pragma unroll
    for (int v = 0; v < V; ++v) lane_ok[v] = ql + v * L < nchunks;
    for (int c0 = 0; c0 < wmax; c0 += 2) {
        const bool c0in = c0 < w, c1in = c0 + 1 < w;
        const float* pw = pf + pt.off + c0;
        const uint4* rp = Fn + ((size_t)pt.y0 * Wf + pt.x0 + c0) * Qtot;
        for (int r0 = 0; r0 < hmax; r0 += 2, pw += 2 * w, rp += 2 * rstride) {
            const bool r0in = r0 < h, r1in = r0 + 1 < h;
            const bool in[4] = {r0in && c0in, r0in && c1in, r1in && c0in, r1in && c1in};
            const float wt[4] = {in[0] ? pw[0] : 0.0f, in[1] ? pw[1] : 0.0f, in[2] ? pw[w] : 0.0f,
                                 in[3] ? pw[w + 1] : 0.0f};
            const uint4* pp[4] = {rp, rp + Qtot, rp + rstride, rp + rstride + Qtot};
            uint4 d[4][V];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < V; ++v)
                    d[u][v] = (in[u] && wt[u] != 0.0f && lane_ok[v]) ? __ldg(pp[u] + v * L) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < V; ++v) Chunk<BF16>::fma(acc[v], d[u][v], wt[u]);
        }
    }
}

// Unmerged path: each bin of the cell (projected by lane zz of the cell's
// lanes) is broadcast to the cell's lanes, which load its four bilinear
// corners and accumulate.  Branch-free: corners outside the map, invalid bins
// and cells with mine == false carry weight 0 and their loads are predicated
// off.  Called by the whole warp.
template <bool BF16, int L, int V, int ZN>
__device__ __forceinline__ void gather_bins(Acc<BF16, V>& acc, const Items<ZN>& it, const float (&rc)[ZN],
                                            int zn, bool mine, int sub, const uint4* Fn, int Hf, int Wf, int Qtot,
                                            int ql, int nchunks) {
    bool lane_ok[V];
#pragma unroll
    for (int v = 0; v < V; ++v) lane_ok[v] = ql + v * L < nchunks;
    const ptrdiff_t rs = (ptrdiff_t)Wf * Qtot;
#pragma unroll
    for (int t = 0; t < ZN; ++t) {
        if (t >= zn) break;
        const float rct = (mine && (it.ok >> t & 1u)) ? rc[t] : 0.0f;
#pragma unroll 2
        for (int zz = 0; zz < L; ++zz) {
            const int src = sub * L + zz;
            const float fx = __shfl_sync(0xffffffffu, it.fx[t], src);
            const float fy = __shfl_sync(0xffffffffu, it.fy[t], src);
            const float r = __shfl_sync(0xffffffffu, rct, src);
            const Corners c = bilinear_corners(fx, fy);
            const bool cx0 = (unsigned)c.x0 < (unsigned)Wf, cx1 = (unsigned)(c.x0 + 1) < (unsigned)Wf;
            const bool cy0 = (unsigned)c.y0 < (unsigned)Hf, cy1 = (unsigned)(c.y0 + 1) < (unsigned)Hf;
            const float wt[4] = {(cy0 && cx0) ? c.w00 * r : 0.0f, (cy0 && cx1) ? c.w01 * r : 0.0f,
                                 (cy1 && cx0) ? c.w10 * r : 0.0f, (cy1 && cx1) ? c.w11 * r : 0.0f};
            const uint4* p = Fn + (ptrdiff_t)(c.y0 * Wf + c.x0) * Qtot;
            const uint4* pp[4] = {p, p + Qtot, p + rs, p + rs + Qtot};
            uint4 d[4][V];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < V; ++v)
                    d[u][v] = (wt[u] != 0.0f && lane_ok[v]) ? __ldg(pp[u] + v * L) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < V; ++v) Chunk<BF16>::fma(acc[v], d[u][v], wt[u]);
        }
    }
}

// One camera's (or one pyramid level's) contribution to the warp's current
// cells: the merged patch walk when it is shorter than the bins' corners,
// else the corners.
template <bool BF16, int L, int V, int ZN>
__device__ __forceinline__ void gather_camera(Acc<BF16, V>& acc, const Items<ZN>& it, const float (&rc)[ZN], int zn,
                                              int sub, int ql, const uint4* Fn, int Hf, int Wf, int Qtot, int nchunks,
                                              int* region) {
    Patch pt = patch_box<L, ZN>(it, zn, Hf, Wf);
    if (!checked(pt.h == 0 || (pt.y0 >= 0 && pt.x0 >= 0 && pt.y0 + pt.h <= Hf && pt.x0 + pt.w <= Wf), kCheckBox)) pt.h = 0;
    if (merge_pays<L>(pt, zn, kMergeStepsFwd)) {
        merge_patches<L, ZN>(pt, it, rc, zn, sub, ql, Hf, Wf, region);
        gather_patch<BF16, L, V>(acc, reinterpret_cast<const float*>(region), pt, Fn, Wf, Qtot, ql, nchunks);
        if (__any_sync(0xffffffffu, pt.overflow))
            gather_bins<BF16, L, V, ZN>(acc, it, rc, zn, pt.overflow, sub, Fn, Hf, Wf, Qtot, ql, nchunks);
        __syncwarp();  // the region is rebuilt for the next camera
    } else {
        gather_bins<BF16, L, V, ZN>(acc, it, rc, zn, true, sub, Fn, Hf, Wf, Qtot, ql, nchunks);
    }
}

// Kernel body.  MS: multi-scale -- each camera's projections are taken to
// every level of a.lv (one projection, one count, per-level sampling).
template <bool BF16, int L, int V, bool MS>
__device__ __forceinline__ void forward_body(const SampleArgs& a) {
    constexpr int P = Chunk<BF16>::kPairs;
    constexpr int G = 32 / L;                // cells a warp works on at once
    constexpr int CG = kCellsPerWarp / G;    // rounds of cells per warp
    static_assert(G * CG == kCellsPerWarp, "lanes per cell must be 4, 8, 16 or 32");
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const CtaSmem s = carve_smem(smem_raw, a.N);
    const GeoParams& g = a.g;

    const int b = blockIdx.y;
    int ti0, tj0;
    tile_origin(a, s, b, s.act + 40, ti0, tj0);
    const int chunk0 = blockIdx.z * a.slice_chunks;
    const int nchunks = min(a.slice_chunks, a.Qtot - chunk0);
    setup_tile(a, s, ti0, tj0);
    const int nA = s.act[32];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / L, ql = lane - sub * L;
    int* region = reinterpret_cast<int*>(s.warps + (size_t)warp * (kWarpBytes + 512));
    const size_t texels = (size_t)g.Hf * g.Wf;
    // single level: this lane's chunks of batch item b (camera 0)
    const uint4* feat = MS ? nullptr
                           : reinterpret_cast<const uint4*>(a.feat) + chunk0 + ql + (size_t)b * a.N * texels * a.Qtot;
    const int i = ti0 + warp;
    const float x = voxel_centre(g.xmin, i, g.dx);
    const bool write_count = a.count != nullptr && blockIdx.z == 0;
    constexpr int ZN = z_per_lane_fwd<BF16, L, V>();
    const int zn = min(ZN, (g.Z + L - 1) / L);  // bins per lane per chunk

    float2 acc[CG][V][P];
#pragma unroll
    for (int q = 0; q < CG; ++q)
#pragma unroll
        for (int v = 0; v < V; ++v)
#pragma unroll
            for (int e = 0; e < P; ++e) acc[q][v][e] = make_float2(0.0f, 0.0f);

#pragma unroll
    for (int q = 0; q < CG; ++q) {
        const int j = tj0 + q * G + sub;
        const bool in_grid = i < g.X && j < g.Y;
        const float y = voxel_centre(g.ymin, j, g.dy);
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
            for (int t = 0; t < ZN; ++t) {
                rc[t] = cnt[t] > 0 ? __frcp_rn((float)cnt[t]) : 0.0f;
                const int z = z0 + ql + L * t;
                if (write_count && t < zn && in_grid && z < g.Z)
                    a.count[(((size_t)b * g.X + i) * g.Y + j) * g.Z + z] = (uint8_t)cnt[t];
            }
            for (int aa = 0; aa < nA; ++aa) {
                const Items<ZN> it = aa == 0 ? keep0
                                   : aa == 1 ? keep1
                                             : project_items<L, ZN, MS>(s.cams + s.act[aa] * kCamFloats, x, y, in_grid, z0, zn, ql, g);
                const int cam = s.act[aa];
                if constexpr (!MS) {
                    gather_camera<BF16, L, V, ZN>(acc[q], it, rc, zn, sub, ql, feat + (size_t)cam * texels * a.Qtot,
                                                  g.Hf, g.Wf, a.Qtot, nchunks, region);
                } else {
                    for (int l = 0; l < a.lv.n; ++l) {
                        const int Hl = a.lv.Hf[l], Wl = a.lv.Wf[l];
                        const uint4* Fn = reinterpret_cast<const uint4*>(a.lv.feat[l]) + chunk0 + ql +
                                          ((size_t)b * a.N + cam) * ((size_t)Hl * Wl) * a.Qtot;
                        gather_camera<BF16, L, V, ZN>(acc[q], at_level(it, a.lv.sW[l], a.lv.sH[l]), rc, zn, sub, ql,
                                                      Fn, Hl, Wl, a.Qtot, nchunks, region);
                    }
                }
            }
        }
    }

    // Store the warp's row: [channel][cell] staging tile in the warp's region,
    // then rows of 8 cells along y.  Lanes of absent cameras still write 0.
    float* stage = reinterpret_cast<float*>(region);
    const int c_base = chunk0 * 2 * P;
    const int c_real = max(0, min(nchunks * 2 * P, a.C - c_base));
#pragma unroll
    for (int q = 0; q < CG; ++q) {
        const int jc = q * G + sub;
#pragma unroll
        for (int v = 0; v < V; ++v) {
            const int c0 = (ql + v * L) * 2 * P;
            if (ql + v * L < nchunks) {
#pragma unroll
                for (int e = 0; e < P; ++e) {
                    stage[(c0 + 2 * e) * kStageStride + jc] = acc[q][v][e].x;
                    stage[(c0 + 2 * e + 1) * kStageStride + jc] = acc[q][v][e].y;
                }
            }
        }
    }
    __syncwarp();
    if (i < g.X) {
        if (a.out_vec) {  // rows of 8 cells start 16-byte aligned: two float4 per channel
            for (int t = lane; t < c_real * 2; t += 32) {
                const int c = t >> 1, jc = (t & 1) * 4;
                if (tj0 + jc < g.Y && checked(c_base + c < a.C, kCheckStore)) {
                    const float* sp = stage + c * kStageStride + jc;
                    float* op = a.out + (((size_t)b * a.C + c_base + c) * g.X + i) * g.Y + tj0 + jc;
                    *reinterpret_cast<float4*>(op) = make_float4(sp[0], sp[1], sp[2], sp[3]);
                }
            }
        } else {
            for (int t = lane; t < c_real * kCellsPerWarp; t += 32) {
                const int c = t >> 3, jc = t & 7;
                if (tj0 + jc < g.Y && checked(c_base + c < a.C, kCheckStore))
                    a.out[(((size_t)b * a.C + c_base + c) * g.X + i) * g.Y + tj0 + jc] = stage[c * kStageStride + jc];
            }
        }
    }
}

template <bool BF16, int L, int V>
__global__ void __launch_bounds__(kThreads, (fwd_ctas_per_sm<BF16, L, V, false>())) sample_forward_kernel(const SampleArgs a) {
    forward_body<BF16, L, V, false>(a);
}

// The level table is indexed at run time: __grid_constant__ lets the body
// read it in place from the parameter space.
template <bool BF16, int L, int V>
__global__ void __launch_bounds__(kThreads, (fwd_ctas_per_sm<BF16, L, V, true>()))
    sample_forward_ms_kernel(const __grid_constant__ SampleArgs a) {
    forward_body<BF16, L, V, true>(a);
}

template <bool MS, bool BF16, int L, int V>
static cudaError_t launch_one(const SampleArgs& a, dim3 grid, size_t smem, cudaStream_t st) {
    void (*k)(const SampleArgs);
    if constexpr (MS)
        k = sample_forward_ms_kernel<BF16, L, V>;
    else
        k = sample_forward_kernel<BF16, L, V>;
    static std::atomic<long long> attrs[kAttrDevices];
    const cudaError_t e = set_smem_attributes(k, smem, carveout_percent(smem, fwd_ctas_per_sm<BF16, L, V, MS>()), attrs);
    if (e != cudaSuccess) return e;
    k<<<grid, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

// (L, V) combinations the host's lane picker can produce: L * V <= 32 chunks
// for fp32 slices, <= 16 for bf16 slices (128 channels either way).
template <bool MS>
static cudaError_t launch_fwd_f32(const SampleArgs& a, int V, dim3 grid, size_t smem, cudaStream_t st) {
    switch (a.L * 16 + V) {
        case 32 * 16 + 1: return launch_one<MS, false, 32, 1>(a, grid, smem, st);
        case 16 * 16 + 1: return launch_one<MS, false, 16, 1>(a, grid, smem, st);
        case 16 * 16 + 2: return launch_one<MS, false, 16, 2>(a, grid, smem, st);
        case 8 * 16 + 1: return launch_one<MS, false, 8, 1>(a, grid, smem, st);
        case 8 * 16 + 2: return launch_one<MS, false, 8, 2>(a, grid, smem, st);
        case 8 * 16 + 3: return launch_one<MS, false, 8, 3>(a, grid, smem, st);
        case 8 * 16 + 4: return launch_one<MS, false, 8, 4>(a, grid, smem, st);
        case 4 * 16 + 1: return launch_one<MS, false, 4, 1>(a, grid, smem, st);
        case 4 * 16 + 2: return launch_one<MS, false, 4, 2>(a, grid, smem, st);
        case 4 * 16 + 3: return launch_one<MS, false, 4, 3>(a, grid, smem, st);
        case 4 * 16 + 4: return launch_one<MS, false, 4, 4>(a, grid, smem, st);
        case 4 * 16 + 5: return launch_one<MS, false, 4, 5>(a, grid, smem, st);
        case 4 * 16 + 6: return launch_one<MS, false, 4, 6>(a, grid, smem, st);
        case 4 * 16 + 7: return launch_one<MS, false, 4, 7>(a, grid, smem, st);
        case 4 * 16 + 8: return launch_one<MS, false, 4, 8>(a, grid, smem, st);
        default: return cudaErrorInvalidValue;
    }
}

template <bool MS>
static cudaError_t launch_fwd_bf16(const SampleArgs& a, int V, dim3 grid, size_t smem, cudaStream_t st) {
    switch (a.L * 16 + V) {
        case 16 * 16 + 1: return launch_one<MS, true, 16, 1>(a, grid, smem, st);
        case 8 * 16 + 1: return launch_one<MS, true, 8, 1>(a, grid, smem, st);
        case 8 * 16 + 2: return launch_one<MS, true, 8, 2>(a, grid, smem, st);
        case 4 * 16 + 1: return launch_one<MS, true, 4, 1>(a, grid, smem, st);
        case 4 * 16 + 2: return launch_one<MS, true, 4, 2>(a, grid, smem, st);
        case 4 * 16 + 3: return launch_one<MS, true, 4, 3>(a, grid, smem, st);
        case 4 * 16 + 4: return launch_one<MS, true, 4, 4>(a, grid, smem, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace row
}  // namespace bev
