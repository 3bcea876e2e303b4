// bev_rows.cuh -- the row-per-warp machinery of the dense forward (sm_100a).
//
// FlashBEV's reading notes recompute the channel-independent geometry for
// every channel ("Method" item 3) and name that recompute as the cost that
// grows with C ("Limitation", second point; their "Takeaway" 4 proposes
// block-level geometry reuse).  Here a CTA owns an 8x8 tile of BEV cells: it
// stages the calibrations once and culls the cameras that cannot see any
// voxel of the tile; from then on each warp works on its own tile row, with
// no CTA-wide barrier.  For G = 32 / L cells at a time a warp
//   1. projects each (cell, camera, height bin) voxel once -- lanes of a cell
//      take consecutive bins -- and counts the valid cameras of each bin in
//      registers;
//   2. per camera, reduces the box of texels the cell's valid voxels touch and
//      lays a patch over it in the warp's shared-memory region;
//   3. merges the bilinear weights w / cnt of all bins into the patch with
//      integer atomics on an exact fixed-point representation, so the merged
//      weight does not depend on the order of the additions, then rounds each
//      merged weight once to fp32;
//   4. hands the patch to the channel loop (lanes of a cell now take channel
//      chunks), which visits each touched texel once, whatever the number of
//      bins that hit it.  Patches that do not fit fall back to visiting the
//      four bilinear corners of each bin.
// (The feature gradient uses the tile-group machinery of bev_tile.cuh, whose
// group-level reductions pay there; for the gather this per-warp form
// measured faster.)
#pragma once

#include <limits.h>

#include "bev_kernels.cuh"

namespace bev {
namespace row {

// BEV tile owned by one CTA: kTileI rows (ego x) by kTileJ columns (ego y).
// Warp w owns tile row w (kTileJ = 8 cells) and works on it on its own: after
// the CTA has staged the calibrations and culled the cameras, no CTA-wide
// barrier is needed.
constexpr int kTileI = 8;
constexpr int kTileJ = 8;
constexpr int kTile = kTileI * kTileJ;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kCellsPerWarp = kTile / kWarps;
static_assert(kCellsPerWarp == kTileJ && kWarps == kTileI, "one warp per tile row");
// Height bins a lane projects per chunk (chunk = lanes per cell * this).  The
// projections of a chunk stay in registers (two of them cached per cell
// group), and taller grids take more chunks.  The forward's accumulators
// already fill the register file: fp32 slices with eight or more lanes per
// cell take one bin per lane (two spill), bf16 slices and four-lane cells
// take two (one is slower there), except fp32 slices of four lanes with five
// chunks each (80 channels), which run two CTAs per SM and measured 2%
// faster with four.  The backward, which holds dout instead, takes four.
template <bool BF16, int L, int V>
constexpr int z_per_lane_fwd() { return (!BF16 && L >= 8) ? 1 : (!BF16 && L == 4 && V == 5) ? 4 : 2; }
constexpr int kZPerLaneBwd = 4;
constexpr int kZPerLaneMax = kZPerLaneBwd;
// Merged-weight entries of one warp for one (camera, height chunk): the
// patches of the cells the warp works on at once.  Each entry is an exact
// fixed-point sum split over two 32-bit words (see merge_patches).
constexpr int kWarpPatchCap = 512;
// Forward: merging the weights of one (cell group, camera) pays when the
// merged patch walk takes fewer steps (four texels of every lane's chunks)
// than the bins' corners unmerged, plus this margin for the merge itself.
// The backward always merges: there a step costs global reductions.
constexpr int kMergeStepsFwd = 0;
// Per-warp shared-memory region: the patch words, reused as the
// [channel][cell] staging tile of the warp's row (kSliceMax x kStageStride).
constexpr int kSliceMax = 128;
constexpr int kStageStride = kCellsPerWarp + 1;
constexpr int kWarpBytes = 2 * sizeof(int) * kWarpPatchCap;
static_assert((int)sizeof(float) * kSliceMax * kStageStride <= kWarpBytes + 512,
              "staging tile must fit the warp region");
// CTAs kept resident per SM, per instantiation: three (at most 85 registers
// a thread) when the per-lane state fits -- the accumulators (cell rounds x
// chunks x fp32 pairs), the four corners' loads of each chunk (16 registers a
// chunk) and the two cached projections -- and two (up to 128 registers)
// when it would spill: the larger slices measured 5 to 14% faster without the
// spills than with the third CTA.  The multi-scale kernel, which also carries
// the level loop, measured faster with two.  Shared memory stays small
// (~38 KB a CTA) so that most of the SM's on-chip array serves as L1 for the
// tiles' texel windows.
template <bool BF16, int L, int V, bool MS>
constexpr int fwd_ctas_per_sm() {
    constexpr int pairs = BF16 ? 4 : 2;                 // fp32 pairs per 16-byte chunk
    constexpr int rounds = kCellsPerWarp / (32 / L);    // cell rounds per warp
    constexpr int zn = z_per_lane_fwd<BF16, L, V>();
    constexpr int regs = rounds * V * pairs * 2 + 16 * V + 8 * zn;
    return (!MS && regs <= 56) ? 3 : 2;
}

// Feature-pyramid levels of the multi-scale operator.  Every level shares
// the voxel's projection, validity and count; level l samples its own map at
// its own scale.  The single-level kernels read g (Hf, Wf, sW, sH) and feat
// instead.
constexpr int kMaxLevels = 4;

struct LevelTable {
    int n;                            // levels, 1 .. kMaxLevels
    int Hf[kMaxLevels], Wf[kMaxLevels];
    float sW[kMaxLevels], sH[kMaxLevels];  // (float)W_l / img_w, (float)H_l / img_h, host IEEE divide
    const void* feat[kMaxLevels];     // forward: channels-last features of level l (16-byte chunks)
};

struct SampleArgs {
    const void* feat;       // channels-last [B*N][Hf*Wf][Qtot chunks of 16 bytes]
    const float* K;         // [B,N,3,3]
    const float* E;         // [B,N,4,4]
    float* out;             // forward: [B,C,X,Y]
    uint8_t* count;         // forward: [B,X,Y,Z] or null
    GeoParams g;
    int B, N, C;
    int Qtot;               // 16-byte chunks per texel in the channels-last buffer
    int chan_per_chunk;     // 4 (fp32) or 8 (bf16)
    int slice_chunks;       // chunks per CTA channel slice
    int L;                  // lanes per cell (4, 8, 16 or 32)
    int tile_j;             // cells per tile row (kTileJ)
    int tiles_i, tiles_j;   // tiles along X and Y
    int out_vec;            // out is 16-byte aligned and Y % 4 == 0
    LevelTable lv;          // multi-scale kernels only
};

// Bytes of dynamic shared memory of one CTA (see carve_smem).
// Byte offsets of the per-CTA shared-memory regions (one source of truth for
// the kernels' carve-up and the launch size).
struct SmemLayout {
    size_t warps, cams, act, total;
};

__host__ __device__ inline SmemLayout smem_layout(int N) {
    SmemLayout l;
    size_t b = 0;
    l.warps = b;  b += (size_t)kWarps * (kWarpBytes + 512);           // per-warp patch / staging regions
    l.cams = b;   b += sizeof(float) * ((N * kCamFloats + 3) & ~3);   // camera constants
    l.act = b;    b += sizeof(int) * 128;                             // active cameras, tile slot, flags
    l.total = b;
    return l;
}

__host__ __device__ inline size_t sample_smem_bytes(int N) { return smem_layout(N).total; }

// Bounds-checked build (-DBEV_BOUNDS_CHECK): each patch box is tested against
// its feature map before the walk and each merge word against the warp's
// region; a violation sets a bit of this translation unit's device error
// word and the access is skipped.  Read back by check_take on the host.
enum : unsigned { kCheckBox = 1u, kCheckMerge = 2u, kCheckStore = 8u };
#ifdef BEV_BOUNDS_CHECK
static __device__ unsigned g_check_word;
__device__ __forceinline__ bool checked(bool ok, unsigned code) {
    if (!ok) atomicOr(&g_check_word, code);
    return ok;
}
static inline unsigned check_take() {
    unsigned w = 0, z = 0;
    if (cudaMemcpyFromSymbol(&w, g_check_word, sizeof(w)) != cudaSuccess) w = ~0u;
    cudaMemcpyToSymbol(g_check_word, &z, sizeof(z));
    return w;
}
#else
__device__ __forceinline__ bool checked(bool, unsigned) { return true; }
#endif


struct CtaSmem {
    unsigned char* warps;  // kWarps regions of kWarpBytes + 512
    float* cams;           // [N][kCamFloats]
    int* act;              // [0..nA) active camera ids, [32] nA, [40..41] tile origin, [64..95] flags
};

__device__ __forceinline__ CtaSmem carve_smem(unsigned char* smem, int N) {
    const SmemLayout l = smem_layout(N);
    CtaSmem s;
    s.warps = smem + l.warps;
    s.cams = reinterpret_cast<float*>(smem + l.cams);
    s.act = reinterpret_cast<int*>(smem + l.act);
    return s;
}

// Calibrations of batch item b into shared memory: E rows 0..2, then K rows
// 0..1, per camera; threads first .. kThreads - 1 take one float at a time.
// Only the per-CTA set-up reads them from global memory.
__device__ __forceinline__ void stage_cams(const SampleArgs& a, const CtaSmem& s, int b, int first) {
    for (int t = (int)threadIdx.x - first; t < a.N * kCamFloats; t += kThreads - first) {
        const int n = t / kCamFloats, r = t - n * kCamFloats;
        s.cams[t] = r < 12 ? a.E[((size_t)b * a.N + n) * 16 + r]
                           : a.K[((size_t)b * a.N + n) * 9 + (r - 12)];
    }
}

// Tile of this CTA.  Tiles are issued in rings of increasing Chebyshev
// distance from the centre tile of the grid: for rigs mounted near the grid
// centre the nearest voxels see the most texels, so the heaviest tiles start
// first and the light outer ring fills the tail of the launch.  Any order
// gives the same results.  Warp 0 maps the block index (the rank) to its
// ring -- its lanes test 32 candidate rings at a time -- then finds the
// position inside the ring with ballots over 32 ring positions at a time.
// The other warps meanwhile stage batch item b's calibrations.
__device__ inline void tile_origin(const SampleArgs& a, const CtaSmem& s, int b, int* slot, int& ti0, int& tj0) {
    const int Ti = a.tiles_i, Tj = a.tiles_j;
    if (threadIdx.x < 32) {
        const int ci = (Ti - 1) >> 1, cj = (Tj - 1) >> 1;
        auto area = [&](int r) -> int {  // tiles within Chebyshev distance r of the centre
            if (r < 0) return 0;
            const int h = min(ci + r, Ti - 1) - max(ci - r, 0) + 1;
            const int w = min(cj + r, Tj - 1) - max(cj - r, 0) + 1;
            return h * w;
        };
        // ring r of rank k: the smallest r with area(r) > k (area grows with
        // r and area(rmax) is every tile)
        const int rmax = max(max(ci, Ti - 1 - ci), max(cj, Tj - 1 - cj));
        const int rank = blockIdx.x;
        int r = rmax;
        for (int r0 = 0; r0 <= rmax; r0 += 32) {
            const int cand = r0 + (int)threadIdx.x;
            const unsigned m = __ballot_sync(0xffffffffu, cand <= rmax && area(cand) > rank);
            if (m) {
                r = r0 + __ffs(m) - 1;
                break;
            }
        }
        int k = rank - area(r - 1);
        const int ring = r == 0 ? 1 : 8 * r;
        int found = -1;
        for (int p0 = 0; p0 < ring && found < 0; p0 += 32) {
            const int p = p0 + (int)threadIdx.x;
            int di = 0, dj = 0;
            if (r > 0 && p < ring) {
                const int side = p / (2 * r), t = p - side * 2 * r;
                if (side == 0)      { di = -r;     dj = -r + t; }
                else if (side == 1) { di = -r + t; dj = r; }
                else if (side == 2) { di = r;      dj = r - t; }
                else                { di = r - t;  dj = -r; }
            }
            const bool inside = p < ring && ci + di >= 0 && ci + di < Ti && cj + dj >= 0 && cj + dj < Tj;
            const unsigned m = __ballot_sync(0xffffffffu, inside);
            if (k < __popc(m)) {
                if (inside && __popc(m & ((1u << threadIdx.x) - 1u)) == k) {
                    slot[0] = (ci + di) * kTileI;
                    slot[1] = (cj + dj) * a.tile_j;
                }
                found = 1;
            } else {
                k -= __popc(m);
            }
        }
    } else {
        stage_cams(a, s, b, 32);
    }
    __syncthreads();
    ti0 = slot[0];
    tj0 = slot[1];
}

// Cull the cameras (staged by tile_origin) against the tile.
// One thread per (camera, corner of the tile's voxel-centre box); the five
// visibility margins are max-reduced over the eight corners with shuffles.
__device__ inline void setup_tile(const SampleArgs& a, const CtaSmem& s, int ti0, int tj0) {
    const int tid = threadIdx.x;
    const GeoParams& g = a.g;
    const int n = tid >> 3, v = tid & 7;  // kThreads == 8 * BEV_MAX_CAMERAS
    if ((tid >> 5) * 4 < a.N) {           // warps holding at least one camera
        float m[5] = {-1e30f, -1e30f, -1e30f, -1e30f, -1e30f};
        if (n < a.N) {
            const int i1 = min(ti0 + kTileI, g.X) - 1, j1 = min(tj0 + a.tile_j, g.Y) - 1;
            const float px = voxel_centre(g.xmin, (v & 1) ? i1 : ti0, g.dx);
            const float py = voxel_centre(g.ymin, (v & 2) ? j1 : tj0, g.dy);
            const float pz = voxel_centre(g.zmin, (v & 4) ? g.Z - 1 : 0, g.dz);
            corner_margins(s.cams + n * kCamFloats, px, py, pz, g.img_w, g.img_h, m);
        }
#pragma unroll
        for (int q = 0; q < 5; ++q) {
            m[q] = fmaxf(m[q], __shfl_xor_sync(0xffffffffu, m[q], 1));
            m[q] = fmaxf(m[q], __shfl_xor_sync(0xffffffffu, m[q], 2));
            m[q] = fmaxf(m[q], __shfl_xor_sync(0xffffffffu, m[q], 4));
        }
        if (v == 0) s.act[64 + n] = (n < a.N) && m[0] >= 0.0f && m[1] >= 0.0f && m[2] >= 0.0f &&
                                    m[3] >= 0.0f && m[4] >= 0.0f;
    } else if (v == 0) {
        s.act[64 + n] = 0;
    }
    __syncthreads();
    if (tid < 32) {
        const bool vis = s.act[64 + tid] != 0;
        const unsigned mask = __ballot_sync(0xffffffffu, vis);
        if (vis) s.act[__popc(mask & ((1u << tid) - 1u))] = tid;
        if (tid == 0) s.act[32] = __popc(mask);
    }
    __syncthreads();
}

// Lanes of one cell: L consecutive lanes (sub = lane / L, ql = lane % L).
// Per-halfword unsigned min / max over the cell's lanes (two 16-bit fields
// reduced at once).
template <int L>
__device__ __forceinline__ unsigned group_min2(unsigned v) {
#pragma unroll
    for (int o = 1; o < L; o <<= 1) v = __vminu2(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

template <int L>
__device__ __forceinline__ unsigned group_max2(unsigned v) {
#pragma unroll
    for (int o = 1; o < L; o <<= 1) v = __vmaxu2(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Exclusive prefix of a per-group value (uniform within each group) over the
// G = 32 / L groups of the warp; *total receives the sum over all groups.
template <int L>
__device__ __forceinline__ int group_prefix(int size, int sub, int* total) {
    constexpr int G = 32 / L;
    int before = 0, all = 0;
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
        const int sz = __shfl_sync(0xffffffffu, size, gg * L);
        before += gg < sub ? sz : 0;
        all += sz;
    }
    *total = all;
    return before;
}

// Exact fixed point of the merged weights.  A contribution v = w / cnt (in
// [0, 1], fp32) is split into hi = RN(v 2^20) and lo = RN((v 2^20 - hi) 2^20),
// |lo| <= 2^19.  Both roundings to an integer are done by adding 1.5 * 2^23 in
// fp32 (the sum lies in [2^23, 2^24), where fp32 spacing is 1) and reading
// the integer off the bit pattern; the residual v 2^20 - hi is exact (one
// fma).  The halves are summed with 32-bit integer atomics (at most
// kZPerLaneMax * 32 contributions reach one entry, so neither overflows), and
// the total hi 2^-20 + lo 2^-40 is independent of the order of the additions.
// It is rounded to fp32 once.
constexpr float kTwo20 = 1048576.0f;
constexpr float kTwoM20 = 9.5367431640625e-07f;
constexpr float kTwoM40 = 9.094947017729282379150390625e-13f;
constexpr float kRound = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ void split_weight(float v, int& hi, int& lo) {
    const float t = __fmaf_rn(v, kTwo20, kRound);
    hi = __float_as_int(t) - __float_as_int(kRound);
    const float r = __fmaf_rn(v, kTwo20, -__fsub_rn(t, kRound));  // exact residual, |r| <= 0.5
    lo = __float_as_int(__fmaf_rn(r, kTwo20, kRound)) - __float_as_int(kRound);
}

// One cell group's projections for one camera in one height chunk: ZN bins
// per lane.
template <int ZN>
struct Items {
    float fx[ZN], fy[ZN];
    unsigned ok;  // bit t: item t is a valid voxel
};

// Project this lane's bins z = z0 + ql + L t (t < zn) of voxel column (x, y)
// through one camera.  UV: keep the image-plane position (u, v) in the fx /
// fy slots, for the multi-scale kernels to take to each level with at_level.
template <int L, int ZN, bool UV = false>
__device__ __forceinline__ Items<ZN> project_items(const float* cam, float x, float y, bool in_grid, int z0,
                                               int zn, int ql, const GeoParams& g) {
    Items<ZN> it;
    it.ok = 0;
#pragma unroll
    for (int t = 0; t < ZN; ++t) {
        it.fx[t] = 0.0f;
        it.fy[t] = 0.0f;
        const int z = z0 + ql + L * t;
        if (t < zn && in_grid && z < g.Z) {
            float fx, fy;
            ProjDetail det;
            if (project_point(cam, x, y, voxel_centre(g.zmin, z, g.dz), g, fx, fy, det)) {
                it.fx[t] = UV ? det.u : fx;
                it.fy[t] = UV ? det.v : fy;
                it.ok |= 1u << t;
            }
        }
    }
    return it;
}

// Sampling positions on one pyramid level from image-plane positions: the
// same two roundings as project_point, fx = u * sW - 0.5.
template <int ZN>
__device__ __forceinline__ Items<ZN> at_level(const Items<ZN>& uv, float sW, float sH) {
    Items<ZN> it;
    it.ok = uv.ok;
#pragma unroll
    for (int t = 0; t < ZN; ++t) {
        it.fx[t] = __fadd_rn(__fmul_rn(uv.fx[t], sW), -0.5f);
        it.fy[t] = __fadd_rn(__fmul_rn(uv.fy[t], sH), -0.5f);
    }
    return it;
}

// Patch of one cell group for one camera: box origin, height, width and
// offset in the warp's region; h == 0 when the cell has no valid voxel or the
// patches of the warp do not fit (then `overflow` is set for the cell).
struct Patch {
    int y0, x0, h, w, off;
    bool overflow;
};

// Box of texels the valid voxels of this lane's cell touch through one
// camera (uniform over the cell's lanes); h == 0 when the cell has no valid
// voxel.  `off` and `overflow` are set by merge_patches.
template <int L, int ZN>
__device__ __forceinline__ Patch patch_box(const Items<ZN>& it, int zn, int Hf, int Wf) {
    // lo = (ylo, xlo), hi = (yhi + 1, xhi + 1) as 16-bit fields (dimensions
    // are below 2^15); an empty cell keeps lo = (0xffff, 0xffff), hi = 0
    unsigned lo = 0xffffffffu, hi = 0u;
#pragma unroll
    for (int t = 0; t < ZN; ++t) {
        if (t < zn && (it.ok >> t & 1u)) {
            const int x0 = (int)floorf(it.fx[t]), y0 = (int)floorf(it.fy[t]);
            const unsigned l = ((unsigned)max(y0, 0) << 16) | (unsigned)max(x0, 0);
            const unsigned h = ((unsigned)min(y0 + 2, Hf) << 16) | (unsigned)min(x0 + 2, Wf);
            lo = __vminu2(lo, l);
            hi = __vmaxu2(hi, h);
        }
    }
    lo = group_min2<L>(lo);
    hi = group_max2<L>(hi);
    Patch p;
    p.y0 = (int)(lo >> 16);
    p.x0 = (int)(lo & 0xffffu);
    const bool any = hi != 0u;
    p.h = any ? (int)(hi >> 16) - p.y0 : 0;
    p.w = any ? (int)(hi & 0xffffu) - p.x0 : 0;
    p.off = 0;
    p.overflow = false;
    return p;
}

// Whether merging pays for one camera: the channel loop then walks the warp's
// largest patch two rows by two columns, against L * zn bin positions (four
// corners each) unmerged; merging itself costs about kMergeSteps such steps.
// Warp-uniform.
template <int L>
__device__ __forceinline__ bool merge_pays(const Patch& p, int zn, int merge_steps) {
    const int hmax = __reduce_max_sync(0xffffffffu, p.h);
    const int wmax = __reduce_max_sync(0xffffffffu, p.w);
    return ((hmax + 1) >> 1) * ((wmax + 1) >> 1) + merge_steps < L * zn;
}

// Placement, exact merge and fp32 rounding of one camera's weights for the
// warp's current cells into the boxes of patch_box.  rc[t] = 1 / cnt of item
// t.  Cells whose patches do not fit the region get h = 0 and `overflow`.
// Ends with the patch values readable by all lanes of the warp (fp32 at words
// [off, off + h * w) of `region`).
template <int L, int ZN>
__device__ __forceinline__ void merge_patches(Patch& p, const Items<ZN>& it, const float (&rc)[ZN], int zn,
                                              int sub, int ql, int Hf, int Wf, int* region) {
    int total;
    p.off = group_prefix<L>(p.h * p.w, sub, &total);
    p.overflow = p.off + p.h * p.w > kWarpPatchCap;
    if (p.overflow) p.h = 0;
    int* lo = region;
    int* hi = region + kWarpPatchCap;
    const int n = p.h * p.w;
    for (int e = ql; e < n; e += L) {
        lo[p.off + e] = 0;
        hi[p.off + e] = 0;
    }
    __syncwarp();
    if (n > 0) {
#pragma unroll
        for (int t = 0; t < ZN; ++t) {
            if (t < zn && (it.ok >> t & 1u)) {
                const Corners c = bilinear_corners(it.fx[t], it.fy[t]);
                const float ws[4] = {c.w00, c.w01, c.w10, c.w11};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int yy = c.y0 + (k >> 1), xx = c.x0 + (k & 1);
                    if ((unsigned)yy >= (unsigned)Hf || (unsigned)xx >= (unsigned)Wf) continue;
                    int qh, ql_;
                    split_weight(__fmul_rn(ws[k], rc[t]), qh, ql_);
                    const int e = p.off + (yy - p.y0) * p.w + (xx - p.x0);
                    if (!checked(e >= p.off && e < p.off + n && e < kWarpPatchCap, kCheckMerge)) continue;
                    if (ql_ != 0) atomicAdd(&lo[e], ql_);
                    if (qh != 0) atomicAdd(&hi[e], qh);
                }
            }
        }
    }
    __syncwarp();
    float* pf = reinterpret_cast<float*>(region);
    for (int e = ql; e < n; e += L) {
        pf[p.off + e] = __fadd_rn((float)hi[p.off + e] * kTwoM20, (float)lo[p.off + e] * kTwoM40);
    }
    __syncwarp();
}


}  // namespace row
}  // namespace bev
