// bev_tile.cuh -- CTA machinery of the dense Sampling-VT feature gradient
// (sm_100a): block-level geometry and shared scatters.
//
// FlashBEV's reading notes recompute the channel-independent geometry for
// every channel ("Method" item 3), name that recompute as the cost that grows
// with C ("Limitation", second point) and propose block-level geometry reuse
// ("Takeaway" 4).  Here one CTA owns an 8 x 8 tile of BEV cells of one batch
// item and one channel slice, and works camera by camera:
//
//   count    every (cell, height bin) voxel of the tile is tested against
//            every camera that can see the tile (exactly as the fixed fp32
//            order of the public header decides it); the valid cameras per
//            bin give the mean's 1 / cnt.  The same pass notes, per camera,
//            the leftmost feature column each cell's valid voxels reach.
//   groups   per camera, cells whose voxels start at the same feature column
//            are grouped, up to kGmax at a time.  A vertical column of voxels
//            projects to a near-vertical segment, so cells of one group share
//            nearly all of their texels (the union box is ~94% filled on the
//            seeded rigs): one reduction per texel then carries the whole
//            group's sum sum_g w_g dout_g, where a per-cell scatter would send
//            one per member.
//   sweep    warps take groups in turn, largest first.  For its group a warp
//            projects the members' voxels exactly (image-plane positions held
//            in registers), bounds their texels, sums the bilinear weights
//            w / cnt of the members' bins per (cell, texel) into a dense
//            [texel][member] array of its own shared-memory region -- 32-bit
//            integer atomics on an exact fixed point split in two words
//            (2^-20 and 2^-40), so the order of the additions does not
//            matter -- rounds them once to fp32, and walks the union box once.
//
// A group whose merged weights would not fit the warp's region is taken
// cell by cell; a cell whose box alone does not fit is swept bin by bin
// ("direct").  With several feature levels, a group is swept level by level
// on the same projections.  Every step is deterministic except the order of
// the global reductions.
#pragma once

#include <limits.h>
#include <math.h>

#include "bev_kernels.cuh"

namespace bev {

// Bounds-checked build (-DBEV_BOUNDS_CHECK).  Before each access whose
// address comes from geometry -- a group's texel box (every gather load and
// every gradient reduction lies inside it), a merge word, a group-table slot,
// an output or count index -- the kernels test it against its buffer or
// shared-memory region; a violation sets a bit of this translation unit's
// device error word and the access is skipped (no assert, no trap).  The host
// side reads and clears the word after the launch (bev_check_take) and turns
// a non-zero word into BEV_ERR_INTERNAL.  Without the flag every check is
// `true` and compiles away.
enum : unsigned {
    kCheckBox = 1u,       // a group's texel box outside its feature map
    kCheckMerge = 2u,     // a merge word outside the group's weight array
    kCheckGroups = 4u,    // a group-table slot or member cell out of range
    kCheckStore = 8u,     // an output / count / dout index outside its tensor
};
#ifdef BEV_BOUNDS_CHECK
static __device__ unsigned g_check_word;
__device__ __forceinline__ bool checked(bool ok, unsigned code) {
    if (!ok) atomicOr(&g_check_word, code);
    return ok;
}
// Read and clear the word of this translation unit (after the stream has
// drained); host side.
static inline unsigned check_take() {
    unsigned w = 0, z = 0;
    if (cudaMemcpyFromSymbol(&w, g_check_word, sizeof(w)) != cudaSuccess) w = ~0u;
    cudaMemcpyToSymbol(g_check_word, &z, sizeof(z));
    return w;
}
#else
__device__ __forceinline__ bool checked(bool, unsigned) { return true; }
#endif

constexpr int kCells = kTileI * kTileJ;  // cell = ci * kTileJ + cj
constexpr int kZc = 16;                  // height bins per chunk of the count
constexpr int kGmax = 8;                 // cells per group
constexpr int kWarpEntries = 512;        // merged-weight entries of a warp's region
constexpr int kTileCtas = 2;             // CTAs per SM
constexpr int kMaxActive = 32;           // active cameras of a tile (at most BEV_MAX_CAMERAS)
static_assert(kThreads == 256 && kCells == 64, "the tile machinery assumes 256 threads and 64 cells");

struct Group {
    int n;                     // member cells, 1 .. kGmax
    unsigned char cell[kGmax];  // member cell indices
    int pad;
};
static_assert(sizeof(Group) == 16, "group descriptor size");

// Control words (ints) of the CTA.
enum {
    kCtlActive = 0,    // [0, 32) active camera ids
    kCtlNA = 32,       // number of active cameras
    kCtlOrigin = 40,   // [40, 41] tile origin
    kCtlGroups = 48,   // groups of the current view
    kCtlNext = 50,     // next group to sweep (warps take groups in turn)
    kCtlSizeHist = 52, // [52, 61) groups per size, then per-size cursors
    kCtlCull = 64,     // [64, 96) per-camera visibility flags of the cull
    kCtlOrder = 96,    // [96, 160) groups, largest first
    kCtlBucket = 160,  // [160, 224) per-column bucket counters
    kCtlGbase = 224,   // [224, 288) first group of each bucket
    kCtlWords = 288,
};

// Byte offsets of the CTA's shared-memory regions.  cpl = channels per lane.
struct TileLayout {
    size_t cams, ctl, rc, xlo, grp, wqh, wql, tile, total;
    int tile_stride;  // floats per cell row of the [cell][channel] tile
};

__host__ __device__ inline TileLayout tile_layout(int N, int cpl) {
    TileLayout l;
    size_t b = 0;
    auto take = [&](size_t bytes) {
        const size_t at = b;
        b += (bytes + 15) & ~(size_t)15;
        return at;
    };
    l.cams = take(sizeof(float) * N * kCamFloats);
    l.ctl = take(sizeof(int) * kCtlWords);
    l.rc = take(sizeof(float) * kCells * kZc);
    l.xlo = take(sizeof(unsigned short) * kMaxActive * kCells);
    l.grp = take(sizeof(Group) * kCells);
    l.wqh = take(sizeof(unsigned) * kWarps * kWarpEntries);
    l.wql = take(sizeof(unsigned) * kWarps * kWarpEntries);
    l.tile_stride = 32 * cpl + 4;
    l.tile = take(sizeof(float) * kCells * l.tile_stride);
    l.total = b;
    return l;
}

struct TileSm {
    float* cams;
    int* ctl;
    float* rc;            // [cell * kZc + bin]: 1 / cnt (0 when no camera sees the voxel)
    unsigned short* xlo;  // [active camera][cell]: leftmost level-0 column of its valid voxels (0xffff: none)
    Group* grp;
    unsigned* wqh;   // per warp: merge words in 2^-20 units, then the fp32 weights
    unsigned* wql;   // per warp: merge words in 2^-40 units
    float* tile;
    int tile_stride;
};

__device__ __forceinline__ TileSm carve_tile(unsigned char* smem, int N, int cpl) {
    const TileLayout l = tile_layout(N, cpl);
    TileSm s;
    s.cams = reinterpret_cast<float*>(smem + l.cams);
    s.ctl = reinterpret_cast<int*>(smem + l.ctl);
    s.rc = reinterpret_cast<float*>(smem + l.rc);
    s.xlo = reinterpret_cast<unsigned short*>(smem + l.xlo);
    s.grp = reinterpret_cast<Group*>(smem + l.grp);
    s.wqh = reinterpret_cast<unsigned*>(smem + l.wqh);
    s.wql = reinterpret_cast<unsigned*>(smem + l.wql);
    s.tile = reinterpret_cast<float*>(smem + l.tile);
    s.tile_stride = l.tile_stride;
    return s;
}

// ---------------------------------------------------------------------------
// Tile set-up: ring order, calibrations, camera culling
// ---------------------------------------------------------------------------

// Calibrations of batch item b into shared memory: E rows 0..2, then K rows
// 0..1, per camera; threads first .. kThreads - 1 take one float at a time.
__device__ __forceinline__ void stage_calibrations(const SampleArgs& a, float* cams, int b, int first) {
    for (int t = (int)threadIdx.x - first; t < a.N * kCamFloats; t += kThreads - first) {
        const int n = t / kCamFloats, r = t - n * kCamFloats;
        cams[t] = r < 12 ? a.E[((size_t)b * a.N + n) * 16 + r] : a.K[((size_t)b * a.N + n) * 9 + (r - 12)];
    }
}

// Tile of this CTA.  Tiles are issued in rings of increasing Chebyshev
// distance from the centre tile of the grid: for rigs mounted near the grid
// centre the nearest voxels see the most texels, so the heaviest tiles start
// first and the light outer ring fills the tail of the launch (any order
// gives the same results).  Warp 0 maps the block index to its ring -- its
// lanes test 32 candidate rings at a time -- then finds the position inside
// the ring with ballots; the other warps meanwhile stage the calibrations.
__device__ inline void locate_tile(const SampleArgs& a, const TileSm& s, int b, int& ti0, int& tj0) {
    const int Ti = a.tiles_i, Tj = a.tiles_j;
    int* slot = s.ctl + kCtlOrigin;
    if (threadIdx.x < 32) {
        const int ci = (Ti - 1) >> 1, cj = (Tj - 1) >> 1;
        auto area = [&](int r) -> int {  // tiles within Chebyshev distance r of the centre
            if (r < 0) return 0;
            const int h = min(ci + r, Ti - 1) - max(ci - r, 0) + 1;
            const int w = min(cj + r, Tj - 1) - max(cj - r, 0) + 1;
            return h * w;
        };
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
                    slot[1] = (cj + dj) * kTileJ;
                }
                found = 1;
            } else {
                k -= __popc(m);
            }
        }
    } else {
        stage_calibrations(a, s.cams, b, 32);
    }
    __syncthreads();
    ti0 = slot[0];
    tj0 = slot[1];
}

// Cull the cameras against the tile: one thread per (camera, corner of the
// tile's voxel-centre box); the five visibility margins are max-reduced over
// the eight corners with shuffles.  Conservative: a culled camera sees no
// voxel of the tile.  Leaves the active camera ids in ctl[0, nA).
__device__ inline void cull_cameras(const SampleArgs& a, const TileSm& s, int ti0, int tj0) {
    const int tid = threadIdx.x;
    const GeoParams& g = a.g;
    const int n = tid >> 3, v = tid & 7;  // kThreads == 8 * BEV_MAX_CAMERAS
    int* flag = s.ctl + kCtlCull;
    if ((tid >> 5) * 4 < a.N) {
        float m[5] = {-1e30f, -1e30f, -1e30f, -1e30f, -1e30f};
        if (n < a.N) {
            const int i1 = min(ti0 + kTileI, g.X) - 1, j1 = min(tj0 + kTileJ, g.Y) - 1;
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
        if (v == 0)
            flag[n] = (n < a.N) && m[0] >= 0.0f && m[1] >= 0.0f && m[2] >= 0.0f && m[3] >= 0.0f && m[4] >= 0.0f;
    } else if (v == 0) {
        flag[n] = 0;
    }
    __syncthreads();
    if (tid < 32) {
        const bool vis = flag[tid] != 0;
        const unsigned mask = __ballot_sync(0xffffffffu, vis);
        if (vis) s.ctl[kCtlActive + __popc(mask & ((1u << tid) - 1u))] = tid;
        if (tid == 0) s.ctl[kCtlNA] = __popc(mask);
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// Per-voxel passes.  Items (cell, bin of the chunk) map to threads with LZ
// consecutive lanes per cell, LZ the power of two >= the chunk's bins.
// ---------------------------------------------------------------------------

struct ItemMap {
    int LZ;      // lanes per cell
    int passes;  // passes over the tile's cells
    int cpp;     // cells per pass
};

__device__ __forceinline__ ItemMap item_map(int zc) {
    ItemMap m;
    m.LZ = zc <= 1 ? 1 : zc <= 2 ? 2 : zc <= 4 ? 4 : zc <= 8 ? 8 : 16;
    m.cpp = kThreads / m.LZ;
    m.passes = (kCells + m.cpp - 1) / m.cpp;
    return m;
}

// One camera's constants (E rows 0..2, K rows 0..1) held in registers.
struct CamRegs {
    float c[kCamFloats];
};

__device__ __forceinline__ CamRegs load_cam(const float* cam) {
    CamRegs r;
#pragma unroll
    for (int k = 0; k < kCamFloats; ++k) r.c[k] = cam[k];
    return r;
}

// Validity of one voxel in one camera, decided exactly as the fixed fp32
// order of project_point decides it.  Depth and the homogeneous image
// coordinates are computed in that order; the divides are taken with an
// approximate quotient first and settled by the IEEE divide only when the
// approximate position lies within 1e-5 (relative, at least 1e-5 px) of an
// image edge, far outside the error of the approximation.  `uv` receives the
// position the decision used (approximate or exact).
__device__ __forceinline__ bool voxel_visible(const CamRegs& cr, float x, float y, float z, const GeoParams& g,
                                              float2& uv) {
    const float* cam = cr.c;
    const float pcx = cam_row(cam + 0, x, y, z);
    const float pcy = cam_row(cam + 4, x, y, z);
    const float depth = cam_row(cam + 8, x, y, z);
    if (!(depth > 0.1f)) return false;
    const float* k = cam + 12;
    float uh = __fadd_rn(__fmul_rn(k[0], pcx), __fmul_rn(k[1], pcy));
    uh = __fadd_rn(uh, __fmul_rn(k[2], depth));
    float vh = __fadd_rn(__fmul_rn(k[3], pcx), __fmul_rn(k[4], pcy));
    vh = __fadd_rn(vh, __fmul_rn(k[5], depth));
    if (depth < 1e30f) {
        const float ua = __fdividef(uh, depth), va = __fdividef(vh, depth);
        const float mu = 1e-5f * fmaxf(fabsf(ua), 1.0f), mv = 1e-5f * fmaxf(fabsf(va), 1.0f);
        uv = make_float2(ua, va);
        if (ua < -mu || ua > g.img_w + mu || va < -mv || va > g.img_h + mv) return false;
        if (ua > mu && ua < g.img_w - mu && va > mv && va < g.img_h - mv) return true;
    }
    const float u = __fdiv_rn(uh, depth), v = __fdiv_rn(vh, depth);
    uv = make_float2(u, v);
    return u >= 0.0f && u <= g.img_w && v >= 0.0f && v <= g.img_h;
}

__device__ __forceinline__ float2 no_uv() { return make_float2(__int_as_float(0x7fc00000), 0.0f); }

// Exact image-plane position of a voxel when it is valid (as project_point
// gives it), else x = NaN.
__device__ __forceinline__ float2 voxel_exact(const CamRegs& cr, float x, float y, float z, const GeoParams& g) {
    float fx, fy;
    ProjDetail det;
    if (project_point(cr.c, x, y, z, g, fx, fy, det)) return make_float2(det.u, det.v);
    return no_uv();
}

// Sampling position of an image-plane position on a level of scale (sW, sH):
// the two roundings of project_point, fx = u * sW - 0.5.
__device__ __forceinline__ void level_position(float2 uv, float sW, float sH, float& fx, float& fy) {
    fx = __fadd_rn(__fmul_rn(uv.x, sW), -0.5f);
    fy = __fadd_rn(__fmul_rn(uv.y, sH), -0.5f);
}

// Count pass over the bins [z0, z0 + zc): 1 / cnt per item, and per (active
// camera, cell) the leftmost level-0
// feature column the cell's valid voxels reach (from the position the
// validity test used; it only steers the grouping).  Cameras are the outer
// loop, so each camera's constants are read once per thread.
constexpr int kMaxPasses = kCells * 16 / kThreads;  // item passes at 16 lanes per cell

__device__ inline void count_pass(const SampleArgs& a, const TileSm& s, int ti0, int tj0, int z0, int zc) {
    const GeoParams& g = a.g;
    const ItemMap im = item_map(zc);
    const int nA = s.ctl[kCtlNA];
    const int zz = threadIdx.x % im.LZ;
    const float sW0 = a.lv.sW[0];
    const int W0 = a.lv.Wf[0];
    bool in[kMaxPasses];
    float px[kMaxPasses], py[kMaxPasses], pz[kMaxPasses];
    int cnt[kMaxPasses];
#pragma unroll
    for (int p = 0; p < kMaxPasses; ++p) {
        const int cell = p * im.cpp + (int)threadIdx.x / im.LZ;
        const int i = ti0 + cell / kTileJ, j = tj0 + cell % kTileJ;
        in[p] = p < im.passes && cell < kCells && zz < zc && i < g.X && j < g.Y;
        px[p] = voxel_centre(g.xmin, i, g.dx);
        py[p] = voxel_centre(g.ymin, j, g.dy);
        pz[p] = voxel_centre(g.zmin, z0 + zz, g.dz);
        cnt[p] = 0;
    }
    for (int aa = 0; aa < nA; ++aa) {
        const CamRegs cr = load_cam(s.cams + s.ctl[kCtlActive + aa] * kCamFloats);
#pragma unroll
        for (int p = 0; p < kMaxPasses; ++p) {
            if (p >= im.passes) break;
            float2 uv;
            unsigned x0 = 0xffffu;
            if (in[p] && voxel_visible(cr, px[p], py[p], pz[p], g, uv)) {
                ++cnt[p];
                x0 = (unsigned)min(max((int)floorf(__fmaf_rn(uv.x, sW0, -0.5f)), 0), W0 - 1);
            }
            // leftmost column over the cell's lanes (warps with none skip it)
            if (__any_sync(0xffffffffu, x0 != 0xffffu)) {
                for (int o = 1; o < im.LZ; o <<= 1) x0 = min(x0, __shfl_xor_sync(0xffffffffu, x0, o));
            }
            const int cell = p * im.cpp + (int)threadIdx.x / im.LZ;
            if (zz == 0 && cell < kCells) s.xlo[aa * kCells + cell] = (unsigned short)x0;
        }
    }
#pragma unroll
    for (int p = 0; p < kMaxPasses; ++p) {
        if (p >= im.passes) break;
        const int cell = p * im.cpp + (int)threadIdx.x / im.LZ;
        if (cell < kCells && zz < zc) s.rc[cell * kZc + zz] = cnt[p] > 0 ? __frcp_rn((float)cnt[p]) : 0.0f;
    }
}

// Tiles that one camera alone can see (one active camera after the cull):
// every valid voxel then has cnt = 1, so 1 / cnt is 1 and the geometry is
// needed only to form the groups.  A cell joins the camera's groups unless
// the five validity margins of corner_margins, taken at the two end voxels
// of its column in the chunk (each margin is linear along the column, so its
// maximum is at an end), rule out every voxel; its key is the leftmost
// level-0 feature column the two end voxels reach (an approximation, which
// only steers the grouping; the sweep projects every voxel exactly).  A
// cell that joins with no valid voxel adds nothing.
__device__ inline void single_camera_pass(const SampleArgs& a, const TileSm& s, int ti0, int tj0, int z0, int zc) {
    const GeoParams& g = a.g;
    for (int t = threadIdx.x; t < kCells * kZc; t += kThreads) s.rc[t] = 1.0f;
    if (threadIdx.x < kCells) {
        const int cell = threadIdx.x;
        const int i = ti0 + cell / kTileJ, j = tj0 + cell % kTileJ;
        unsigned short key = 0xffffu;
        if (i < g.X && j < g.Y) {
            const float* cam = s.cams + s.ctl[kCtlActive] * kCamFloats;
            const float px = voxel_centre(g.xmin, i, g.dx), py = voxel_centre(g.ymin, j, g.dy);
            const float sW0 = a.lv.sW[0];
            const int W0 = a.lv.Wf[0];
            float m[5] = {-1e30f, -1e30f, -1e30f, -1e30f, -1e30f};
            int x0 = INT_MAX;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float pz = voxel_centre(g.zmin, e ? z0 + zc - 1 : z0, g.dz);
                float me[5];
                corner_margins(cam, px, py, pz, g.img_w, g.img_h, me);
#pragma unroll
                for (int q = 0; q < 5; ++q) m[q] = fmaxf(m[q], me[q]);
                const float depth = cam_row(cam + 8, px, py, pz);
                if (depth > 0.1f) {
                    const float* k = cam + 12;
                    const float uh = k[0] * cam_row(cam, px, py, pz) + k[1] * cam_row(cam + 4, px, py, pz) + k[2] * depth;
                    x0 = min(x0, min(max((int)floorf(__fdividef(uh, depth) * sW0 - 0.5f), 0), W0 - 1));
                }
            }
            if (m[0] >= 0.0f && m[1] >= 0.0f && m[2] >= 0.0f && m[3] >= 0.0f && m[4] >= 0.0f)
                key = (unsigned short)(x0 == INT_MAX ? 0 : x0);
        }
        s.xlo[cell] = key;
    }
}

// ---------------------------------------------------------------------------
// Grouping (warp 0)
// ---------------------------------------------------------------------------

__device__ __forceinline__ int warp_inclusive_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    return v;
}


// Groups of the current view from the cells' boxes: cells whose boxes start
// at the same feature column form buckets, split into groups of at most
// kGmax cells; cells more than 63 columns right of the leftmost form groups
// of their own.  The groups are listed largest first, so that the warps that
// take them in turn finish close together.  Warp 0 only.
__device__ inline void form_groups(const TileSm& s, const unsigned short* xl) {
    const int lane = threadIdx.x & 31;
    int* ctl = s.ctl;
    int* bcnt = ctl + kCtlBucket;
    int* gbase = ctl + kCtlGbase;
    int* hist = ctl + kCtlSizeHist;  // [0, kGmax]: count per size, reused as cursors
    bool val[2];
    int xlo[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int c = lane + 32 * k;
        xlo[k] = (int)xl[c];
        val[k] = xlo[k] != 0xffff;
    }
    const int xm = __reduce_min_sync(0xffffffffu, (unsigned)min(val[0] ? xlo[0] : 0xffff, val[1] ? xlo[1] : 0xffff));
    bcnt[lane] = 0;
    bcnt[lane + 32] = 0;
    if (lane <= kGmax) hist[lane] = 0;
    __syncwarp();
    int key[2], rank[2] = {0, 0};
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        key[k] = val[k] ? xlo[k] - xm : INT_MAX;
        if (key[k] < 64) rank[k] = atomicAdd(&bcnt[key[k]], 1);
    }
    __syncwarp();
    const int nb0 = bcnt[lane], nb1 = bcnt[lane + 32];
    const int gb0 = (nb0 + kGmax - 1) / kGmax, gb1 = (nb1 + kGmax - 1) / kGmax;
    const int in0 = warp_inclusive_scan(gb0), in1 = warp_inclusive_scan(gb1);
    const int t0 = __shfl_sync(0xffffffffu, in0, 31);
    const int nbg = t0 + __shfl_sync(0xffffffffu, in1, 31);
    gbase[lane] = in0 - gb0;
    gbase[lane + 32] = t0 + in1 - gb1;
    const unsigned far0 = __ballot_sync(0xffffffffu, val[0] && key[0] >= 64);
    const unsigned far1 = __ballot_sync(0xffffffffu, val[1] && key[1] >= 64);
    const int ng = nbg + __popc(far0) + __popc(far1);
    __syncwarp();
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int c = lane + 32 * k;
        if (val[k]) {
            int gi, slot, n;
            if (key[k] < 64) {
                gi = gbase[key[k]] + rank[k] / kGmax;
                slot = rank[k] % kGmax;
                n = min(kGmax, bcnt[key[k]] - (rank[k] / kGmax) * kGmax);
            } else {
                gi = nbg + (k == 0 ? __popc(far0 & lt) : __popc(far0) + __popc(far1 & lt));
                slot = 0;
                n = 1;
            }
            if (!checked(gi >= 0 && gi < kCells && slot < kGmax, kCheckGroups)) continue;
            s.grp[gi].cell[slot] = (unsigned char)c;
            if (slot == 0) {
                s.grp[gi].n = n;
                atomicAdd(&hist[n], 1);
            }
        }
    }
    __syncwarp();
    // largest first: groups of size n start after all larger ones
    if (lane == 0) {
        int at = 0;
        for (int n = kGmax; n >= 1; --n) {
            const int c = hist[n];
            hist[n] = at;
            at += c;
        }
        ctl[kCtlGroups] = ng;
        ctl[kCtlNext] = 0;
    }
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int gi = lane + 32 * k;
        if (gi < ng) {
            const int n = s.grp[gi].n;
            if (!checked(n >= 1 && n <= kGmax, kCheckGroups)) continue;
            const int pos = atomicAdd(&hist[n], 1);
            if (checked(pos >= 0 && pos < kCells, kCheckGroups)) ctl[kCtlOrder + pos] = gi;
        }
    }
}

// ---------------------------------------------------------------------------
// Per-warp merge of one group's weights
// ---------------------------------------------------------------------------

// Exact fixed point of the merged weights.  A contribution v = w / cnt (in
// [0, 1], fp32) is split into hi = RN(v 2^20) and lo = RN((v - hi 2^-20)
// 2^40), |lo| <= 2^19; both splits are exact integer roundings done by adding
// 1.5 * 2^23 in fp32 (the sum lies in [2^23, 2^24), where the spacing of fp32
// is 1, so the addition rounds to an integer) and the residual is exact.  At
// most kZc contributions reach one entry, so the word sums stay within 2^24 in
// magnitude and convert to fp32 exactly: the merged weight
// hi 2^-20 + lo 2^-40 does not depend on the order of the additions and is
// rounded once.
constexpr float kTwo20 = 1048576.0f;
constexpr float kTwoM20 = 9.5367431640625e-07f;
constexpr float kTwoM40 = 9.094947017729282379150390625e-13f;
constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
static_assert(kZc * (1 << 20) <= (1 << 24), "merge words must stay exact in fp32");

__device__ __forceinline__ void split_weight(float v, int& hi, int& lo) {
    const float t = __fmaf_rn(v, kTwo20, kRound);
    hi = __float_as_int(t) - __float_as_int(kRound);
    const float r = __fmaf_rn(v, kTwo20, -__fsub_rn(t, kRound));  // exact residual, |r| <= 0.5
    lo = __float_as_int(__fmaf_rn(r, kTwo20, kRound)) - __float_as_int(kRound);
}

// A group's voxels, as the warp that sweeps the group holds them: lane l
// takes bin l % LZ of member cell t * (32 / LZ) + l / LZ at step t.
constexpr int kItemSteps = kGmax * kZc / 32;

struct GroupItems {
    float2 uv[kItemSteps];  // exact image-plane position; x = NaN when the camera does not see the voxel
};

// Exact projections of the members' voxels through one camera.
__device__ inline GroupItems project_members(const SampleArgs& a, const TileSm& s, const unsigned char* cells, int n,
                                             int cam, int ti0, int tj0, int z0, int zc) {
    const GeoParams& g = a.g;
    const int lane = threadIdx.x & 31;
    const ItemMap im = item_map(zc);
    const int zz = lane % im.LZ, per = 32 / im.LZ;
    const CamRegs cr = load_cam(s.cams + cam * kCamFloats);
    GroupItems it;
#pragma unroll
    for (int t = 0; t < kItemSteps; ++t) {
        it.uv[t] = no_uv();
        const int k = t * per + lane / im.LZ;
        if (t * per < n && k < n && zz < zc) {
            const int cell = cells[k];
            const int i = ti0 + cell / kTileJ, j = tj0 + cell % kTileJ;
            it.uv[t] = voxel_exact(cr, voxel_centre(g.xmin, i, g.dx), voxel_centre(g.ymin, j, g.dy),
                                   voxel_centre(g.zmin, z0 + zz, g.dz), g);
        }
    }
    return it;
}

// A set of member cells and the union of their texel boxes on the current
// level, as one warp processes it.  When the map allows, the box is widened
// to even height and width inside the map (extra rows and columns carry zero
// weight), so that the sweep's two-by-two steps need no edge predicates.
struct Members {
    int n;                      // cells (1 .. kGmax)
    int slots;                  // weights per texel (1, 2, 4 or 8)
    int y0, x0, h, w;           // union box
    bool even;                  // h and w are even
    const unsigned char* cell;  // member cell indices (shared memory)
    int entries;                // h * w * slots rounded up to 4
};

__device__ __forceinline__ int slots_for(int n) { return n == 1 ? 1 : n == 2 ? 2 : n <= 4 ? 4 : 8; }

// Union of the bilinear corners (inside the map) of the group's valid voxels
// on one level; warp-uniform.  Every member has a valid voxel, so the box is
// not empty.
__device__ __forceinline__ Members members_box(const GroupItems& it, const unsigned char* cells, int n, int Hf, int Wf,
                                               float sW, float sH) {
    unsigned lo = 0xffffffffu, hi = 0u;
#pragma unroll
    for (int t = 0; t < kItemSteps; ++t) {
        if (!isnan(it.uv[t].x)) {
            float fx, fy;
            level_position(it.uv[t], sW, sH, fx, fy);
            const int x0 = (int)floorf(fx), y0 = (int)floorf(fy);
            lo = __vminu2(lo, ((unsigned)max(y0, 0) << 16) | (unsigned)max(x0, 0));
            hi = __vmaxu2(hi, ((unsigned)min(y0 + 2, Hf) << 16) | (unsigned)min(x0 + 2, Wf));
        }
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        lo = __vminu2(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = __vmaxu2(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    Members m;
    m.n = n;
    m.slots = slots_for(n);
    m.y0 = (int)(lo >> 16);
    m.x0 = (int)(lo & 0xffffu);
    m.h = (int)(hi >> 16) - m.y0;
    m.w = (int)(hi & 0xffffu) - m.x0;
    const int h2 = (m.h + 1) & ~1, w2 = (m.w + 1) & ~1;
    m.even = h2 <= Hf && w2 <= Wf;
    if (m.even) {  // the widened box still covers the union and stays inside the map
        m.y0 = min(m.y0, Hf - h2);
        m.x0 = min(m.x0, Wf - w2);
        m.h = h2;
        m.w = w2;
    }
    m.cell = cells;
    m.entries = (m.h * m.w * m.slots + 3) & ~3;
    return m;
}

// Whether a group's box lies inside its feature map (every gather load and
// every gradient reduction of the group is inside the box); always true
// outside the checked build.
__device__ __forceinline__ bool box_inside(const Members& m, int Hf, int Wf) {
    return checked(m.h <= 0 || m.w <= 0 || (m.y0 >= 0 && m.x0 >= 0 && m.y0 + m.h <= Hf && m.x0 + m.w <= Wf),
                   kCheckBox);
}

// Sum w / cnt of every valid voxel of the members into the warp's region
// ([texel of the union box][member] words), then round each entry to fp32
// in place (the weights replace the 2^-20 words; the 2^-40 words are
// cleared).  Ends with the weights readable by the whole warp.
__device__ inline void merge_members(const TileSm& s, const Members& m, const GroupItems& it, int zc, int Hf, int Wf,
                                     float sW, float sH, unsigned* wh, unsigned* wl) {
    const int lane = threadIdx.x & 31;
    const ItemMap im = item_map(zc);
    const int zz = lane % im.LZ, per = 32 / im.LZ;
    const int rowe = m.w * m.slots;
#pragma unroll
    for (int t = 0; t < kItemSteps; ++t) {
        const int k = t * per + lane / im.LZ;
        if (isnan(it.uv[t].x) || k >= m.n) continue;
        float fx, fy;
        level_position(it.uv[t], sW, sH, fx, fy);
        const Corners c = bilinear_corners(fx, fy);
        const float rc = s.rc[m.cell[k] * kZc + zz];
        const bool cx0 = (unsigned)c.x0 < (unsigned)Wf, cx1 = (unsigned)(c.x0 + 1) < (unsigned)Wf;
        const bool cy0 = (unsigned)c.y0 < (unsigned)Hf, cy1 = (unsigned)(c.y0 + 1) < (unsigned)Hf;
        const int e = ((c.y0 - m.y0) * m.w + (c.x0 - m.x0)) * m.slots + k;
        const float ws[4] = {c.w00, c.w01, c.w10, c.w11};
        const bool ok[4] = {cy0 && cx0, cy0 && cx1, cy1 && cx0, cy1 && cx1};
        const int off[4] = {0, m.slots, rowe, rowe + m.slots};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float v = __fmul_rn(ws[q], rc);
            if (!ok[q] || v == 0.0f) continue;
            int hi, lo;
            split_weight(v, hi, lo);
            const int eq = e + off[q];
            if (!checked(eq >= 0 && eq < m.entries && eq < kWarpEntries && k < m.slots, kCheckMerge)) continue;
            if (hi != 0) atomicAdd(&wh[eq], (unsigned)hi);
            if (lo != 0) atomicAdd(reinterpret_cast<int*>(wl) + eq, lo);
        }
    }
    __syncwarp();
    for (int e = 4 * lane; e < m.entries; e += 128) {
        const uint4 qh = *reinterpret_cast<const uint4*>(wh + e);
        const int4 ql = *reinterpret_cast<const int4*>(wl + e);
        *reinterpret_cast<uint4*>(wl + e) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<float4*>(wh + e) =
            make_float4(__fadd_rn((float)qh.x * kTwoM20, (float)ql.x * kTwoM40),
                        __fadd_rn((float)qh.y * kTwoM20, (float)ql.y * kTwoM40),
                        __fadd_rn((float)qh.z * kTwoM20, (float)ql.z * kTwoM40),
                        __fadd_rn((float)qh.w * kTwoM20, (float)ql.w * kTwoM40));
    }
    __syncwarp();
}

// Clear the weights of the warp's region after its sweep (the region must be
// zero before the next merge).
__device__ __forceinline__ void clear_members(const Members& m, unsigned* wh) {
    __syncwarp();
    const int lane = threadIdx.x & 31;
    for (int e = 4 * lane; e < m.entries; e += 128) *reinterpret_cast<uint4*>(wh + e) = make_uint4(0u, 0u, 0u, 0u);
    __syncwarp();
}

// S weights of one texel of a group's array.
template <int S>
__device__ __forceinline__ void load_weights(float (&wt)[S], const float* p) {
    if constexpr (S == 8) {
        const float4 a = *reinterpret_cast<const float4*>(p);
        const float4 b = *reinterpret_cast<const float4*>(p + 4);
        wt[0] = a.x; wt[1] = a.y; wt[2] = a.z; wt[3] = a.w;
        wt[4] = b.x; wt[5] = b.y; wt[6] = b.z; wt[7] = b.w;
    } else if constexpr (S == 4) {
        const float4 a = *reinterpret_cast<const float4*>(p);
        wt[0] = a.x; wt[1] = a.y; wt[2] = a.z; wt[3] = a.w;
    } else if constexpr (S == 2) {
        const float2 a = *reinterpret_cast<const float2*>(p);
        wt[0] = a.x; wt[1] = a.y;
    } else {
        wt[0] = *p;
    }
}

}  // namespace bev
