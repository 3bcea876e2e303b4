// bev_tile.cuh -- CTA machinery shared by the dense Sampling-VT forward and
// backward kernels (sm_100a): block-level geometry and texel reuse.
//
// FlashBEV's reading notes recompute the channel-independent geometry for
// every channel ("Method" item 3), name that recompute as the cost that grows
// with C ("Limitation", second point) and propose block-level geometry reuse
// ("Takeaway" 4).  Here one CTA owns an 8 x 8 tile of BEV cells of one batch
// item and one channel slice, and works camera by camera:
//
//   count    every (cell, height bin) voxel of the tile is tested against
//            every camera that can see the tile; the valid cameras per bin
//            give the mean's 1 / cnt.
//   project  per camera, the image-plane position (u, v) of every voxel the
//            camera sees, in the fixed fp32 order of the public header.
//   boxes    per camera and feature level, the texel box each cell's valid
//            samples touch (bilinear corners inside the map).
//   groups   cells whose boxes start at the same feature column are grouped,
//            up to kGmax at a time.  A vertical column of voxels projects to
//            a near-vertical segment, so cells of one group share nearly all
//            of their texels (the union box is ~94% filled on the seeded
//            rigs): a texel's channel vector is then loaded once for the
//            whole group and applied to every member cell from registers.
//   merge    the bilinear weights w / cnt of all bins of a cell are summed
//            per (cell, texel) into a dense [texel][slot] array per group,
//            with integer atomics on an exact 2^-40 fixed point (order of the
//            additions does not matter), then rounded once to fp32.
//   sweep    warps take groups in turn and walk each union box once (the
//            forward gathers, the backward scatters).
//
// A group's merged weights that would not fit the shared-memory budget go
// in further rounds; a group whose box alone is too large for a round is
// swept bin by bin instead ("direct").  Every step is deterministic except
// the order of the backward's global reductions.
#pragma once

#include <limits.h>
#include <math.h>

#include "bev_kernels.cuh"

namespace bev {

constexpr int kCells = kTileI * kTileJ;  // cell = ci * kTileJ + cj
constexpr int kZc = 16;                  // height bins per chunk of the count
constexpr int kGmax = 8;                 // cells per group
constexpr int kEntries = 2048;           // merged-weight entries per round
constexpr int kTileCtas = 2;             // CTAs per SM
static_assert(kThreads == 256 && kCells == 64, "the tile machinery assumes 256 threads and 64 cells");

struct Group {
    int y0, x0, h, w;  // union box of the member cells' texel boxes
    int off;           // first fp32 weight of the group in its round
    int n;             // member cells, 1 .. kGmax
    int slots;         // weights stored per texel: 1, 2, 4 or 8 (>= n)
    int round;         // merge round
    int direct;        // 1: swept bin by bin (box too large for a round)
    int pad[3];
    unsigned char cell[kGmax];
};
static_assert(sizeof(Group) == 56, "group descriptor size");

// Control words (ints) of the CTA.
enum {
    kCtlActive = 0,    // [0, 32) active camera ids
    kCtlNA = 32,       // number of active cameras
    kCtlOrigin = 40,   // [40, 41] tile origin
    kCtlGroups = 48,   // groups of the current view
    kCtlRounds = 49,   // merge rounds of the current view
    kCtlNext = 50,     // next group to sweep (warps take groups in turn)
    kCtlCull = 64,     // [64, 96) per-camera visibility flags of the cull
    kCtlRstart = 128,  // [128, 128 + 65) first group of each round
    kCtlNent = 208,    // [208, 208 + 64) weight entries of each round
    kCtlBucket = 288,  // [288, 352) per-column bucket counters
    kCtlGbase = 352,   // [352, 416) first group of each bucket
    kCtlBounds = 416,  // [416, 416 + 4 * 64) union bounds while grouping
    kCtlWords = 672,
};

// Byte offsets of the CTA's shared-memory regions.  cpl = channels per lane.
struct TileLayout {
    size_t cams, ctl, rc, vmask, uv, box, cellg, grp, wq, wf, tile, total;
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
    l.vmask = take(sizeof(unsigned) * kCells * kZc);
    l.uv = take(sizeof(float2) * kCells * kZc);
    l.box = take(sizeof(unsigned) * 2 * kCells);
    l.cellg = take(sizeof(int) * kCells);
    l.grp = take(sizeof(Group) * kCells);
    l.wq = take(sizeof(unsigned long long) * kEntries);
    l.wf = take(sizeof(float) * kEntries);
    l.tile_stride = 32 * cpl + 4;
    l.tile = take(sizeof(float) * kCells * l.tile_stride);
    l.total = b;
    return l;
}

struct TileSm {
    float* cams;
    int* ctl;
    float* rc;
    unsigned* vmask;
    float2* uv;
    unsigned* box;
    int* cellg;
    Group* grp;
    unsigned long long* wq;
    float* wf;
    float* tile;
    int tile_stride;
};

__device__ __forceinline__ TileSm carve_tile(unsigned char* smem, int N, int cpl) {
    const TileLayout l = tile_layout(N, cpl);
    TileSm s;
    s.cams = reinterpret_cast<float*>(smem + l.cams);
    s.ctl = reinterpret_cast<int*>(smem + l.ctl);
    s.rc = reinterpret_cast<float*>(smem + l.rc);
    s.vmask = reinterpret_cast<unsigned*>(smem + l.vmask);
    s.uv = reinterpret_cast<float2*>(smem + l.uv);
    s.box = reinterpret_cast<unsigned*>(smem + l.box);
    s.cellg = reinterpret_cast<int*>(smem + l.cellg);
    s.grp = reinterpret_cast<Group*>(smem + l.grp);
    s.wq = reinterpret_cast<unsigned long long*>(smem + l.wq);
    s.wf = reinterpret_cast<float*>(smem + l.wf);
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

// Validity of one voxel in one camera, decided exactly as the fixed fp32
// order of project_point decides it.  Depth and the homogeneous image
// coordinates are computed in that order; the divides are taken with an
// approximate quotient first and settled by the IEEE divide only when the
// approximate position lies within 1e-5 (relative, at least 1e-5 px) of an
// image edge, far outside the error of the approximation.
__device__ __forceinline__ bool voxel_visible(const float* cam, float x, float y, float z, const GeoParams& g) {
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
        const bool out_u = ua < -mu || ua > g.img_w + mu, out_v = va < -mv || va > g.img_h + mv;
        if (out_u || out_v) return false;
        if (ua > mu && ua < g.img_w - mu && va > mv && va < g.img_h - mv) return true;
    }
    const float u = __fdiv_rn(uh, depth), v = __fdiv_rn(vh, depth);
    return u >= 0.0f && u <= g.img_w && v >= 0.0f && v <= g.img_h;
}

// Count pass over the bins [z0, z0 + zc): 1 / cnt per item, a bit per
// active camera that sees the item, and the optional uint8 count output.
__device__ inline void count_pass(const SampleArgs& a, const TileSm& s, int b, int ti0, int tj0, int z0, int zc,
                                  bool write_count) {
    const GeoParams& g = a.g;
    const ItemMap im = item_map(zc);
    const int nA = s.ctl[kCtlNA];
    const int zz = threadIdx.x % im.LZ;
    for (int p = 0; p < im.passes; ++p) {
        const int cell = p * im.cpp + (int)threadIdx.x / im.LZ;
        if (cell >= kCells || zz >= zc) continue;
        const int i = ti0 + cell / kTileJ, j = tj0 + cell % kTileJ, z = z0 + zz;
        const bool in = i < g.X && j < g.Y;
        unsigned m = 0;
        int cnt = 0;
        if (in) {
            const float x = voxel_centre(g.xmin, i, g.dx), y = voxel_centre(g.ymin, j, g.dy);
            const float zf = voxel_centre(g.zmin, z, g.dz);
            for (int aa = 0; aa < nA; ++aa) {
                if (voxel_visible(s.cams + s.ctl[kCtlActive + aa] * kCamFloats, x, y, zf, g)) {
                    m |= 1u << aa;
                    ++cnt;
                }
            }
            if (write_count) a.count[(((size_t)b * g.X + i) * g.Y + j) * g.Z + z] = (uint8_t)cnt;
        }
        s.rc[cell * kZc + zz] = cnt > 0 ? __frcp_rn((float)cnt) : 0.0f;
        s.vmask[cell * kZc + zz] = m;
    }
}

// Image-plane positions of the voxels that active camera slot aa sees (x =
// NaN elsewhere), in the fixed order of project_point.
__device__ inline void project_pass(const SampleArgs& a, const TileSm& s, int ti0, int tj0, int z0, int zc, int aa) {
    const GeoParams& g = a.g;
    const ItemMap im = item_map(zc);
    const float* cam = s.cams + s.ctl[kCtlActive + aa] * kCamFloats;
    const int zz = threadIdx.x % im.LZ;
    for (int p = 0; p < im.passes; ++p) {
        const int cell = p * im.cpp + (int)threadIdx.x / im.LZ;
        if (cell >= kCells || zz >= zc) continue;
        const int item = cell * kZc + zz;
        float2 uv = make_float2(__int_as_float(0x7fc00000), 0.0f);
        if ((s.vmask[item] >> aa) & 1u) {
            const int i = ti0 + cell / kTileJ, j = tj0 + cell % kTileJ;
            float fx, fy;
            ProjDetail det;
            if (project_point(cam, voxel_centre(g.xmin, i, g.dx), voxel_centre(g.ymin, j, g.dy),
                              voxel_centre(g.zmin, z0 + zz, g.dz), g, fx, fy, det))
                uv = make_float2(det.u, det.v);
        }
        s.uv[item] = uv;
    }
}

// Sampling position of an image-plane position on a level of scale (sW, sH):
// the two roundings of project_point, fx = u * sW - 0.5.
__device__ __forceinline__ void level_position(float2 uv, float sW, float sH, float& fx, float& fy) {
    fx = __fadd_rn(__fmul_rn(uv.x, sW), -0.5f);
    fy = __fadd_rn(__fmul_rn(uv.y, sH), -0.5f);
}

// Texel box of each cell on one level: (ylo, xlo) and (yhi, xhi) exclusive,
// as 16-bit fields; an empty box is lo = 0xffffffff, hi = 0.
__device__ inline void box_pass(const TileSm& s, int zc, int Hf, int Wf, float sW, float sH) {
    const ItemMap im = item_map(zc);
    const int zz = threadIdx.x % im.LZ;
    for (int p = 0; p < im.passes; ++p) {
        const int cell = p * im.cpp + (int)threadIdx.x / im.LZ;
        unsigned lo = 0xffffffffu, hi = 0u;
        if (cell < kCells && zz < zc) {
            const float2 uv = s.uv[cell * kZc + zz];
            if (!isnan(uv.x)) {
                float fx, fy;
                level_position(uv, sW, sH, fx, fy);
                const int x0 = (int)floorf(fx), y0 = (int)floorf(fy);
                lo = ((unsigned)max(y0, 0) << 16) | (unsigned)max(x0, 0);
                hi = ((unsigned)min(y0 + 2, Hf) << 16) | (unsigned)min(x0 + 2, Wf);
            }
        }
        for (int o = 1; o < im.LZ; o <<= 1) {
            lo = __vminu2(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            hi = __vmaxu2(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        if (zz == 0 && cell < kCells) {
            s.box[2 * cell] = lo;
            s.box[2 * cell + 1] = hi;
        }
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

__device__ __forceinline__ int slots_for(int n) { return n == 1 ? 1 : n == 2 ? 2 : n <= 4 ? 4 : 8; }

// Groups of the current view from the cells' boxes: cells whose boxes start
// at the same feature column form buckets, split into groups of at most
// kGmax cells; cells more than 63 columns right of the leftmost form groups
// of their own.  Then the union boxes, the weight layout and the merge
// rounds.  Warp 0 only.
__device__ inline void form_groups(const TileSm& s) {
    const int lane = threadIdx.x & 31;
    int* ctl = s.ctl;
    int* bcnt = ctl + kCtlBucket;
    int* gbase = ctl + kCtlGbase;
    int* gy0 = ctl + kCtlBounds;
    int* gx0 = gy0 + kCells;
    int* gy1 = gx0 + kCells;
    int* gx1 = gy1 + kCells;
    unsigned lo[2], hi[2];
    bool val[2];
    int xlo[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int c = lane + 32 * k;
        lo[k] = s.box[2 * c];
        hi[k] = s.box[2 * c + 1];
        val[k] = hi[k] != 0u;
        xlo[k] = (int)(lo[k] & 0xffffu);
    }
    const int xm = __reduce_min_sync(0xffffffffu, (unsigned)min(val[0] ? xlo[0] : 0xffff, val[1] ? xlo[1] : 0xffff));
    bcnt[lane] = 0;
    bcnt[lane + 32] = 0;
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
    int grp[2] = {-1, -1}, slot[2] = {0, 0};
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int c = lane + 32 * k;
        int cg = -1;
        if (val[k]) {
            int gi, n;
            if (key[k] < 64) {
                gi = gbase[key[k]] + rank[k] / kGmax;
                slot[k] = rank[k] % kGmax;
                n = min(kGmax, bcnt[key[k]] - (rank[k] / kGmax) * kGmax);
            } else {
                gi = nbg + (k == 0 ? __popc(far0 & lt) : __popc(far0) + __popc(far1 & lt));
                slot[k] = 0;
                n = 1;
            }
            grp[k] = gi;
            cg = (gi << 8) | slot[k];
            s.grp[gi].cell[slot[k]] = (unsigned char)c;
            if (slot[k] == 0) {
                s.grp[gi].n = n;
                gy0[gi] = (int)(lo[k] >> 16);
                gx0[gi] = (int)(lo[k] & 0xffffu);
                gy1[gi] = (int)(hi[k] >> 16);
                gx1[gi] = (int)(hi[k] & 0xffffu);
            }
        }
        s.cellg[c] = cg;
    }
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        if (grp[k] >= 0 && slot[k] != 0) {
            atomicMin(&gy0[grp[k]], (int)(lo[k] >> 16));
            atomicMin(&gx0[grp[k]], (int)(lo[k] & 0xffffu));
            atomicMax(&gy1[grp[k]], (int)(hi[k] >> 16));
            atomicMax(&gx1[grp[k]], (int)(hi[k] & 0xffffu));
        }
    }
    __syncwarp();
    // weight entries per group; boxes too large for half a round go direct
    int e[2], sl[2], h[2], w[2], dir[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int gi = lane + 32 * k;
        e[k] = 0;
        sl[k] = 1;
        h[k] = w[k] = 0;
        dir[k] = 0;
        if (gi < ng) {
            h[k] = gy1[gi] - gy0[gi];
            w[k] = gx1[gi] - gx0[gi];
            sl[k] = slots_for(s.grp[gi].n);
            // padded to 4 entries so that every group's weights start 16-byte aligned
            const long long ent = ((long long)h[k] * w[k] * sl[k] + 3) & ~3ll;
            if (ent > kEntries / 2) {
                dir[k] = 1;
            } else {
                e[k] = (int)ent;
            }
        }
    }
    const int emax = __reduce_max_sync(0xffffffffu, (unsigned)max(e[0], e[1]));
    const int step = kEntries - emax;  // >= kEntries / 2
    const int s0 = warp_inclusive_scan(e[0]), s1 = warp_inclusive_scan(e[1]);
    const int tot0 = __shfl_sync(0xffffffffu, s0, 31);
    const int off[2] = {s0 - e[0], tot0 + s1 - e[1]};
    int* rstart = ctl + kCtlRstart;
    int* nent = ctl + kCtlNent;
    nent[lane] = 0;
    nent[lane + 32] = 0;
    __syncwarp();
    int rnd[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int gi = lane + 32 * k;
        rnd[k] = off[k] / step;
        if (gi < ng) {
            Group& gp = s.grp[gi];
            gp.y0 = gy0[gi];
            gp.x0 = gx0[gi];
            gp.h = h[k];
            gp.w = w[k];
            gp.slots = sl[k];
            gp.round = rnd[k];
            gp.off = off[k] - rnd[k] * step;
            gp.direct = dir[k];
            atomicMax(&nent[rnd[k]], gp.off + e[k]);
        }
    }
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int gi = lane + 32 * k;
        if (gi < ng && (gi == 0 || s.grp[gi - 1].round != rnd[k])) rstart[rnd[k]] = gi;
    }
    if (lane == 0) {
        const int nr = ng > 0 ? s.grp[ng - 1].round + 1 : 0;
        rstart[nr] = ng;
        ctl[kCtlGroups] = ng;
        ctl[kCtlRounds] = nr;
    }
}

// ---------------------------------------------------------------------------
// Merge of one round's weights
// ---------------------------------------------------------------------------

constexpr float kFix = 1099511627776.0f;  // 2^40: fixed point of the merged weights
constexpr double kFixInv = 9.094947017729282379150390625e-13;  // 2^-40

// Sum w / cnt of every valid bin into its cell's slot of its group's
// [texel][slot] array (groups of round r that are not direct).
__device__ inline void merge_pass(const TileSm& s, int zc, int Hf, int Wf, float sW, float sH, int r) {
    const ItemMap im = item_map(zc);
    const int zz = threadIdx.x % im.LZ;
    for (int p = 0; p < im.passes; ++p) {
        const int cell = p * im.cpp + (int)threadIdx.x / im.LZ;
        if (cell >= kCells || zz >= zc) continue;
        const int item = cell * kZc + zz;
        const float2 uv = s.uv[item];
        const int cg = s.cellg[cell];
        if (isnan(uv.x) || cg < 0) continue;
        const Group& gp = s.grp[cg >> 8];
        if (gp.round != r || gp.direct) continue;
        float fx, fy;
        level_position(uv, sW, sH, fx, fy);
        const Corners c = bilinear_corners(fx, fy);
        const float rc = s.rc[item];
        const float ws[4] = {c.w00, c.w01, c.w10, c.w11};
        const int slot = cg & 255;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int yy = c.y0 + (k >> 1), xx = c.x0 + (k & 1);
            if ((unsigned)yy >= (unsigned)Hf || (unsigned)xx >= (unsigned)Wf) continue;
            const unsigned long long q = __float2ull_rn(__fmul_rn(ws[k], rc) * kFix);
            if (q == 0ull) continue;
            const int e = gp.off + ((yy - gp.y0) * gp.w + (xx - gp.x0)) * gp.slots + slot;
            atomicAdd(&s.wq[e], q);
        }
    }
}

// Round r's fixed-point sums to fp32 (one rounding each); the fixed-point
// words are cleared for the next round.
__device__ __forceinline__ void convert_pass(const TileSm& s, int r) {
    const int n = s.ctl[kCtlNent + r];
    for (int e = threadIdx.x; e < n; e += kThreads) {
        const unsigned long long q = s.wq[e];
        s.wq[e] = 0ull;
        s.wf[e] = __double2float_rn(__ull2double_rn(q) * kFixInv);
    }
}

// ---------------------------------------------------------------------------
// Per-lane channel vectors
// ---------------------------------------------------------------------------

// CPL channels of one texel for this lane, widened to fp32.  Raw words:
// fp32 CPL channels, or bf16 pairs (the bf16 bits are the high half of the
// fp32 word, so widening is exact).
template <bool BF16, int CPL>
struct LaneVec {
    static constexpr int kWords = BF16 ? CPL / 2 : CPL;
    unsigned w[kWords];

    __device__ __forceinline__ void load(const unsigned char* p) {
        if constexpr (kWords == 4) {
            const uint4 d = __ldg(reinterpret_cast<const uint4*>(p));
            w[0] = d.x; w[1] = d.y; w[2] = d.z; w[3] = d.w;
        } else if constexpr (kWords == 2) {
            const uint2 d = __ldg(reinterpret_cast<const uint2*>(p));
            w[0] = d.x; w[1] = d.y;
        } else {
            w[0] = __ldg(reinterpret_cast<const unsigned*>(p));
        }
    }
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int k = 0; k < kWords; ++k) w[k] = 0u;
    }
    __device__ __forceinline__ float get(int c) const {
        if constexpr (BF16)
            return (c & 1) ? __uint_as_float(w[c >> 1] & 0xffff0000u) : __uint_as_float(w[c >> 1] << 16);
        else
            return __uint_as_float(w[c]);
    }
};

// acc += wt * v over the lane's CPL channels (packed fp32x2 FMA of sm_100,
// each half an IEEE fma.rn).
template <int CPL>
__device__ __forceinline__ void fma_lane(float (&acc)[CPL], float wt, const float (&v)[CPL]) {
    if constexpr (CPL == 1) {
        acc[0] = __fmaf_rn(wt, v[0], acc[0]);
    } else {
#pragma unroll
        for (int p = 0; p < CPL / 2; ++p) {
            const float2 r = __ffma2_rn(make_float2(wt, wt), make_float2(v[2 * p], v[2 * p + 1]),
                                        make_float2(acc[2 * p], acc[2 * p + 1]));
            acc[2 * p] = r.x;
            acc[2 * p + 1] = r.y;
        }
    }
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
