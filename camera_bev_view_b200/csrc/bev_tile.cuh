// bev_tile.cuh -- per-CTA BEV tile machinery shared by the forward and backward
// kernels.
//
// FlashBEV's reading notes ("Method" item 3) recompute the channel-independent
// geometry for every channel and name that recompute as the cost that grows
// with C ("Limitation", second point; their "Takeaway" 4 proposes block-level
// geometry reuse).  Here a CTA owns a kTileI x kTileJ tile of BEV cells and:
//   1. stages the calibrations and culls cameras that cannot see any voxel of
//      the tile (conservative box test, one thread per (camera, box corner));
//   2. per chunk of height bins, projects every (cell, active camera, bin)
//      voxel once: (fx, fy) into shared memory and the per-(cell, bin) valid
//      count;
//   3. per (cell, camera) lays a patch over the bounding box of the texels its
//      valid voxels touch, and merges into it the bilinear weights w / cnt of
//      all bins.  One thread owns a (cell, camera) patch and adds in height-bin
//      order, so the merged weights are fp32 sums in a fixed order: results do
//      not depend on thread timing.
// The channel loops of the forward and backward then visit each touched
// texel of a (cell, camera) once, whatever the number of bins that hit it.
#pragma once

#include <limits.h>

#include "bev_kernels.cuh"

namespace bev {

struct TileSmem {
    float2* items;  // [kItemCap] (fx, fy) per (camera aa, bin zl, cell); fx = NaN: invalid
    float* patch;   // [kPatchCap] merged weights
    float* obuf;    // [kGroupCh][kObufStride] channel-major staging tile, aliases items + patch
    int* cnt;       // [zl][cell / 4] valid cameras per (cell, bin), one byte each
    int4* pinfo;    // [aa][cell] patch (y0, x0, h << 16 | w, offset)
    int4* win;      // [aa] union of the camera's texel boxes over the tile (ymin, ymax, xmin, xmax)
    float* cams;    // [N][kCamFloats]
    int* act;       // [0..nA) active camera ids; act[32] = nA
    int* scan;      // [64] block-scan scratch
};

// Valid-camera count of (cell, bin zl) from the packed table.
__device__ __forceinline__ int cell_count(const int* cnt, int zl, int cell) {
    return (cnt[zl * (kTile / 4) + (cell >> 2)] >> (8 * (cell & 3))) & 0xff;
}

__device__ __forceinline__ TileSmem carve_smem(unsigned char* smem, int N) {
    const SmemLayout l = smem_layout(N);
    TileSmem s;
    s.items = reinterpret_cast<float2*>(smem + l.items);
    s.obuf = reinterpret_cast<float*>(smem + l.items);
    s.patch = reinterpret_cast<float*>(smem + l.patch);
    s.cnt = reinterpret_cast<int*>(smem + l.cnt);
    s.pinfo = reinterpret_cast<int4*>(smem + l.pinfo);
    s.win = reinterpret_cast<int4*>(smem + l.win);
    s.cams = reinterpret_cast<float*>(smem + l.cams);
    s.act = reinterpret_cast<int*>(smem + l.act);
    s.scan = reinterpret_cast<int*>(smem + l.scan);
    return s;
}

// Tile of this CTA.  Tiles are issued in rings of increasing Chebyshev
// distance from the centre tile of the grid: for rigs mounted near the grid
// centre the nearest voxels see the most texels, so the heaviest tiles start
// first and the light outer ring fills the tail of the launch.  Any order
// gives the same results.  Warp 0 maps the block index (the rank) to its
// ring, then finds the position inside the ring with ballots over 32 ring
// positions at a time; the result is shared through `slot`.
__device__ inline void tile_origin(const SampleArgs& a, int* slot, int& ti0, int& tj0) {
    const int Ti = a.tiles_i, Tj = a.tiles_j;
    if (threadIdx.x < 32) {
        const int ci = (Ti - 1) >> 1, cj = (Tj - 1) >> 1;
        auto area = [&](int r) -> int {  // tiles within Chebyshev distance r of the centre
            if (r < 0) return 0;
            const int h = min(ci + r, Ti - 1) - max(ci - r, 0) + 1;
            const int w = min(cj + r, Tj - 1) - max(cj - r, 0) + 1;
            return h * w;
        };
        int k = blockIdx.x, r = 0;
        while (k >= area(r) - area(r - 1)) {
            k -= area(r) - area(r - 1);
            ++r;
        }
        // positions of ring r: p = 0 .. 8r - 1 (or just the centre for r = 0)
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
    }
    __syncthreads();
    ti0 = slot[0];
    tj0 = slot[1];
}

// Stage camera constants of batch item b and cull cameras against the tile.
// One thread per (camera, corner of the tile's voxel-centre box); the five
// visibility margins are max-reduced over the eight corners with shuffles.
__device__ inline void setup_tile(const SampleArgs& a, const TileSmem& s, int b, int ti0, int tj0) {
    const int tid = threadIdx.x;
    for (int t = tid; t < a.N * kCamFloats; t += kThreads) {
        const int n = t / kCamFloats, r = t - n * kCamFloats;
        s.cams[t] = r < 12 ? a.E[((size_t)b * a.N + n) * 16 + r]
                           : a.K[((size_t)b * a.N + n) * 9 + (r - 12)];
    }
    __syncthreads();
    const GeoParams& g = a.g;
    const int n = tid >> 3, v = tid & 7;  // kThreads == 8 * BEV_MAX_CAMERAS
    double m[5] = {-1e300, -1e300, -1e300, -1e300, -1e300};
    if (n < a.N) {
        const int i1 = min(ti0 + kTileI, g.X) - 1, j1 = min(tj0 + kTileJ, g.Y) - 1;
        const float px = voxel_centre(g.xmin, (v & 1) ? i1 : ti0, g.dx);
        const float py = voxel_centre(g.ymin, (v & 2) ? j1 : tj0, g.dy);
        const float pz = voxel_centre(g.zmin, (v & 4) ? g.Z - 1 : 0, g.dz);
        corner_margins(s.cams + n * kCamFloats, px, py, pz, g.img_w, g.img_h, m);
    }
#pragma unroll
    for (int q = 0; q < 5; ++q) {
        m[q] = fmax(m[q], __shfl_xor_sync(0xffffffffu, m[q], 1));
        m[q] = fmax(m[q], __shfl_xor_sync(0xffffffffu, m[q], 2));
        m[q] = fmax(m[q], __shfl_xor_sync(0xffffffffu, m[q], 4));
    }
    if (v == 0) s.scan[n] = (n < a.N) && m[0] >= 0.0 && m[1] >= 0.0 && m[2] >= 0.0 &&
                             m[3] >= 0.0 && m[4] >= 0.0;
    __syncthreads();
    if (tid < 32) {
        const bool vis = s.scan[tid] != 0;
        const unsigned mask = __ballot_sync(0xffffffffu, vis);
        if (vis) s.act[__popc(mask & ((1u << tid) - 1u))] = tid;
        if (tid == 0) s.act[32] = __popc(mask);
    }
    __syncthreads();
}

// Height bins per chunk so that kTile * nA * zc geometry slots fit.
__device__ __forceinline__ int z_chunk(int Z, int nA) {
    return max(1, min(Z, min(kZChunkMax, kItemCap / (kTile * nA))));
}

// Index of the (fx, fy) slot of (cell, active camera aa, bin zl): cells are
// fastest, so a warp touches 32 consecutive slots (no bank conflicts).
__device__ __forceinline__ int item_index(int cell, int aa, int zl, int zlen) {
    return (aa * zlen + zl) * kTile + cell;
}

// (aa, zl) of slice index sl = aa * zlen + zl (exact for the small integers involved).
__device__ __forceinline__ void split_slice(int sl, int zlen, float inv_zlen, int& aa, int& zl) {
    aa = __float2int_rz(((float)sl + 0.5f) * inv_zlen);
    zl = sl - aa * zlen;
}

// Geometry of bins [z0, z0 + zlen) for every (cell, active camera): fills
// s.items (item_index) and the packed s.cnt.  Ends with a CTA barrier.
__device__ inline void geometry_chunk(const SampleArgs& a, const TileSmem& s, int ti0, int tj0,
                                      int nA, int z0, int zlen) {
    const GeoParams& g = a.g;
    const int tid = threadIdx.x;
    __syncthreads();  // previous users of items / cnt are done
    for (int t = tid; t < (kTile / 4) * zlen; t += kThreads) s.cnt[t] = 0;
    __syncthreads();
    const float inv_zlen = 1.0f / (float)zlen;
    const int cell = tid & (kTile - 1);
    const int i = ti0 + cell / kTileJ, j = tj0 + cell % kTileJ;
    const bool in_grid = i < g.X && j < g.Y;
    const float x = voxel_centre(g.xmin, i, g.dx);
    const float y = voxel_centre(g.ymin, j, g.dy);
    for (int it = tid; it < kTile * nA * zlen; it += kThreads) {
        int aa, zl;
        split_slice(it / kTile, zlen, inv_zlen, aa, zl);
        float2 res = make_float2(__int_as_float(0x7fc00000), 0.0f);
        if (in_grid) {
            const float z = voxel_centre(g.zmin, z0 + zl, g.dz);
            float fx, fy;
            if (project_voxel(s.cams + s.act[aa] * kCamFloats, x, y, z, g, fx, fy)) {
                res = make_float2(fx, fy);
                atomicAdd(&s.cnt[zl * (kTile / 4) + (cell >> 2)], 1 << (8 * (cell & 3)));
            }
        }
        s.items[it] = res;
    }
    __syncthreads();
}

// Exclusive block-wide scan of one int per thread; returns the prefix and
// writes the total to *total (all threads).
__device__ inline int block_exclusive_scan(int v, int* scratch, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kWarps ? scratch[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < kWarps) scratch[32 + lane] = w;
    }
    __syncthreads();
    const int before = (warp > 0 ? scratch[32 + warp - 1] : 0) + x - v;
    *total = scratch[32 + kWarps - 1];
    __syncthreads();
    return before;
}

// Texel box (ymin, ymax, xmin, xmax) of one (cell, camera): the in-range
// bilinear corners of its valid voxels; ymax < ymin when there are none.
__device__ __forceinline__ int4 texel_box(const TileSmem& s, int cell, int aa, int zlen, int Hf, int Wf) {
    int ylo = INT_MAX, yhi = -1, xlo = INT_MAX, xhi = -1;
    for (int zl = 0; zl < zlen; ++zl) {
        const float2 f = s.items[item_index(cell, aa, zl, zlen)];
        if (!(f.x == f.x)) continue;
        const int x0 = (int)floorf(f.x), y0 = (int)floorf(f.y);
        ylo = min(ylo, max(y0, 0));
        yhi = max(yhi, min(y0 + 1, Hf - 1));
        xlo = min(xlo, max(x0, 0));
        xhi = max(xhi, min(x0 + 1, Wf - 1));
    }
    return make_int4(ylo, yhi, xlo, xhi);
}

// Lay out the patches of cameras [a0, a1) over their texel boxes.  Returns the
// number of patch entries, or -1 (uniformly) if they would not fit in
// kPatchCap.  On success s.pinfo[aa][cell] holds (y0, x0, h << 16 | w, offset)
// and s.win[aa] the union of camera aa's boxes.  Ends with a CTA barrier.
__device__ inline int layout_patches(const SampleArgs& a, const TileSmem& s, int zlen, int a0, int a1) {
    const int pairs = kTile * (a1 - a0);  // <= kTile * BEV_MAX_CAMERAS = 8 * kThreads
    int4 box[8];
    int sizes = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int p = threadIdx.x + k * kThreads;  // cells fastest
        box[k] = make_int4(0, -1, 0, -1);
        if (p < pairs) {
            box[k] = texel_box(s, p & (kTile - 1), a0 + p / kTile, zlen, a.g.Hf, a.g.Wf);
            if (box[k].y >= box[k].x) sizes += (box[k].y - box[k].x + 1) * (box[k].w - box[k].z + 1);
        }
    }
    if (threadIdx.x < a1 - a0) s.win[a0 + threadIdx.x] = make_int4(INT_MAX, -1, INT_MAX, -1);
    int total;
    int off = block_exclusive_scan(sizes, s.scan, &total);  // its barriers order the reset above
    if (total > kPatchCap) return -1;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int p = threadIdx.x + k * kThreads;
        if (p < pairs) {
            const int4 bx = box[k];
            int4 slot = make_int4(0, 0, 0, 0);
            if (bx.y >= bx.x) {
                const int h = bx.y - bx.x + 1, w = bx.w - bx.z + 1;
                slot = make_int4(bx.x, bx.z, (h << 16) | w, off);
                off += h * w;
                int* wn = reinterpret_cast<int*>(&s.win[a0 + p / kTile]);
                atomicMin(wn + 0, bx.x);
                atomicMax(wn + 1, bx.y);
                atomicMin(wn + 2, bx.z);
                atomicMax(wn + 3, bx.w);
            }
            s.pinfo[(a0 + p / kTile) * kTile + (p & (kTile - 1))] = slot;
        }
    }
    __syncthreads();
    return total;
}

// Ask L1 for the texel windows of cameras [a0, a1): every 128-byte line of
// their channel vectors (channels-last rows [xmin, xmax] of rows [ymin, ymax],
// chunks [chunk0, chunk0 + nchunks)).  Issued before the patches are filled,
// so the lines are on chip when the channel loop reaches them.
__device__ inline void prefetch_windows(const TileSmem& s, const uint4* feat_b, size_t cam_stride, int Wf,
                                        int Qtot, int chunk0, int nchunks, int a0, int a1) {
    for (int aa = a0; aa < a1; ++aa) {
        const int4 wn = s.win[aa];
        if (wn.y < wn.x) continue;
        const uint4* Fn = feat_b + (size_t)s.act[aa] * cam_stride;
        const int ww = wn.w - wn.z + 1;
        // bytes of one window row, from the first texel's first chunk to the last texel's last chunk
        const int span = ((ww - 1) * Qtot + nchunks) * 16;
        const int lines = (span + 127) / 128 + 1;
        const int rows = wn.y - wn.x + 1;
        for (int t = threadIdx.x; t < rows * lines; t += kThreads) {
            const int r = t / lines, l = t - r * lines;
            const char* row = reinterpret_cast<const char*>(Fn + ((size_t)(wn.x + r) * Wf + wn.z) * Qtot + chunk0);
            const char* p = row + 128 * l;
            if (p < row + span) asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
        }
    }
}

// Merge w / cnt of the valid voxels of cameras [a0, a1) into their patches.
// One thread per (cell, camera): it clears its own patch, then adds the four
// corner weights of each valid bin in increasing bin order (fp32 sums in a
// fixed order; patches of different pairs are disjoint).  Ends with a CTA
// barrier.
__device__ inline void fill_patches(const SampleArgs& a, const TileSmem& s, int zlen, int a0, int a1) {
    const GeoParams& g = a.g;
    const int pairs = kTile * (a1 - a0);
    for (int p = threadIdx.x; p < pairs; p += kThreads) {
        const int cell = p & (kTile - 1), aa = a0 + p / kTile;
        const int4 pi = s.pinfo[aa * kTile + cell];
        const int w = pi.z & 0xffff;
        float* pw = s.patch + pi.w;
        for (int e = 0; e < (pi.z >> 16) * w; ++e) pw[e] = 0.0f;
        for (int zl = 0; zl < zlen; ++zl) {
            const float2 f = s.items[item_index(cell, aa, zl, zlen)];
            if (!(f.x == f.x)) continue;
            const float rc = __frcp_rn((float)cell_count(s.cnt, zl, cell));
            const Corners c = bilinear_corners(f.x, f.y);
            const float ws[4] = {c.w00, c.w01, c.w10, c.w11};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int yy = c.y0 + (k >> 1), xx = c.x0 + (k & 1);
                if ((unsigned)yy >= (unsigned)g.Hf || (unsigned)xx >= (unsigned)g.Wf) continue;
                pw[(yy - pi.x) * w + (xx - pi.y)] += ws[k] * rc;
            }
        }
    }
    __syncthreads();
}

// Valid-camera counts of the tile for bins [z0, z0 + zlen) (zeros when cnt is null).
__device__ inline void store_counts(const SampleArgs& a, const int* cnt, int b, int ti0, int tj0,
                                    int z0, int zlen) {
    const GeoParams& g = a.g;
    for (int t = threadIdx.x; t < kTile * zlen; t += kThreads) {
        const int cell = t / zlen, zl = t - cell * zlen;
        const int i = ti0 + cell / kTileJ, j = tj0 + cell % kTileJ;
        if (i < g.X && j < g.Y)
            a.count[(((size_t)b * g.X + i) * g.Y + j) * g.Z + z0 + zl] =
                cnt ? (uint8_t)cell_count(cnt, zl, cell) : (uint8_t)0;
    }
}

}  // namespace bev
