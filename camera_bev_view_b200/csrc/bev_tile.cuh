// bev_tile.cuh -- per-CTA BEV tile machinery shared by the forward and backward
// kernels: shared-memory carve-up, camera staging and culling, and the
// per-z-chunk geometry pass.
//
// FlashBEV's reading notes ("Method" item 3) recompute the channel-independent
// geometry for every channel, and name that recompute as the cost that grows
// with C ("Limitation", second point; block-level geometry reuse is their
// suggested fix).  Here a CTA owns a kTileI x kTileJ tile of BEV cells and
// computes each (cell, camera, height bin) projection exactly once into shared
// memory; the channel loop then reads it.  Cameras that cannot see any voxel
// of the tile are dropped up front by a conservative box test.
#pragma once

#include "bev_kernels.cuh"

namespace bev {

struct TileSmem {
    float2* items;  // [kItemCap] (fx, fy) per (cell, active camera, bin); fx = NaN: invalid
    float* obuf;    // [kSliceMax][kObufStride] channel-major staging of the tile
    int* cnt;       // [kTile][zlen] valid cameras per (cell, bin)
    float* cams;    // [N][kCamFloats]
    int* act;       // [0..nA) active camera ids, act[32] = nA
};

__device__ __forceinline__ TileSmem carve_smem(unsigned char* smem, int N) {
    TileSmem s;
    s.items = reinterpret_cast<float2*>(smem);
    smem += sizeof(float2) * kItemCap;
    s.obuf = reinterpret_cast<float*>(smem);
    smem += sizeof(float) * kSliceMax * kObufStride;
    s.cnt = reinterpret_cast<int*>(smem);
    smem += sizeof(int) * kTile * kZChunkMax;
    s.cams = reinterpret_cast<float*>(smem);
    smem += sizeof(float) * ((N * kCamFloats + 3) & ~3);
    s.act = reinterpret_cast<int*>(smem);
    return s;
}

// Stage camera constants of batch item b and cull cameras against the tile.
__device__ inline void setup_tile(const SampleArgs& a, const TileSmem& s, int b, int ti0, int tj0) {
    const int tid = threadIdx.x;
    for (int t = tid; t < a.N * kCamFloats; t += kThreads) {
        const int n = t / kCamFloats, r = t - n * kCamFloats;
        s.cams[t] = r < 12 ? a.E[((size_t)b * a.N + n) * 16 + r]
                           : a.K[((size_t)b * a.N + n) * 9 + (r - 12)];
    }
    __syncthreads();
    if (tid < 32) {
        const GeoParams& g = a.g;
        bool vis = false;
        if (tid < a.N) {
            const int i1 = min(ti0 + kTileI, g.X) - 1, j1 = min(tj0 + kTileJ, g.Y) - 1;
            vis = box_may_be_visible(s.cams + tid * kCamFloats, voxel_centre(g.xmin, ti0, g.dx),
                                     voxel_centre(g.xmin, i1, g.dx), voxel_centre(g.ymin, tj0, g.dy),
                                     voxel_centre(g.ymin, j1, g.dy), voxel_centre(g.zmin, 0, g.dz),
                                     voxel_centre(g.zmin, g.Z - 1, g.dz), g.img_w, g.img_h);
        }
        const unsigned m = __ballot_sync(0xffffffffu, vis);
        if (vis) s.act[__popc(m & ((1u << tid) - 1u))] = tid;
        if (tid == 0) s.act[32] = __popc(m);
    }
    __syncthreads();
}

// Height bins per chunk so that kTile * nA * zc geometry slots fit.
__device__ __forceinline__ int z_chunk(int Z, int nA) {
    return min(Z, min(kZChunkMax, kItemCap / (kTile * nA)));
}

// Geometry of bins [z0, z0 + zlen) for every (cell, active camera): fills
// s.items (index ((cell * nA) + a) * zlen + zl) and s.cnt (cell * zlen + zl).
// Starts and ends with a CTA barrier.
__device__ inline void geometry_chunk(const SampleArgs& a, const TileSmem& s, int ti0, int tj0,
                                      int nA, int z0, int zlen) {
    const GeoParams& g = a.g;
    const int tid = threadIdx.x;
    __syncthreads();
    for (int t = tid; t < kTile * zlen; t += kThreads) s.cnt[t] = 0;
    __syncthreads();
    const int per_cell = nA * zlen;
    for (int it = tid; it < kTile * per_cell; it += kThreads) {
        const int cell = it / per_cell;
        const int r = it - cell * per_cell;
        const int aa = r / zlen;
        const int zl = r - aa * zlen;
        const int i = ti0 + cell / kTileJ, j = tj0 + cell % kTileJ;
        float2 res = make_float2(__int_as_float(0x7fc00000), 0.0f);
        if (i < g.X && j < g.Y) {
            const float x = voxel_centre(g.xmin, i, g.dx);
            const float y = voxel_centre(g.ymin, j, g.dy);
            const float z = voxel_centre(g.zmin, z0 + zl, g.dz);
            float fx, fy;
            if (project_voxel(s.cams + s.act[aa] * kCamFloats, x, y, z, g, fx, fy)) {
                res = make_float2(fx, fy);
                atomicAdd(&s.cnt[cell * zlen + zl], 1);
            }
        }
        s.items[it] = res;
    }
    __syncthreads();
}

// Valid-camera counts of the tile for bins [z0, z0 + zlen) (or zeros when the
// tile sees no camera: cnt == nullptr).
__device__ inline void store_counts(const SampleArgs& a, const int* cnt, int b, int ti0, int tj0,
                                    int z0, int zlen) {
    const GeoParams& g = a.g;
    for (int t = threadIdx.x; t < kTile * zlen; t += kThreads) {
        const int cell = t / zlen, zl = t - cell * zlen;
        const int i = ti0 + cell / kTileJ, j = tj0 + cell % kTileJ;
        if (i < g.X && j < g.Y)
            a.count[(((size_t)b * g.X + i) * g.Y + j) * g.Z + z0 + zl] =
                cnt ? (uint8_t)cnt[t] : (uint8_t)0;
    }
}

}  // namespace bev
