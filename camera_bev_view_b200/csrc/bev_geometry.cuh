// bev_geometry.cuh -- device-side voxel geometry for the dense Sampling-VT.
//
// Projection and validity follow the SparseDriveV2 notes, "Deformable
// Aggregation" step 2 ([u v 1]^T ~ K (R p + t); keep the camera only when the
// projection lands in [0, W] x [0, H]) with the depth test depth > 0.1 and the
// bilinear convention align_corners=False.  Every product and sum is rounded
// on its own (__fmul_rn / __fadd_rn never fuse into FMA) and the divide is the
// IEEE one, in the order the public header states, so validity counts and
// corner indices are reproducible bit for bit.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace bev {

// Per-camera constants staged in shared memory: E rows 0..2 then K rows 0..1.
constexpr int kCamFloats = 18;

struct GeoParams {
    float xmin, ymin, zmin;
    float dx, dy, dz;
    float img_w, img_h;   // image size as float (exact for sizes < 2^24)
    float sW, sH;         // (float)Wf / (float)img_w, (float)Hf / (float)img_h, host IEEE divide
    int X, Y, Z;
    int Hf, Wf;
};

__device__ __forceinline__ float voxel_centre(float lo, int i, float d) {
    return __fadd_rn(lo, __fmul_rn(__fadd_rn((float)i, 0.5f), d));
}

// Row r of the ego-to-camera transform: ((e0 x + e1 y) + e2 z) + e3.
__device__ __forceinline__ float cam_row(const float* e, float x, float y, float z) {
    float t = __fadd_rn(__fmul_rn(e[0], x), __fmul_rn(e[1], y));
    t = __fadd_rn(t, __fmul_rn(e[2], z));
    return __fadd_rn(t, e[3]);
}

// Image-plane quantities of one projection, for derivatives through it.
struct ProjDetail {
    float u, v, depth;
};

// Project one point (ego frame) through one camera.  On success writes the
// feature-map sampling position (fx, fy) and returns true; `det` receives
// u, v and the depth whenever the depth test passes.
__device__ __forceinline__ bool project_point(const float* cam, float x, float y, float z, const GeoParams& g,
                                              float& fx, float& fy, ProjDetail& det) {
    const float pcx = cam_row(cam + 0, x, y, z);
    const float pcy = cam_row(cam + 4, x, y, z);
    const float depth = cam_row(cam + 8, x, y, z);
    if (!(depth > 0.1f)) return false;
    const float* k = cam + 12;
    float uh = __fadd_rn(__fmul_rn(k[0], pcx), __fmul_rn(k[1], pcy));
    uh = __fadd_rn(uh, __fmul_rn(k[2], depth));
    float vh = __fadd_rn(__fmul_rn(k[3], pcx), __fmul_rn(k[4], pcy));
    vh = __fadd_rn(vh, __fmul_rn(k[5], depth));
    const float u = __fdiv_rn(uh, depth);
    const float v = __fdiv_rn(vh, depth);
    det.u = u;
    det.v = v;
    det.depth = depth;
    if (!(u >= 0.0f && u <= g.img_w && v >= 0.0f && v <= g.img_h)) return false;
    fx = __fadd_rn(__fmul_rn(u, g.sW), -0.5f);
    fy = __fadd_rn(__fmul_rn(v, g.sH), -0.5f);
    return true;
}

// Project one voxel centre through one camera (see project_point).
__device__ __forceinline__ bool project_voxel(const float* cam, float x, float y, float z,
                                              const GeoParams& g, float& fx, float& fy) {
    ProjDetail det;
    return project_point(cam, x, y, z, g, fx, fy, det);
}

// Bilinear corners of (fx, fy): top-left texel and the four weights
// w00 (y0,x0), w01 (y0,x0+1), w10 (y0+1,x0), w11 (y0+1,x0+1).
struct Corners {
    int x0, y0;
    float w00, w01, w10, w11;
};

__device__ __forceinline__ Corners bilinear_corners(float fx, float fy) {
    const float x0f = floorf(fx), y0f = floorf(fy);
    const float wx1 = __fsub_rn(fx, x0f), wy1 = __fsub_rn(fy, y0f);
    const float wx0 = __fsub_rn(1.0f, wx1), wy0 = __fsub_rn(1.0f, wy1);
    Corners c;
    c.x0 = (int)x0f;
    c.y0 = (int)y0f;
    c.w00 = __fmul_rn(wy0, wx0);
    c.w01 = __fmul_rn(wy0, wx1);
    c.w10 = __fmul_rn(wy1, wx0);
    c.w11 = __fmul_rn(wy1, wx1);
    return c;
}

// Conservative visibility of an axis-aligned box of voxel centres from one
// camera, evaluated one box corner at a time.  For a corner p this writes
// each of the five validity conditions (depth > 0.1, uh >= 0,
// W pc_z - uh >= 0, vh >= 0, H pc_z - vh >= 0) plus a margin of 1e-3 of the
// terms' magnitude (four orders above the fp32 evaluation error of both this
// test and the projection it stands for).  Each such quantity is convex in p,
// so its maximum over the box is at a corner: a camera can be skipped for the
// box when one of the five maxima is negative.
__device__ inline void corner_margins(const float* cam, float px, float py, float pz, float img_w,
                                      float img_h, float m[5]) {
    const float W = img_w, H = img_h;
    float pc[3], mag[3];
    for (int r = 0; r < 3; ++r) {
        const float* e = cam + 4 * r;
        pc[r] = e[0] * px + e[1] * py + e[2] * pz + e[3];
        mag[r] = fabsf(e[0] * px) + fabsf(e[1] * py) + fabsf(e[2] * pz) + fabsf(e[3]);
    }
    const float k0 = cam[12], k1 = cam[13], k2 = cam[14], k3 = cam[15], k4 = cam[16], k5 = cam[17];
    const float uh = k0 * pc[0] + k1 * pc[1] + k2 * pc[2];
    const float vh = k3 * pc[0] + k4 * pc[1] + k5 * pc[2];
    const float umag = fabsf(k0) * mag[0] + fabsf(k1) * mag[1] + fabsf(k2) * mag[2];
    const float vmag = fabsf(k3) * mag[0] + fabsf(k4) * mag[1] + fabsf(k5) * mag[2];
    const float t = 1e-3f, a = 1e-4f;
    m[0] = pc[2] - 0.1f + t * mag[2] + a;
    m[1] = uh + t * umag + a;
    m[2] = W * pc[2] - uh + t * (umag + W * mag[2]) + a;
    m[3] = vh + t * vmag + a;
    m[4] = H * pc[2] - vh + t * (vmag + H * mag[2]) + a;
}

}  // namespace bev
