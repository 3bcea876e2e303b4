/*
 * bevsample.h -- C ABI of the B200-native exact dense Sampling-VT library
 * (libbevsample.so, sm_100a).
 *
 * The operation (FlashBEV reading notes, arxiv cs.RO 2607.10071, "Core Idea"
 * and "Method" items 1-4): for every BEV output element (b, c, i, j) visit
 * each height bin k and camera n, project the voxel centre through the
 * camera's ego-to-camera extrinsic and intrinsic (SparseDriveV2 notes,
 * "Deformable Aggregation" step 2: [u v 1]^T ~ K (R p + t)), keep the camera
 * when depth > 0.1 and (u, v) lies in [0, W_img] x [0, H_img], sample the
 * feature map bilinearly (align_corners=False, zero padding), average over the
 * valid cameras of the bin and sum the bin means over height ("Key Insight":
 * a height sum).  No voxel grid, projected-coordinate tensor, mask or
 * Features3D volume is written to memory; the notes' "Method" item 4 holds:
 * results equal the materialised form up to floating-point order.
 *
 * Conventions shared by every entry point
 *  - Pointers are DEVICE pointers on the current CUDA device unless marked
 *    "host".  All tensors are dense, row-major, without padding.
 *  - The caller owns every buffer.  The library allocates nothing, keeps no
 *    global state between calls and may be called from several host threads.
 *  - Work is enqueued asynchronously on `stream` (0 = legacy default stream).
 *    No call synchronises the device or copies between host and device.
 *  - Errors are returned as status codes, never thrown; no call aborts.  An
 *    argument error is detected before anything is enqueued.
 *  - Ego frame: x forward, y left, z up.  out[b, c, i, j]: row i indexes ego x,
 *    column j indexes ego y (the LSS tutorial's "Splat" step: x to row, y to
 *    column).  Camera frame: x right, y down, z forward (depth = camera z).
 *  - Geometry is evaluated in fp32 in one fixed order, each product and sum
 *    rounded separately, with an IEEE divide:
 *      centre   x_i = xmin + ((float)i + 0.5f) * dx   (same for y_j, z_k)
 *      camera   pc_r = ((E_r0 x + E_r1 y) + E_r2 z) + E_r3
 *      image    u = ((K_00 pc_x + K_01 pc_y) + K_02 pc_z) / pc_z, v likewise
 *      feature  fx = u * ((float)Wf / (float)W_img) - 0.5f, fy likewise
 *      weights  x0 = floor(fx), wx1 = fx - x0, wx0 = 1 - wx1; w = wy * wx
 *    so validity counts are reproducible bit for bit by any IEEE evaluation
 *    of the same expression.  Accumulation is fp32.
 *  - Preconditions not checked on the device: K's last row is [0 0 1]; E's
 *    bottom row is ignored; calibrations are finite.
 */
#ifndef BEVSAMPLE_H
#define BEVSAMPLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* CUDA stream handle (identical to cudaStream_t / CUstream). */
typedef struct CUstream_st* bev_stream_t;

/* Feature storage type. */
enum { BEV_F32 = 0, BEV_BF16 = 1 };
/* Feature layout: [B,N,C,Hf,Wf] (per-camera NCHW) or [B,N,Hf,Wf,C] (channels last). */
enum { BEV_NCHW = 0, BEV_NHWC = 1 };

/* Status codes. */
enum {
    BEV_OK = 0,
    BEV_ERR_INVALID_ARG = -1, /* NULL pointer, bad size, bad grid, host pointer where a device one is due */
    BEV_ERR_UNSUPPORTED = -2, /* valid request outside what this build implements */
    BEV_ERR_WORKSPACE = -3,   /* workspace NULL, too small or misaligned */
    BEV_ERR_CUDA = -4,        /* a CUDA runtime call or launch failed */
    BEV_ERR_INTERNAL = -5     /* a device-side consistency check failed */
};

/* Limits of this build. */
#define BEV_MAX_CAMERAS 32  /* N; counts are stored as uint8 */
#define BEV_MAX_DIM 16384   /* X, Y, Hf, Wf, img sizes */
#define BEV_MAX_Z 1024

/* BEV voxel grid.  X, Y, Z counts; ranges in metres; dx, dy, dz = extent /
 * count in fp32.  Voxel centres: xmin + ((float)i + 0.5f) * dx. */
typedef struct bev_grid_t {
    int X, Y, Z;
    float xmin, xmax, ymin, ymax, zmin, zmax;
    float dx, dy, dz;
} bev_grid_t;

/* Build a grid from ranges and cell sizes (LSS tutorial, "Splat": the range
 * divided by the cell size gives the count, e.g. [-50, 50] m at 0.5 m -> 200).
 *   range  host float[6]: xmin, xmax, ymin, ymax, zmin, zmax (max > min, finite)
 *   res    host float[3]: dx, dy, dz (> 0)
 *   out    host, written on success
 * Each extent / res must lie within 1e-4 of an integer in [1, BEV_MAX_DIM]
 * (Z: [1, BEV_MAX_Z]); the stored cell size is recomputed as extent / count
 * in fp32.  Returns BEV_OK or BEV_ERR_INVALID_ARG.  Host only. */
int bev_grid_spec(const float range[6], const float res[3], bev_grid_t* out);

/* Bytes of device workspace bev_sample_forward (for_backward = 0) or
 * bev_sample_backward (for_backward = 1) needs for these sizes; 0 when none is
 * needed.  dtype/layout are ignored for the backward.  Returns (size_t)-1 for
 * invalid sizes. */
size_t bev_workspace_size(int dtype, int layout, int B, int N, int C, int Hf, int Wf,
                          int for_backward);

/* Forward: out[b, c, i, j] = sum_k [cnt > 0] (1 / cnt) sum_{valid n} bilinear(F[b, n, c], u, v)
 * (FlashBEV reading notes, "Method" items 1-2).
 *   features     [B,N,C,Hf,Wf] (BEV_NCHW) or [B,N,Hf,Wf,C] (BEV_NHWC); dtype BEV_F32 or BEV_BF16
 *   intrinsics   [B,N,3,3] fp32, pixel units of a W_img x H_img image
 *   ego2cam      [B,N,4,4] fp32, maps ego coordinates into the camera frame
 *   img_h/img_w  image size the intrinsics refer to (>= 1)
 *   grid         host pointer, from bev_grid_spec (or filled consistently)
 *   out          [B,C,X,Y] fp32, fully overwritten
 *   valid_count  [B,X,Y,Z] uint8 number of valid cameras per voxel, or NULL
 *   workspace    device scratch of at least bev_workspace_size(dtype, layout, ..., 0)
 *                bytes, 256-byte aligned (may be NULL when that size is 0).  The
 *                library reuses it inside the call only; do not share one
 *                workspace between calls that may overlap on the device.
 * 1 <= N <= BEV_MAX_CAMERAS; B, C >= 1.
 * Returns BEV_OK, BEV_ERR_INVALID_ARG, BEV_ERR_UNSUPPORTED, BEV_ERR_WORKSPACE
 * or BEV_ERR_CUDA.  Outputs are undefined after an error. */
int bev_sample_forward(const void* features, int dtype, int layout,
                       int B, int N, int C, int Hf, int Wf,
                       const float* intrinsics, const float* ego2cam,
                       int img_h, int img_w, const bev_grid_t* grid,
                       float* out, uint8_t* valid_count,
                       void* workspace, size_t workspace_bytes, bev_stream_t stream);

/* Backward with respect to the features only (the operator is linear in them):
 *   dF[b, n, c, y, x] = sum over valid (i, j, k, n) samples touching texel (y, x)
 *                       of w * dout[b, c, i, j] / cnt_k
 * (FlashBEV reading notes, "Method" item 4: forward and backward differ from the
 * materialised form only by floating-point order).  No gradient flows to K, E
 * or the grid.
 *   dout        [B,C,X,Y] fp32
 *   dfeatures   [B,N,C,Hf,Wf] fp32, fully overwritten
 *   workspace   at least bev_workspace_size(.., 1) bytes, 256-byte aligned
 * Other arguments as for bev_sample_forward.  Accumulation order across cells
 * is not fixed (atomics), so repeated calls may differ in the last bits. */
int bev_sample_backward(const float* dout, int B, int N, int C, int Hf, int Wf,
                        const float* intrinsics, const float* ego2cam,
                        int img_h, int img_w, const bev_grid_t* grid,
                        float* dfeatures, void* workspace, size_t workspace_bytes,
                        bev_stream_t stream);

/* 1 when this library was built with device-side bounds checks
 * (-DBEV_BOUNDS_CHECK, libbevsample_checked.so), else 0.  In that build the
 * dense forward and backward kernels test every geometry-derived address --
 * each group's texel box, merge word, group-table slot, output, count and dout
 * index -- before using it; a failed test skips the access and sets a device
 * error word, which the call reads back after draining `stream` (the call is
 * then synchronous) and reports as BEV_ERR_INTERNAL.  Host only. */
int bev_bounds_checked(void);

/* Size of the built-in scratch array used by bev_sample_backward_noalloc. */
#define BEV_NOALLOC_SCRATCH_BYTES (16u << 20)

/* The feature gradient of bev_sample_backward for callers that cannot
 * allocate device memory or hand the library a workspace -- for example a
 * plugin inside an engine that pre-plans every device buffer and gives its
 * plugins no allocator, a deployment that forbids device allocation after
 * start-up, or a real-time loop in which cudaMalloc / cudaFree would stall the
 * device.  (The pages have no counterpart: this is a packaging variant of the
 * backward above, with the same arguments minus the workspace and the same
 * results.)
 *
 * The accumulation buffer lives in a fixed array of BEV_NOALLOC_SCRATCH_BYTES
 * (16 MiB) in the library's own device memory, which every GPU that loads the
 * library keeps until the process exits.  Shapes whose buffer,
 * B * N * Hf * Wf * round_up(C, 4) * 4 bytes, exceeds it are rejected with
 * BEV_ERR_UNSUPPORTED before anything is enqueued.
 *
 * The first call in each CUDA context looks up that context's address of the
 * array (cudaGetSymbolAddress, with the context current) and caches it by
 * device and context id, so make the first call on a device (and again after
 * a cudaDeviceReset) before capturing any stream.  All calls share the one
 * array and leave their contents in it; each call clears what it uses before
 * accumulating.  Calls whose work may overlap on the GPU (other streams, other
 * host threads) race on the array: serialise them.  Nothing is allocated and
 * no cudaMalloc / cudaFree is made.  Other arguments, results and errors as for
 * bev_sample_backward. */
int bev_sample_backward_noalloc(const float* dout, int B, int N, int C, int Hf, int Wf,
                                const float* intrinsics, const float* ego2cam,
                                int img_h, int img_w, const bev_grid_t* grid,
                                float* dfeatures, bev_stream_t stream);

/* Channels-last copy of the features: out[b, n, y, x, c] = features[b, n, c, y, x].
 * The forward performs this step itself for BEV_NCHW input; calling it
 * separately lets a caller keep one channels-last copy for several forward
 * calls, and pass it with layout BEV_NHWC (used in place when C is a multiple
 * of 4 for fp32 or 8 for bf16).  A bandwidth-bound tiled transpose.
 *   features  [B,N,C,Hf,Wf], dtype BEV_F32 or BEV_BF16
 *   out       [B,N,Hf,Wf,C], same dtype, must not overlap features
 * Returns BEV_OK, BEV_ERR_INVALID_ARG, BEV_ERR_UNSUPPORTED or BEV_ERR_CUDA. */
int bev_features_to_channels_last(const void* features, int dtype, int B, int N, int C, int Hf, int Wf,
                                  void* out, bev_stream_t stream);

/* ---------------------------------------------------------------------------
 * Multi-scale dense Sampling-VT (FlashBEV reading notes, "Takeaway" 4:
 * multi-scale fused view transformation; SparseDriveV2 notes, "Image
 * Encoder": FPN levels P_l with one channel count).  Each voxel is projected
 * once per camera, with the validity test and count of bev_sample_forward;
 * level l samples its own map at its own scale, fx_l = u * (W_l / W_img) - 0.5
 * (fy_l likewise), and the samples of all levels are summed inside the valid
 * mean:
 *   out[b, c, i, j] = sum_k [cnt > 0] (1 / cnt) sum_{valid n} sum_l bilinear(F_l[b, n, c], fx_l, fy_l)
 * With one level this is bev_sample_forward.  The levels are combined by an
 * unweighted sum (the notes name the direction, not a combination rule); a
 * corner outside level l's map contributes zero at that level only.
 * ------------------------------------------------------------------------- */

/* Pyramid levels accepted by the multi-scale calls. */
#define BEV_MAX_LEVELS 4

/* Workspace bytes of bev_sample_forward_multiscale (for_backward = 0) or
 * bev_sample_backward_multiscale (for_backward = 1): the per-level sizes of
 * bev_workspace_size, each rounded up to 256 bytes, summed.  Hf, Wf are host
 * arrays of nlevels entries.  Returns (size_t)-1 for invalid sizes. */
size_t bev_multiscale_workspace_size(int dtype, int layout, int B, int N, int C, int nlevels,
                                     const int* Hf, const int* Wf, int for_backward);

/* Forward over nlevels (1..BEV_MAX_LEVELS) pyramid levels.
 *   features    host array of nlevels device pointers; level l is
 *               [B,N,C,Hf[l],Wf[l]] (BEV_NCHW) or [B,N,Hf[l],Wf[l],C] (BEV_NHWC),
 *               all levels of one dtype and layout
 *   Hf, Wf      host arrays of nlevels map sizes (any sizes; not necessarily halvings)
 *   out         [B,C,X,Y] fp32, fully overwritten; valid_count as for bev_sample_forward
 *   workspace   at least bev_multiscale_workspace_size(.., 0) bytes, 256-byte aligned
 *               (may be NULL when that size is 0)
 * Other arguments, checks and errors as for bev_sample_forward; nlevels
 * outside 1..BEV_MAX_LEVELS or a NULL level pointer -> BEV_ERR_INVALID_ARG. */
int bev_sample_forward_multiscale(const void* const* features, int nlevels, const int* Hf, const int* Wf,
                                  int dtype, int layout, int B, int N, int C,
                                  const float* intrinsics, const float* ego2cam,
                                  int img_h, int img_w, const bev_grid_t* grid,
                                  float* out, uint8_t* valid_count,
                                  void* workspace, size_t workspace_bytes, bev_stream_t stream);

/* Backward of bev_sample_forward_multiscale with respect to every level's
 * features: dF_l[b, n, c, y, x] = sum of w_l * dout[b, c, i, j] / cnt_k over
 * the valid samples whose level-l corners touch texel (y, x).
 *   dfeatures   host array of nlevels device pointers, level l [B,N,C,Hf[l],Wf[l]]
 *               fp32, fully overwritten
 *   workspace   at least bev_multiscale_workspace_size(.., 1) bytes, 256-byte aligned
 * Other arguments and errors as for bev_sample_backward. */
int bev_sample_backward_multiscale(const float* dout, int nlevels, const int* Hf, const int* Wf,
                                   int B, int N, int C, const float* intrinsics, const float* ego2cam,
                                   int img_h, int img_w, const bev_grid_t* grid,
                                   float* const* dfeatures, void* workspace, size_t workspace_bytes,
                                   bev_stream_t stream);

/* ---------------------------------------------------------------------------
 * Deformable aggregation (SparseDriveV2 notes, "Deformable Aggregation",
 * steps 1-3).  Each query q of batch item b has a 3-D anchor a and Kp
 * keypoint offsets d_k; its keypoints p_k = a + d_k (fp32 sums, ego frame)
 * are projected into every camera with the same geometry and validity test
 * as bev_sample_forward, sampled bilinearly (align_corners=False, zero
 * padding) where valid, and summed with per-(camera, keypoint) weights:
 *   out[b, q, c] = sum_n sum_k [valid(b, n, p_k)] w[b, q, n, k] * bilinear(F[b, n, c], p_k)
 * There is no normalisation beyond the given weights.
 * ------------------------------------------------------------------------- */

/* Keypoints per query accepted by the deformable-aggregation calls. */
#define BEV_DEFORM_MAX_KEYPOINTS 64

/* Device scratch (bytes, 256-byte aligned) that bev_deform_forward
 * (for_backward = 0) or bev_deform_backward (for_backward = 1) needs; 0 when
 * none.  (size_t)-1 for invalid arguments. */
size_t bev_deform_workspace_size(int dtype, int layout, int B, int N, int C, int Hf, int Wf, int for_backward);

/* Forward of the deformable aggregation.
 *   features     as for bev_sample_forward; C <= 512 (fp32) or 1024 (bf16)
 *   intrinsics, ego2cam, img_h, img_w   as for bev_sample_forward
 *   anchors      [B,Q,3] fp32, ego frame
 *   offsets      [B,Q,Kp,3] fp32
 *   weights      [B,Q,N,Kp] fp32
 *   Q, Kp        queries per batch item (>= 1), keypoints per query
 *                (1..BEV_DEFORM_MAX_KEYPOINTS)
 *   out          [B,Q,C] fp32, fully overwritten
 *   workspace    at least bev_deform_workspace_size(dtype, layout, ..., 0) bytes
 * Each query is one CTA whose warps split its (camera, keypoint) pairs and
 * add their partial sums in a fixed order, so results are reproducible bit
 * for bit.  Returns BEV_OK, BEV_ERR_INVALID_ARG,
 * BEV_ERR_UNSUPPORTED, BEV_ERR_WORKSPACE or BEV_ERR_CUDA. */
int bev_deform_forward(const void* features, int dtype, int layout, int B, int N, int C, int Hf, int Wf,
                       const float* intrinsics, const float* ego2cam, int img_h, int img_w,
                       const float* anchors, const float* offsets, const float* weights, int Q, int Kp,
                       float* out, void* workspace, size_t workspace_bytes, bev_stream_t stream);

/* Backward of the deformable aggregation for dout [B,Q,C] fp32:
 *   dfeatures  [B,N,C,Hf,Wf] fp32   adjoint in the features
 *   dweights   [B,Q,N,Kp] fp32      the sample against dout for valid (n, k), else 0
 *   doffsets   [B,Q,Kp,3] fp32      through the sampling position: the bilinear
 *              derivative inside its cell, carried through u = uh / depth and
 *              the extrinsic rotation; the validity test and the choice of cell
 *              are held fixed (no gradient flows through them).  The anchor
 *              gradient is the sum of a query's keypoint rows.
 * All three are fully overwritten.  features as for bev_deform_forward (the
 * backward reads them for dweights and doffsets); workspace at least
 * bev_deform_workspace_size(.., 1) bytes.  dweights and doffsets are
 * reproducible bit for bit; dfeatures is accumulated with atomics, so repeated
 * calls may differ in the last bits. */
int bev_deform_backward(const void* features, int dtype, int layout, int B, int N, int C, int Hf, int Wf,
                        const float* intrinsics, const float* ego2cam, int img_h, int img_w,
                        const float* anchors, const float* offsets, const float* weights, int Q, int Kp,
                        const float* dout, float* dfeatures, float* dweights, float* doffsets,
                        void* workspace, size_t workspace_bytes, bev_stream_t stream);

/* ---------------------------------------------------------------------------
 * Lift-splat BEV pooling (LSS tutorial, "Lift" and "Splat").  Every feature
 * pixel (h, w) of camera n spreads D depth bins along its ray; bin k sits at
 * depth dmin + k * dstep, at the pixel centre u = (w + 0.5) W_img / Wf,
 * v = (h + 0.5) H_img / Hf.  Its point, depth * K^-1 [u v 1]^T in the camera
 * frame, is placed in the ego frame as R^T (pc - t) (E = [R | t] maps ego to
 * camera, R a rotation; K upper triangular) and carries
 * depth[b,n,k,h,w] * feat[b,n,:,h,w].  Points are summed into the BEV pillar
 * (i, j) = (floor((x - xmin) / dx), floor((y - ymin) / dy)); z is not binned
 * and points outside [xmin, xmax) x [ymin, ymax) x [zmin, zmax) are dropped:
 *   out[b, c, i, j] = sum over points in pillar (i, j) of depth * feat[c]
 * grid: from bev_grid_spec; X, Y, xmin, ymin, zmin, zmax, dx, dy are used, Z
 * is ignored.  The fp32 order of the geometry is fixed (separate roundings,
 * IEEE divides):
 *   yn = (v - K12) / K11;  xn = ((u - K02) - K01 yn) / K00;  pc = (xn d, yn d, d)
 *   q = pc - t;  x = (R00 q0 + R10 q1) + R20 q2  (likewise y, z)
 * ------------------------------------------------------------------------- */

/* Device scratch (bytes, 256-byte aligned) of bev_lss_forward (for_backward
 * = 0) or bev_lss_backward (1); (size_t)-1 for invalid arguments. */
size_t bev_lss_workspace_size(int B, int N, int C, int D, int Hf, int Wf, int X, int Y, int for_backward);

/* Forward of the lift-splat pooling.
 *   depth      [B,N,D,Hf,Wf] fp32 (for instance a softmax over the bins)
 *   feat       [B,N,C,Hf,Wf] fp32, C <= 256
 *   intrinsics [B,N,3,3], ego2cam [B,N,4,4] fp32; img_h, img_w the image size
 *   dmin, dstep  depth of bin 0 and the bin spacing (> 0)
 *   out        [B,C,X,Y] fp32, fully overwritten
 * Each term depth * feat is rounded to a 64-bit fixed point with s fraction
 * bits, s = 62 - e(max|depth| max|feat|) - e(N D Hf Wf) (e(v): the smallest e
 * with v < 2^e) clamped to [-126, 127] (max|depth| max|feat| must be finite in
 * fp32), and the pillar sums are exact integer sums, so results are
 * reproducible bit for bit whatever the order of the points; the absolute
 * error of a pillar is at most (its points) * 2^-(s+1) plus the final
 * rounding to fp32.  Returns BEV_OK, BEV_ERR_INVALID_ARG, BEV_ERR_UNSUPPORTED,
 * BEV_ERR_WORKSPACE or BEV_ERR_CUDA. */
int bev_lss_forward(const float* depth, const float* feat, int B, int N, int D, int C, int Hf, int Wf,
                    const float* intrinsics, const float* ego2cam, int img_h, int img_w, float dmin, float dstep,
                    const bev_grid_t* grid, float* out, void* workspace, size_t workspace_bytes,
                    bev_stream_t stream);

/* Backward of the lift-splat pooling for dout [B,C,X,Y] fp32:
 *   ddepth [B,N,D,Hf,Wf] = dout[pillar of the point] . feat (0 for dropped points)
 *   dfeat  [B,N,C,Hf,Wf] = sum_k depth * dout[pillar of bin k]
 * Both fully overwritten; a gather in a fixed order, so reproducible bit for
 * bit.  Other arguments as for bev_lss_forward. */
int bev_lss_backward(const float* depth, const float* feat, const float* dout, int B, int N, int D, int C,
                     int Hf, int Wf, const float* intrinsics, const float* ego2cam, int img_h, int img_w,
                     float dmin, float dstep, const bev_grid_t* grid, float* ddepth, float* dfeat,
                     void* workspace, size_t workspace_bytes, bev_stream_t stream);

/* Static, human-readable text for a status code. */
const char* bev_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* BEVSAMPLE_H */
