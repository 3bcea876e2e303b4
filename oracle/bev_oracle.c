/*
 * bev_oracle.c -- CPU oracle for the exact dense Sampling-VT gather-reduction.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links or calls this
 * file; only the tests, the smoke check and the bench's CPU-baseline leg do.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (FlashBEV reading notes, "Core Idea" and "Method" item 1):
 * for every BEV output element (b, c, i, j) and every height bin k, each camera
 * n projects the voxel centre, the valid cameras' bilinear samples are averaged
 * ("valid mean" per height bin), and the per-bin means are summed over height
 * (the notes' "Key Insight": a height sum, not a learned height reduction).
 *
 *   voxel centre      x_i = xmin + (i + 0.5) dx  (same for y_j, z_k)
 *   projection        [u v 1]^T ~ K (R p + t)    (SparseDriveV2 notes,
 *                     "Deformable Aggregation", step 2; E = [R|t] maps ego to
 *                     camera, per the same section's pitfalls)
 *   validity          depth = camera z > 0.1 and (u, v) in [0, W_img] x [0, H_img]
 *                     (same step: the projection must land inside the image)
 *   sampling          bilinear, align_corners=False, zero padding:
 *                     fx = u * Wf / W_img - 0.5, fy = v * Hf / H_img - 0.5
 *                     (same section's pitfalls: bilinear, so gradients flow)
 *   reduction         out = sum_k [cnt_k > 0] (1 / cnt_k) sum_{n valid} sample_n
 *
 * Precision.  Geometry follows one fixed fp32 expression order, every product
 * and sum rounded on its own (this file must be compiled with
 * -ffp-contract=off and SSE float arithmetic), so that the validity counts --
 * integers decided by floating point -- come out identical on any IEEE
 * machine that evaluates the same expression:
 *   pc_r = ((E_r0 x + E_r1 y) + E_r2 z) + E_r3
 *   uh   = (K_00 pc_x + K_01 pc_y) + K_02 pc_z,   u = uh / pc_z   (IEEE divide)
 *   fx   = u * (Wf / W_img) - 0.5,  x0 = floor(fx), wx1 = fx - x0, wx0 = 1 - wx1
 *   corner weight w = wy * wx
 * Accumulation of features times weights is done in fp64.  Alongside each
 * result the oracle returns a condition bound: the same sum taken over
 * absolute values of the terms, which scales the parity tolerance.
 *
 * Where the notes are silent this oracle takes these readings: the image test
 * is closed on both ends; a camera that passes the test counts towards the
 * mean even if some bilinear corners fall outside the feature map (those
 * corners contribute zero); an empty height bin contributes zero; K's last row
 * is taken to be [0 0 1] and E's bottom row is ignored.
 *
 * Backward: the operator is linear in the features, so dL/dF is the adjoint:
 *   dF[b,n,c,y,x] += w * dout[b,c,i,j] / cnt_k  over every valid sample and
 *   in-range corner (y, x) it touches.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Grid from ranges and resolutions.  counts = round(extent / res) when that
 * ratio is within 1e-4 of an integer, else failure; the cell size used for
 * the centres is recomputed as extent / count in fp32.  Returns 0 on success. */
int oracle_grid_spec(const float range[6], const float res[3], int counts[3], float cell[3])
{
    for (int a = 0; a < 3; ++a) {
        float lo = range[2 * a], hi = range[2 * a + 1];
        if (!(isfinite(lo) && isfinite(hi) && isfinite(res[a]))) return 1;
        if (!(hi > lo) || !(res[a] > 0.0f)) return 1;
        float extent = hi - lo;
        double ratio = (double)extent / (double)res[a];
        double nearest = floor(ratio + 0.5);
        if (fabs(ratio - nearest) > 1e-4 || nearest < 1.0 || nearest > 1e6) return 1;
        counts[a] = (int)nearest;
        cell[a] = extent / (float)counts[a];
    }
    return 0;
}

/* Voxel centre along one axis, fp32: lo + ((float)i + 0.5f) * d. */
static float centre(float lo, int i, float d)
{
    float t = (float)i + 0.5f;
    t = t * d;
    return lo + t;
}

/* Project one ego point through one camera.  Returns 1 when valid and writes
 * the feature-map sampling position (fx, fy) and the image position (u, v). */
int oracle_project(const float* K, const float* E, float px, float py, float pz,
                   int img_h, int img_w, int Hf, int Wf,
                   float* u_out, float* v_out, float* fx_out, float* fy_out)
{
    float pc[3];
    for (int r = 0; r < 3; ++r) {
        float t = E[4 * r + 0] * px;
        float s = E[4 * r + 1] * py;
        t = t + s;
        s = E[4 * r + 2] * pz;
        t = t + s;
        t = t + E[4 * r + 3];
        pc[r] = t;
    }
    float depth = pc[2];
    if (!(depth > 0.1f)) return 0;
    float uh = K[0] * pc[0];
    float s = K[1] * pc[1];
    uh = uh + s;
    s = K[2] * pc[2];
    uh = uh + s;
    float vh = K[3] * pc[0];
    s = K[4] * pc[1];
    vh = vh + s;
    s = K[5] * pc[2];
    vh = vh + s;
    float u = uh / depth;
    float v = vh / depth;
    *u_out = u;
    *v_out = v;
    if (!(u >= 0.0f && u <= (float)img_w && v >= 0.0f && v <= (float)img_h)) return 0;
    float sW = (float)Wf / (float)img_w;
    float sH = (float)Hf / (float)img_h;
    float fx = u * sW;
    fx = fx - 0.5f;
    float fy = v * sH;
    fy = fy - 0.5f;
    *fx_out = fx;
    *fy_out = fy;
    return 1;
}

/* The four bilinear corners of (fx, fy): feature-map row/col and weight. */
static void corners(float fx, float fy, int ys[4], int xs[4], float ws[4])
{
    float x0f = floorf(fx), y0f = floorf(fy);
    float wx1 = fx - x0f, wy1 = fy - y0f;
    float wx0 = 1.0f - wx1, wy0 = 1.0f - wy1;
    int x0 = (int)x0f, y0 = (int)y0f;
    ys[0] = y0;     xs[0] = x0;     ws[0] = wy0 * wx0;
    ys[1] = y0;     xs[1] = x0 + 1; ws[1] = wy0 * wx1;
    ys[2] = y0 + 1; xs[2] = x0;     ws[2] = wy1 * wx0;
    ys[3] = y0 + 1; xs[3] = x0 + 1; ws[3] = wy1 * wx1;
}

/* Forward.  features [B,N,C,Hf,Wf] fp64 (exact copies of the fp32/bf16
 * inputs); K [B,N,3,3], E [B,N,4,4] fp32; counts X,Y,Z; lo = (xmin,ymin,zmin);
 * cell = (dx,dy,dz).  Writes out and bound [B,C,X,Y] fp64 and count
 * [B,X,Y,Z] int32.  Rows (b, i) are independent and may run on `threads`
 * OpenMP threads; each output element's arithmetic is unchanged by that. */
void oracle_forward(const double* F, int B, int N, int C, int Hf, int Wf,
                    const float* K, const float* E, int img_h, int img_w,
                    int X, int Y, int Z, const float lo[3], const float cell[3],
                    double* out, double* bound, int32_t* count, int threads)
{
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel for schedule(dynamic)
#endif
    for (long bi = 0; bi < (long)B * X; ++bi) {
        int b = (int)(bi / X), i = (int)(bi % X);
        double* acc = (double*)malloc(sizeof(double) * 4 * (size_t)C);
        double* abs_acc = acc + C;
        double* s = acc + 2 * C;
        double* a = acc + 3 * C;
        float x = centre(lo[0], i, cell[0]);
        for (int j = 0; j < Y; ++j) {
            float y = centre(lo[1], j, cell[1]);
            for (int c = 0; c < C; ++c) { acc[c] = 0.0; abs_acc[c] = 0.0; }
            for (int k = 0; k < Z; ++k) {
                float z = centre(lo[2], k, cell[2]);
                for (int c = 0; c < C; ++c) { s[c] = 0.0; a[c] = 0.0; }
                int cnt = 0;
                for (int n = 0; n < N; ++n) {
                    const float* Kn = K + ((size_t)b * N + n) * 9;
                    const float* En = E + ((size_t)b * N + n) * 16;
                    float u, v, fx, fy;
                    if (!oracle_project(Kn, En, x, y, z, img_h, img_w, Hf, Wf, &u, &v, &fx, &fy))
                        continue;
                    ++cnt;
                    int ys[4], xs[4];
                    float ws[4];
                    corners(fx, fy, ys, xs, ws);
                    for (int q = 0; q < 4; ++q) {
                        if (ys[q] < 0 || ys[q] >= Hf || xs[q] < 0 || xs[q] >= Wf) continue;
                        const double* Fp = F + (((size_t)b * N + n) * C * Hf + ys[q]) * Wf + xs[q];
                        for (int c = 0; c < C; ++c) {
                            double term = (double)ws[q] * Fp[(size_t)c * Hf * Wf];
                            s[c] += term;
                            a[c] += fabs(term);
                        }
                    }
                }
                count[(((size_t)b * X + i) * Y + j) * Z + k] = cnt;
                if (cnt > 0) {
                    for (int c = 0; c < C; ++c) {
                        acc[c] += s[c] / cnt;
                        abs_acc[c] += a[c] / cnt;
                    }
                }
            }
            for (int c = 0; c < C; ++c) {
                size_t o = (((size_t)b * C + c) * X + i) * Y + j;
                out[o] = acc[c];
                bound[o] = abs_acc[c];
            }
        }
        free(acc);
    }
}

/* Backward (gradient with respect to the features only).  dout [B,C,X,Y]
 * fp64.  Writes dF and dbound [B,N,C,Hf,Wf] fp64 (overwritten).  Work is split
 * over (b, n) pairs so that each thread owns its slice of dF. */
void oracle_backward(const double* dout, int B, int N, int C, int Hf, int Wf,
                     const float* K, const float* E, int img_h, int img_w,
                     int X, int Y, int Z, const float lo[3], const float cell[3],
                     double* dF, double* dbound, int threads)
{
    memset(dF, 0, sizeof(double) * (size_t)B * N * C * Hf * Wf);
    memset(dbound, 0, sizeof(double) * (size_t)B * N * C * Hf * Wf);
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel for schedule(dynamic)
#endif
    for (long bn = 0; bn < (long)B * N; ++bn) {
        int b = (int)(bn / N), n = (int)(bn % N);
        const float* Kn = K + ((size_t)b * N + n) * 9;
        const float* En = E + ((size_t)b * N + n) * 16;
        double* dFn = dF + ((size_t)b * N + n) * C * Hf * Wf;
        double* dBn = dbound + ((size_t)b * N + n) * C * Hf * Wf;
        for (int i = 0; i < X; ++i) {
            float x = centre(lo[0], i, cell[0]);
            for (int j = 0; j < Y; ++j) {
                float y = centre(lo[1], j, cell[1]);
                for (int k = 0; k < Z; ++k) {
                    float z = centre(lo[2], k, cell[2]);
                    float u, v, fx, fy;
                    int cnt = 0;
                    for (int m = 0; m < N; ++m) {
                        const float* Km = K + ((size_t)b * N + m) * 9;
                        const float* Em = E + ((size_t)b * N + m) * 16;
                        cnt += oracle_project(Km, Em, x, y, z, img_h, img_w, Hf, Wf, &u, &v, &fx, &fy);
                    }
                    if (!oracle_project(Kn, En, x, y, z, img_h, img_w, Hf, Wf, &u, &v, &fx, &fy))
                        continue;
                    int ys[4], xs[4];
                    float ws[4];
                    corners(fx, fy, ys, xs, ws);
                    for (int q = 0; q < 4; ++q) {
                        if (ys[q] < 0 || ys[q] >= Hf || xs[q] < 0 || xs[q] >= Wf) continue;
                        for (int c = 0; c < C; ++c) {
                            double g = dout[(((size_t)b * C + c) * X + i) * Y + j];
                            double term = (double)ws[q] * g / cnt;
                            size_t o = ((size_t)c * Hf + ys[q]) * Wf + xs[q];
                            dFn[o] += term;
                            dBn[o] += fabs(term);
                        }
                    }
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------
 * Multi-scale dense Sampling-VT (FlashBEV reading notes, "Takeaway" 4:
 * multi-scale fused view transformation; SparseDriveV2 notes, "Image
 * Encoder": an FPN gives each camera feature maps P_l at several resolutions
 * with a common channel count).  The geometry of a voxel is that of the
 * single-level operator above: one projection (u, v) in image pixels, one
 * validity test, one count per height bin.  Each level l samples its own map
 * at its own scale, fx_l = u * (W_l / W_img) - 0.5 (fy_l likewise), and the
 * samples of all levels are summed inside the valid mean:
 *
 *   out[b,c,i,j] = sum_k [cnt_k > 0] (1 / cnt_k) sum_{n valid} sum_l bilinear(F_l[b,n,c], fx_l, fy_l)
 *
 * Readings (the notes name the direction only): the levels are combined by
 * an unweighted sum, so that with one level this is the operator above; the
 * count does not depend on the level (validity is an image-plane test); a
 * corner outside level l's map contributes zero at that level only.
 * ---------------------------------------------------------------------- */

/* Forward.  F[l] = level l's features [B,N,C,H[l],W[l]] fp64; the rest as in
 * oracle_forward. */
void oracle_ms_forward(const double* const* F, int nlev, const int* H, const int* W, int B, int N, int C,
                       const float* K, const float* E, int img_h, int img_w,
                       int X, int Y, int Z, const float lo[3], const float cell[3],
                       double* out, double* bound, int32_t* count, int threads)
{
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel for schedule(dynamic)
#endif
    for (long bi = 0; bi < (long)B * X; ++bi) {
        int b = (int)(bi / X), i = (int)(bi % X);
        double* acc = (double*)malloc(sizeof(double) * 4 * (size_t)C);
        double* abs_acc = acc + C;
        double* s = acc + 2 * C;
        double* a = acc + 3 * C;
        float x = centre(lo[0], i, cell[0]);
        for (int j = 0; j < Y; ++j) {
            float y = centre(lo[1], j, cell[1]);
            for (int c = 0; c < C; ++c) { acc[c] = 0.0; abs_acc[c] = 0.0; }
            for (int k = 0; k < Z; ++k) {
                float z = centre(lo[2], k, cell[2]);
                for (int c = 0; c < C; ++c) { s[c] = 0.0; a[c] = 0.0; }
                int cnt = 0;
                for (int n = 0; n < N; ++n) {
                    const float* Kn = K + ((size_t)b * N + n) * 9;
                    const float* En = E + ((size_t)b * N + n) * 16;
                    float u, v, fx, fy;
                    /* validity is the image-plane test: any level's sizes give it */
                    if (!oracle_project(Kn, En, x, y, z, img_h, img_w, H[0], W[0], &u, &v, &fx, &fy))
                        continue;
                    ++cnt;
                    for (int l = 0; l < nlev; ++l) {
                        oracle_project(Kn, En, x, y, z, img_h, img_w, H[l], W[l], &u, &v, &fx, &fy);
                        int ys[4], xs[4];
                        float ws[4];
                        corners(fx, fy, ys, xs, ws);
                        for (int q = 0; q < 4; ++q) {
                            if (ys[q] < 0 || ys[q] >= H[l] || xs[q] < 0 || xs[q] >= W[l]) continue;
                            const double* Fp = F[l] + (((size_t)b * N + n) * C * H[l] + ys[q]) * W[l] + xs[q];
                            for (int c = 0; c < C; ++c) {
                                double term = (double)ws[q] * Fp[(size_t)c * H[l] * W[l]];
                                s[c] += term;
                                a[c] += fabs(term);
                            }
                        }
                    }
                }
                count[(((size_t)b * X + i) * Y + j) * Z + k] = cnt;
                if (cnt > 0) {
                    for (int c = 0; c < C; ++c) {
                        acc[c] += s[c] / cnt;
                        abs_acc[c] += a[c] / cnt;
                    }
                }
            }
            for (int c = 0; c < C; ++c) {
                size_t o = (((size_t)b * C + c) * X + i) * Y + j;
                out[o] = acc[c];
                bound[o] = abs_acc[c];
            }
        }
        free(acc);
    }
}

/* Backward: dF[l] and dbound[l] [B,N,C,H[l],W[l]] fp64 (overwritten). */
void oracle_ms_backward(const double* dout, int nlev, const int* H, const int* W, int B, int N, int C,
                        const float* K, const float* E, int img_h, int img_w,
                        int X, int Y, int Z, const float lo[3], const float cell[3],
                        double* const* dF, double* const* dbound, int threads)
{
    for (int l = 0; l < nlev; ++l) {
        memset(dF[l], 0, sizeof(double) * (size_t)B * N * C * H[l] * W[l]);
        memset(dbound[l], 0, sizeof(double) * (size_t)B * N * C * H[l] * W[l]);
    }
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel for schedule(dynamic)
#endif
    for (long bn = 0; bn < (long)B * N; ++bn) {
        int b = (int)(bn / N), n = (int)(bn % N);
        const float* Kn = K + ((size_t)b * N + n) * 9;
        const float* En = E + ((size_t)b * N + n) * 16;
        for (int i = 0; i < X; ++i) {
            float x = centre(lo[0], i, cell[0]);
            for (int j = 0; j < Y; ++j) {
                float y = centre(lo[1], j, cell[1]);
                for (int k = 0; k < Z; ++k) {
                    float z = centre(lo[2], k, cell[2]);
                    float u, v, fx, fy;
                    int cnt = 0;
                    for (int m = 0; m < N; ++m) {
                        const float* Km = K + ((size_t)b * N + m) * 9;
                        const float* Em = E + ((size_t)b * N + m) * 16;
                        cnt += oracle_project(Km, Em, x, y, z, img_h, img_w, H[0], W[0], &u, &v, &fx, &fy);
                    }
                    if (!oracle_project(Kn, En, x, y, z, img_h, img_w, H[0], W[0], &u, &v, &fx, &fy))
                        continue;
                    for (int l = 0; l < nlev; ++l) {
                        oracle_project(Kn, En, x, y, z, img_h, img_w, H[l], W[l], &u, &v, &fx, &fy);
                        double* dFn = dF[l] + ((size_t)b * N + n) * C * H[l] * W[l];
                        double* dBn = dbound[l] + ((size_t)b * N + n) * C * H[l] * W[l];
                        int ys[4], xs[4];
                        float ws[4];
                        corners(fx, fy, ys, xs, ws);
                        for (int q = 0; q < 4; ++q) {
                            if (ys[q] < 0 || ys[q] >= H[l] || xs[q] < 0 || xs[q] >= W[l]) continue;
                            for (int c = 0; c < C; ++c) {
                                double g = dout[(((size_t)b * C + c) * X + i) * Y + j];
                                double term = (double)ws[q] * g / cnt;
                                size_t o = ((size_t)c * H[l] + ys[q]) * W[l] + xs[q];
                                dFn[o] += term;
                                dBn[o] += fabs(term);
                            }
                        }
                    }
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------
 * Deformable aggregation (SparseDriveV2 notes, "Deformable Aggregation",
 * steps 1-3): a query with 3-D anchor a and keypoint offsets d_k samples the
 * cameras at its keypoints p_k = a + d_k (step 1), each projected as above
 * and kept only where valid (step 2), and sums the bilinear samples with
 * weights w_{n,k} (step 3):
 *
 *   out[b,q,c] = sum_n sum_k [valid(b,n,p_k)] w[b,q,n,k] * bilinear(F[b,n,c], fx, fy)
 *
 * Readings: the keypoint is a + d_k rounded to fp32 once per coordinate; the
 * sampler phi of the notes is the same bilinear (align_corners=False, zero
 * padding) as the dense path, the "small neighbourhood" being its 2x2 taps;
 * no normalisation beyond the given weights; validity as in oracle_project.
 * ---------------------------------------------------------------------- */

static void keypoint(const float* anchors, const float* offsets, int b, int q, int k, int Q, int Kp,
                     float p[3])
{
    const float* a = anchors + ((size_t)b * Q + q) * 3;
    const float* d = offsets + (((size_t)b * Q + q) * Kp + k) * 3;
    for (int r = 0; r < 3; ++r) p[r] = a[r] + d[r];
}

/* Forward.  F [B,N,C,Hf,Wf] fp64 (exact copies); anchors [B,Q,3], offsets
 * [B,Q,Kp,3], weights [B,Q,N,Kp] fp32.  Writes out and bound [B,Q,C] fp64. */
void oracle_deform_forward(const double* F, int B, int N, int C, int Hf, int Wf,
                           const float* K, const float* E, int img_h, int img_w,
                           const float* anchors, const float* offsets, const float* W, int Q, int Kp,
                           double* out, double* bound, int threads)
{
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel for schedule(dynamic)
#endif
    for (long bq = 0; bq < (long)B * Q; ++bq) {
        int b = (int)(bq / Q), q = (int)(bq % Q);
        double* acc = out + (size_t)bq * C;
        double* abs_acc = bound + (size_t)bq * C;
        for (int c = 0; c < C; ++c) { acc[c] = 0.0; abs_acc[c] = 0.0; }
        for (int n = 0; n < N; ++n) {
            const float* Kn = K + ((size_t)b * N + n) * 9;
            const float* En = E + ((size_t)b * N + n) * 16;
            for (int k = 0; k < Kp; ++k) {
                float p[3], u, v, fx, fy;
                keypoint(anchors, offsets, b, q, k, Q, Kp, p);
                if (!oracle_project(Kn, En, p[0], p[1], p[2], img_h, img_w, Hf, Wf, &u, &v, &fx, &fy))
                    continue;
                double w = W[(((size_t)b * Q + q) * N + n) * Kp + k];
                int ys[4], xs[4];
                float ws[4];
                corners(fx, fy, ys, xs, ws);
                for (int t = 0; t < 4; ++t) {
                    if (ys[t] < 0 || ys[t] >= Hf || xs[t] < 0 || xs[t] >= Wf) continue;
                    const double* Fp = F + (((size_t)b * N + n) * C * Hf + ys[t]) * Wf + xs[t];
                    for (int c = 0; c < C; ++c) {
                        double term = w * (double)ws[t] * Fp[(size_t)c * Hf * Wf];
                        acc[c] += term;
                        abs_acc[c] += fabs(term);
                    }
                }
            }
        }
    }
}

/* Backward for dout [B,Q,C] fp64:
 *   dF [B,N,C,Hf,Wf]  adjoint of the forward in F;
 *   dW [B,Q,N,Kp]     sum_c dout * bilinear(F, fx, fy)  for valid (n, k), else 0;
 *   dOff [B,Q,Kp,3]   derivative through the sampling position: with
 *                     g = sum_c dout_c dphi_c/d(fx, fy) (the derivative of the
 *                     zero-padded bilinear interpolant inside its cell),
 *                     fx = u Wf/W_img - 0.5, u = uh / pc_z, pc = R p + t:
 *                     dOff += w * R^T (g_x (Wf/W_img) du/dpc + g_y (Hf/H_img) dv/dpc),
 *                     du/dpc = (K_00, K_01, K_02 - u) / pc_z, likewise v.
 *                     The validity test and the corner choice are held fixed
 *                     (no gradient flows through them), as for the dense path.
 * Each output gets a bound (sum of absolute terms) of the same shape.  dF is
 * split over (b, n), dW and dOff over (b, q). */
void oracle_deform_backward(const double* F, const double* dout, int B, int N, int C, int Hf, int Wf,
                            const float* K, const float* E, int img_h, int img_w,
                            const float* anchors, const float* offsets, const float* W, int Q, int Kp,
                            double* dF, double* dFb, double* dW, double* dWb, double* dOff, double* dOffb,
                            int threads)
{
    memset(dF, 0, sizeof(double) * (size_t)B * N * C * Hf * Wf);
    memset(dFb, 0, sizeof(double) * (size_t)B * N * C * Hf * Wf);
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel for schedule(dynamic)
#endif
    for (long bn = 0; bn < (long)B * N; ++bn) {
        int b = (int)(bn / N), n = (int)(bn % N);
        const float* Kn = K + ((size_t)b * N + n) * 9;
        const float* En = E + ((size_t)b * N + n) * 16;
        double* dFn = dF + (size_t)bn * C * Hf * Wf;
        double* dBn = dFb + (size_t)bn * C * Hf * Wf;
        for (int q = 0; q < Q; ++q) {
            const double* g = dout + ((size_t)b * Q + q) * C;
            for (int k = 0; k < Kp; ++k) {
                float p[3], u, v, fx, fy;
                keypoint(anchors, offsets, b, q, k, Q, Kp, p);
                if (!oracle_project(Kn, En, p[0], p[1], p[2], img_h, img_w, Hf, Wf, &u, &v, &fx, &fy))
                    continue;
                double w = W[(((size_t)b * Q + q) * N + n) * Kp + k];
                int ys[4], xs[4];
                float ws[4];
                corners(fx, fy, ys, xs, ws);
                for (int t = 0; t < 4; ++t) {
                    if (ys[t] < 0 || ys[t] >= Hf || xs[t] < 0 || xs[t] >= Wf) continue;
                    for (int c = 0; c < C; ++c) {
                        double term = w * (double)ws[t] * g[c];
                        size_t o = ((size_t)c * Hf + ys[t]) * Wf + xs[t];
                        dFn[o] += term;
                        dBn[o] += fabs(term);
                    }
                }
            }
        }
    }
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic)
#endif
    for (long bq = 0; bq < (long)B * Q; ++bq) {
        int b = (int)(bq / Q), q = (int)(bq % Q);
        const double* g = dout + (size_t)bq * C;
        double* dO = dOff + (size_t)bq * Kp * 3;
        double* dOb = dOffb + (size_t)bq * Kp * 3;
        for (int t = 0; t < Kp * 3; ++t) { dO[t] = 0.0; dOb[t] = 0.0; }
        for (int n = 0; n < N; ++n) {
            const float* Kn = K + ((size_t)b * N + n) * 9;
            const float* En = E + ((size_t)b * N + n) * 16;
            for (int k = 0; k < Kp; ++k) {
                size_t wi = (((size_t)b * Q + q) * N + n) * Kp + k;
                dW[wi] = 0.0;
                dWb[wi] = 0.0;
                float p[3], u, v, fx, fy;
                keypoint(anchors, offsets, b, q, k, Q, Kp, p);
                if (!oracle_project(Kn, En, p[0], p[1], p[2], img_h, img_w, Hf, Wf, &u, &v, &fx, &fy))
                    continue;
                double w = W[wi];
                int ys[4], xs[4];
                float ws[4];
                corners(fx, fy, ys, xs, ws);
                /* d(weight of corner t)/dfx and /dfy inside the cell */
                double wx1 = (double)fx - floor((double)fx), wy1 = (double)fy - floor((double)fy);
                double wx0 = 1.0 - wx1, wy0 = 1.0 - wy1;
                double dwx[4] = {-wy0, wy0, -wy1, wy1};
                double dwy[4] = {-wx0, -wx1, wx0, wx1};
                double s = 0.0, sb = 0.0, gx = 0.0, gxb = 0.0, gy = 0.0, gyb = 0.0;
                for (int t = 0; t < 4; ++t) {
                    if (ys[t] < 0 || ys[t] >= Hf || xs[t] < 0 || xs[t] >= Wf) continue;
                    const double* Fp = F + (((size_t)b * N + n) * C * Hf + ys[t]) * Wf + xs[t];
                    for (int c = 0; c < C; ++c) {
                        double fg = Fp[(size_t)c * Hf * Wf] * g[c];
                        s += (double)ws[t] * fg;
                        sb += fabs((double)ws[t] * fg);
                        gx += dwx[t] * fg;
                        gxb += fabs(dwx[t] * fg);
                        gy += dwy[t] * fg;
                        gyb += fabs(dwy[t] * fg);
                    }
                }
                dW[wi] = s;
                dWb[wi] = sb;
                /* chain rule through the projection, in fp64 */
                double pc[3];
                for (int r = 0; r < 3; ++r)
                    pc[r] = (double)En[4 * r] * p[0] + (double)En[4 * r + 1] * p[1] + (double)En[4 * r + 2] * p[2] +
                            (double)En[4 * r + 3];
                double uu = ((double)Kn[0] * pc[0] + (double)Kn[1] * pc[1] + (double)Kn[2] * pc[2]) / pc[2];
                double vv = ((double)Kn[3] * pc[0] + (double)Kn[4] * pc[1] + (double)Kn[5] * pc[2]) / pc[2];
                double sW = (double)((float)Wf / (float)img_w), sH = (double)((float)Hf / (float)img_h);
                double du[3] = {Kn[0] / pc[2], Kn[1] / pc[2], (Kn[2] - uu) / pc[2]};
                double dv[3] = {Kn[3] / pc[2], Kn[4] / pc[2], (Kn[5] - vv) / pc[2]};
                /* magnitudes for the bound: K_02 - u cancels near the principal
                 * point, so its rounding scales with |K_02| + |u| */
                double adu[3] = {fabs(du[0]), fabs(du[1]), (fabs(Kn[2]) + fabs(uu)) / fabs(pc[2])};
                double adv[3] = {fabs(dv[0]), fabs(dv[1]), (fabs(Kn[5]) + fabs(vv)) / fabs(pc[2])};
                for (int d = 0; d < 3; ++d) {
                    double val = 0.0, vb = 0.0;
                    for (int r = 0; r < 3; ++r) {
                        double R = En[4 * r + d];
                        val += R * (gx * sW * du[r] + gy * sH * dv[r]);
                        vb += fabs(R) * (gxb * sW * adu[r] + gyb * sH * adv[r]);
                    }
                    dO[k * 3 + d] += w * val;
                    dOb[k * 3 + d] += fabs(w) * vb;
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------
 * Lift-splat BEV pooling (LSS tutorial, "Lift" and "Splat" sections): every
 * feature pixel (h, w) of camera n spreads D depth bins along its ray; the
 * point of bin k carries depth[b,n,k,h,w] * feat[b,n,:,h,w] (the outer
 * product of the depth distribution and the context vector), is placed in
 * the ego frame with the camera's calibration, and is summed into the BEV
 * pillar (i, j) it falls in; z is not binned (one pillar per cell), and
 * points outside [xmin,xmax) x [ymin,ymax) x [zmin,zmax) are dropped:
 *
 *   out[b, c, i, j] = sum over (n, k, h, w) with cell (i, j) of depth[b,n,k,h,w] feat[b,n,c,h,w]
 *
 * Readings: the pixel of feature texel (h, w) is its centre in image pixels,
 * u = (w + 0.5) W_img / Wf, v = (h + 0.5) H_img / Hf (the inverse of the
 * sampling convention above); bin k sits at depth dmin + k * dstep (the bin's
 * lower edge, as the tutorial lists depths 4, 5, ..., 44 for [4, 45) at 1 m);
 * the camera point is depth * K^-1 [u v 1]^T with K upper triangular; E maps
 * ego to camera with a rotation R, so ego = R^T (pc - t).  The fp32 order:
 *   yn = (v - cy) / fy;  xn = ((u - cx) - s * yn) / fx;  pc = (xn d, yn d, d)
 *   q = pc - t;  x = (R00 q0 + R10 q1) + R20 q2  (likewise y, z)
 *   i = floor((x - xmin) / dx), j = floor((y - ymin) / dy)
 * ---------------------------------------------------------------------- */

/* Cell of one frustum point, or -1 when it falls outside the grid. */
int oracle_lss_cell(const float* K, const float* E, int h, int w, int k, int img_h, int img_w, int Hf, int Wf,
                    float dmin, float dstep, int X, int Y, const float lo[3], float zmax, const float cell[2],
                    float p_out[3])
{
    float sWi = (float)img_w / (float)Wf, sHi = (float)img_h / (float)Hf;
    float u = ((float)w + 0.5f) * sWi;
    float v = ((float)h + 0.5f) * sHi;
    float d = (float)k * dstep;
    d = dmin + d;
    float yn = (v - K[5]) / K[4];
    float t = K[1] * yn;
    float xn = ((u - K[2]) - t) / K[0];
    float pc[3] = {xn * d, yn * d, d};
    float q[3];
    for (int r = 0; r < 3; ++r) q[r] = pc[r] - E[4 * r + 3];
    float p[3];
    for (int a = 0; a < 3; ++a) {
        float s0 = E[a] * q[0];
        float s1 = E[4 + a] * q[1];
        float s2 = E[8 + a] * q[2];
        float acc = s0 + s1;
        p[a] = acc + s2;
    }
    if (p_out) { p_out[0] = p[0]; p_out[1] = p[1]; p_out[2] = p[2]; }
    if (!(p[2] >= lo[2] && p[2] < zmax)) return -1;
    float fi = floorf((p[0] - lo[0]) / cell[0]);
    float fj = floorf((p[1] - lo[1]) / cell[1]);
    if (!(fi >= 0.0f && fi < (float)X && fj >= 0.0f && fj < (float)Y)) return -1;
    return (int)fi * Y + (int)fj;
}

/* Forward.  depth [B,N,D,Hf,Wf], feat [B,N,C,Hf,Wf] fp64 (exact copies of the
 * inputs); K [B,N,3,3], E [B,N,4,4]; grid lo = (xmin, ymin, zmin), zmax,
 * cell = (dx, dy).  Writes out and bound [B,C,X,Y] fp64 and count [B,X,Y]
 * (points per pillar). */
void oracle_lss_forward(const double* depth, const double* feat, int B, int N, int D, int C, int Hf, int Wf,
                        const float* K, const float* E, int img_h, int img_w, float dmin, float dstep,
                        int X, int Y, const float lo[3], float zmax, const float cell[2],
                        double* out, double* bound, int32_t* count)
{
    memset(out, 0, sizeof(double) * (size_t)B * C * X * Y);
    memset(bound, 0, sizeof(double) * (size_t)B * C * X * Y);
    memset(count, 0, sizeof(int32_t) * (size_t)B * X * Y);
    for (int b = 0; b < B; ++b)
        for (int n = 0; n < N; ++n) {
            const float* Kn = K + ((size_t)b * N + n) * 9;
            const float* En = E + ((size_t)b * N + n) * 16;
            for (int h = 0; h < Hf; ++h)
                for (int w = 0; w < Wf; ++w)
                    for (int k = 0; k < D; ++k) {
                        int cl = oracle_lss_cell(Kn, En, h, w, k, img_h, img_w, Hf, Wf, dmin, dstep, X, Y, lo, zmax,
                                                 cell, NULL);
                        if (cl < 0) continue;
                        ++count[(size_t)b * X * Y + cl];
                        double a = depth[((((size_t)b * N + n) * D + k) * Hf + h) * Wf + w];
                        for (int c = 0; c < C; ++c) {
                            double term = a * feat[((((size_t)b * N + n) * C + c) * Hf + h) * Wf + w];
                            size_t o = ((size_t)b * C + c) * X * Y + cl;
                            out[o] += term;
                            bound[o] += fabs(term);
                        }
                    }
        }
}

/* Backward for dout [B,C,X,Y] fp64: ddepth [B,N,D,Hf,Wf] = sum_c dout[cell] feat,
 * dfeat [B,N,C,Hf,Wf] = sum_k depth dout[cell_k]; bounds of the same shapes. */
void oracle_lss_backward(const double* depth, const double* feat, const double* dout, int B, int N, int D, int C,
                         int Hf, int Wf, const float* K, const float* E, int img_h, int img_w, float dmin,
                         float dstep, int X, int Y, const float lo[3], float zmax, const float cell[2],
                         double* ddepth, double* ddb, double* dfeat, double* dfb)
{
    memset(ddepth, 0, sizeof(double) * (size_t)B * N * D * Hf * Wf);
    memset(ddb, 0, sizeof(double) * (size_t)B * N * D * Hf * Wf);
    memset(dfeat, 0, sizeof(double) * (size_t)B * N * C * Hf * Wf);
    memset(dfb, 0, sizeof(double) * (size_t)B * N * C * Hf * Wf);
    for (int b = 0; b < B; ++b)
        for (int n = 0; n < N; ++n) {
            const float* Kn = K + ((size_t)b * N + n) * 9;
            const float* En = E + ((size_t)b * N + n) * 16;
            for (int h = 0; h < Hf; ++h)
                for (int w = 0; w < Wf; ++w)
                    for (int k = 0; k < D; ++k) {
                        int cl = oracle_lss_cell(Kn, En, h, w, k, img_h, img_w, Hf, Wf, dmin, dstep, X, Y, lo, zmax,
                                                 cell, NULL);
                        if (cl < 0) continue;
                        size_t di = ((((size_t)b * N + n) * D + k) * Hf + h) * Wf + w;
                        double a = depth[di];
                        for (int c = 0; c < C; ++c) {
                            size_t fi = ((((size_t)b * N + n) * C + c) * Hf + h) * Wf + w;
                            double g = dout[((size_t)b * C + c) * X * Y + cl];
                            ddepth[di] += g * feat[fi];
                            ddb[di] += fabs(g * feat[fi]);
                            dfeat[fi] += a * g;
                            dfb[fi] += fabs(a * g);
                        }
                    }
        }
}
