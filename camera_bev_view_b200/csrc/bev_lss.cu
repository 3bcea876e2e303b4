// bev_lss.cu -- lift-splat BEV pooling, forward and backward (sm_100a).
//
// LSS tutorial, "Lift" and "Splat": every feature pixel (h, w) of camera n
// spreads D depth bins along its ray; the point of bin k carries
// depth[b,n,k,h,w] * feat[b,n,:,h,w] (the outer product), is placed in the
// ego frame and summed into the BEV pillar it falls in:
//   out[b, c, i, j] = sum over (n, k, h, w) in pillar (i, j) of depth * feat[c]
// The tutorial makes the variable-length sum per pillar deterministic by
// sorting the points by pillar and differencing a prefix sum.  Here every
// term is instead converted to a 64-bit fixed-point integer (2^-s units, s
// chosen per call from max|depth| max|feat| and the number of points per
// batch item, so no pillar sum can overflow) and added with integer
// reductions in L2: integer addition is exact and associative, so the sums
// do not depend on the order in which the points arrive, and one pass over
// the points suffices.  Consecutive rows of one image column whose bins of
// one depth land in the same pillar are merged in registers first.  A final
// transpose converts the channels-last integer sums to the fp32 [B,C,X,Y]
// output.
//
// Backward (a gather, deterministic): dout is made channels-last; each
// pixel's bins read the dout vector of their pillar:
//   ddepth[b,n,k,h,w] = dout[pillar] . feat[b,n,:,h,w]
//   dfeat[b,n,c,h,w]  = sum_k depth[b,n,k,h,w] dout[pillar_k, c]
// Four warps per pixel split its bins; their dfeat partials are added in warp
// order.
//
// The frustum geometry follows one fixed fp32 order (separate roundings, IEEE
// divides), the same as the oracle's, so pillar assignments are reproducible
// bit for bit:
//   u = (w + 0.5) (W_img / Wf);  v = (h + 0.5) (H_img / Hf);  d = dmin + k dstep
//   yn = (v - cy) / fy;  xn = ((u - cx) - s yn) / fx;  pc = (xn d, yn d, d)
//   q = pc - t;  x = (R00 q0 + R10 q1) + R20 q2 (likewise y, z)
//   i = floor((x - xmin) / dx), j = floor((y - ymin) / dy), zmin <= z < zmax
#include <stdint.h>

#include "bev_lss.cuh"

namespace bev {

namespace {

// Ray of feature pixel (h, w) through one camera: (xn, yn) with the camera
// point of depth d at (xn d, yn d, d).
struct Ray {
    float xn, yn;
};

__device__ __forceinline__ Ray lss_ray(const LssArgs& a, const float* K, int h, int w) {
    const float u = __fmul_rn(__fadd_rn((float)w, 0.5f), a.sWi);
    const float v = __fmul_rn(__fadd_rn((float)h, 0.5f), a.sHi);
    Ray r;
    r.yn = __fdiv_rn(__fsub_rn(v, K[5]), K[4]);
    const float t = __fmul_rn(K[1], r.yn);
    r.xn = __fdiv_rn(__fsub_rn(__fsub_rn(u, K[2]), t), K[0]);
    return r;
}

// Pillar (i * Y + j) of bin k of a pixel's ray, or -1.
__device__ __forceinline__ int lss_cell(const LssArgs& a, const Ray& ray, const float* E, int k) {
    const float d = __fadd_rn(a.dmin, __fmul_rn((float)k, a.dstep));
    const float xn = ray.xn, yn = ray.yn;
    const float pc[3] = {__fmul_rn(xn, d), __fmul_rn(yn, d), d};
    float q[3];
#pragma unroll
    for (int r = 0; r < 3; ++r) q[r] = __fsub_rn(pc[r], E[4 * r + 3]);
    float p[3];
#pragma unroll
    for (int c = 0; c < 3; ++c)
        p[c] = __fadd_rn(__fadd_rn(__fmul_rn(E[c], q[0]), __fmul_rn(E[4 + c], q[1])), __fmul_rn(E[8 + c], q[2]));
    if (!(p[2] >= a.zmin && p[2] < a.zmax)) return -1;
    const float fi = floorf(__fdiv_rn(__fsub_rn(p[0], a.xmin), a.dx));
    const float fj = floorf(__fdiv_rn(__fsub_rn(p[1], a.ymin), a.dy));
    if (!(fi >= 0.0f && fi < (float)a.X && fj >= 0.0f && fj < (float)a.Y)) return -1;
    return (int)fi * a.Y + (int)fj;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Fraction bits s of the fixed point: |sum| <= points * max|depth| max|feat|
// must stay below 2^62.  Clamped to [-126, 127] so that 2^s is an fp32
// number (a smaller s only costs resolution).
__device__ __forceinline__ int lss_frac_bits(const LssArgs& a) {
    const float m = __fmul_rn(__uint_as_float(a.maxabs[0]), __uint_as_float(a.maxabs[1]));
    if (!(m > 0.0f)) return 0;
    int e_m, e_p;
    frexpf(m, &e_m);                       // m < 2^e_m
    frexp((double)a.points_per_batch, &e_p);  // points < 2^e_p
    return max(-126, min(127, 62 - e_m - e_p));
}

// 2^s as fp32, s in [-126, 127], built from its exponent bits (exact).
__device__ __forceinline__ float pow2f(int s) { return __int_as_float((s + 127) << 23); }

}  // namespace

// max |depth| and max |feat| (non-negative floats compare like their bits)
__global__ void __launch_bounds__(256) lss_maxabs_kernel(const float* __restrict__ depth, size_t nd,
                                                         const float* __restrict__ feat, size_t nf,
                                                         unsigned* __restrict__ maxabs) {
    unsigned md = 0, mf = 0;
    const size_t tid = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    auto absmax = [&](const float* p, size_t n) -> unsigned {
        unsigned m = 0;
        // 16-byte loads, four in flight per thread, when the array allows
        if (((uintptr_t)p & 15) == 0) {
            const float4* p4 = reinterpret_cast<const float4*>(p);
            const size_t n4 = n / 4;
            size_t i = tid;
            for (; i + 3 * stride < n4; i += 4 * stride) {
                float4 v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) v[u] = __ldg(p4 + i + u * stride);
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    m = max(m, max(max(__float_as_uint(fabsf(v[u].x)), __float_as_uint(fabsf(v[u].y))),
                                   max(__float_as_uint(fabsf(v[u].z)), __float_as_uint(fabsf(v[u].w)))));
            }
            for (; i < n4; i += stride) {
                const float4 v = __ldg(p4 + i);
                m = max(m, max(max(__float_as_uint(fabsf(v.x)), __float_as_uint(fabsf(v.y))),
                               max(__float_as_uint(fabsf(v.z)), __float_as_uint(fabsf(v.w)))));
            }
            for (size_t j = 4 * n4 + tid; j < n; j += stride) m = max(m, __float_as_uint(fabsf(p[j])));
        } else {
            for (size_t j = tid; j < n; j += stride) m = max(m, __float_as_uint(fabsf(p[j])));
        }
        return m;
    };
    md = absmax(depth, nd);
    mf = absmax(feat, nf);
    md = __reduce_max_sync(0xffffffffu, md);
    mf = __reduce_max_sync(0xffffffffu, mf);
    // one pair of atomics per CTA: the global maxima live at two addresses,
    // so per-warp atomics would queue up behind each other in L2
    __shared__ unsigned sd[8], sf[8];
    if ((threadIdx.x & 31) == 0) {
        sd[threadIdx.x >> 5] = md;
        sf[threadIdx.x >> 5] = mf;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        md = threadIdx.x < 8 ? sd[threadIdx.x] : 0u;
        mf = threadIdx.x < 8 ? sf[threadIdx.x] : 0u;
        md = __reduce_max_sync(0xffffffffu, md);
        mf = __reduce_max_sync(0xffffffffu, mf);
        if (threadIdx.x == 0) {
            atomicMax(maxabs, md);
            atomicMax(maxabs + 1, mf);
        }
    }
}

// Forward over a block of the feature map: rows h0 .. h0 + kLssRows and
// columns w0 .. w0 + kLssCols of one camera (b, n), depth bins k0 .. k0 +
// a.bins_per_cta (at most kLssBins; fewer when the launch would otherwise
// give under two CTAs per SM).  The CTA stages the block's rays, depths and pillars, then the
// features channels-last in chunks of kLssChunk channels (global loads run
// along w, the contiguous axis).  A warp then takes one (column, bin) at a
// time and walks its rows.  For a camera without pitch or roll the image row
// moves a point only in ego height, so the bins of one depth along one image
// column share their pillar (LSS tutorial, "Splat": pillars bin the ground
// plane only); consecutive rows with one pillar are summed in registers and
// sent as one 64-bit reduction per channel, and rows of other pillars (a
// tilted camera) start new runs.  Each term is converted to fixed point on its own, so the integer
// sums, and the output, do not depend on how the terms are grouped.
constexpr int kLssCols = 8, kLssRows = 16, kLssBins = 8, kLssChunk = 64;
constexpr int kLssPix = kLssCols * kLssRows;
constexpr int kLssThreads = 256;

__global__ void __launch_bounds__(kLssThreads) lss_forward_kernel(const LssArgs a) {
    __shared__ float fs[kLssPix * (kLssChunk + 1)];  // [pixel][channel of the chunk]; pixel = r * kLssCols + x
    __shared__ float ds[kLssBins * kLssPix];         // [bin][pixel]: depth probability
    __shared__ int ps[kLssBins * kLssPix];           // [bin][pixel]: pillar, or -1
    __shared__ float rx[kLssPix], ry[kLssPix];       // the pixels' rays
    const int nwb = (a.Wf + kLssCols - 1) / kLssCols;
    const int w0 = (int)(blockIdx.x % nwb) * kLssCols, h0 = (int)(blockIdx.x / nwb) * kLssRows;
    const int k0 = blockIdx.y * a.bins_per_cta, kn = min(a.bins_per_cta, a.D - k0);
    const long long bn = blockIdx.z;
    const int b = (int)(bn / a.N);
    const float* K = a.K + bn * 9;
    const float* E = a.E + bn * 16;
    const size_t hw = (size_t)a.Hf * a.Wf;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid < kLssPix) {
        const int h = h0 + tid / kLssCols, w = w0 + tid % kLssCols;
        Ray ray = {0.0f, 0.0f};
        if (h < a.Hf && w < a.Wf) ray = lss_ray(a, K, h, w);
        rx[tid] = ray.xn;
        ry[tid] = ray.yn;
    }
    __syncthreads();
    for (int t = tid; t < kLssBins * kLssPix; t += kLssThreads) {
        const int kk = t / kLssPix, pix = t % kLssPix;
        const int h = h0 + pix / kLssCols, w = w0 + pix % kLssCols;
        int cell = -1;
        float al = 0.0f;
        if (kk < kn && h < a.Hf && w < a.Wf) {
            const Ray ray = {rx[pix], ry[pix]};
            cell = lss_cell(a, ray, E, k0 + kk);
            al = a.depth[((size_t)bn * a.D + k0 + kk) * hw + (size_t)h * a.Wf + w];
        }
        ps[t] = cell;
        ds[t] = al;
    }
    const float scale = pow2f(lss_frac_bits(a));
    unsigned long long* acc = a.acc + (size_t)b * a.X * a.Y * a.C;
    for (int c0 = 0; c0 < a.C; c0 += kLssChunk) {
        __syncthreads();  // pillars staged; the previous chunk's reads done
        for (int t = tid; t < kLssChunk * kLssPix; t += kLssThreads) {
            const int cl = t / kLssPix, pix = t % kLssPix;
            const int h = h0 + pix / kLssCols, w = w0 + pix % kLssCols, c = c0 + cl;
            fs[pix * (kLssChunk + 1) + cl] =
                (c < a.C && h < a.Hf && w < a.Wf) ? a.feat[((size_t)bn * a.C + c) * hw + (size_t)h * a.Wf + w] : 0.0f;
        }
        __syncthreads();
        bool on[2];
#pragma unroll
        for (int v = 0; v < 2; ++v) on[v] = c0 + lane + 32 * v < a.C;
        for (int it = warp; it < kLssCols * kn; it += kLssThreads / 32) {
            const int x = it % kLssCols, kk = it / kLssCols;
            long long run[2] = {0, 0};
            int run_cell = -1;
            for (int r = 0; r < kLssRows; ++r) {
                const int pix = r * kLssCols + x;
                const int ck = ps[kk * kLssPix + pix];
                if (ck < 0) continue;
                if (ck != run_cell) {
                    if (run_cell >= 0) {
#pragma unroll
                        for (int v = 0; v < 2; ++v)
                            if (on[v]) atomicAdd(acc + (size_t)run_cell * a.C + c0 + lane + 32 * v, (unsigned long long)run[v]);
                    }
                    run_cell = ck;
                    run[0] = run[1] = 0;
                }
                const float ak = ds[kk * kLssPix + pix];
#pragma unroll
                for (int v = 0; v < 2; ++v)
                    run[v] += __float2ll_rn(__fmul_rn(__fmul_rn(ak, fs[pix * (kLssChunk + 1) + lane + 32 * v]), scale));
            }
            if (run_cell >= 0) {
#pragma unroll
                for (int v = 0; v < 2; ++v)
                    if (on[v]) atomicAdd(acc + (size_t)run_cell * a.C + c0 + lane + 32 * v, (unsigned long long)run[v]);
            }
        }
    }
}

// Fixed-point channels-last sums [B][X*Y][C] -> fp32 out [B][C][X*Y], 32x32
// tiles through shared memory.  Each sum is widened to double and scaled by
// 2^-s (an exact multiply by a power of two), then rounded to fp32.  A thread
// issues its four loads before converting any of them.
__global__ void __launch_bounds__(256) lss_convert_kernel(const LssArgs a) {
    __shared__ float tile[32][33];
    const int b = blockIdx.z;
    const int p0 = blockIdx.x * 32, c0 = blockIdx.y * 32;
    const int XY = a.X * a.Y;
    const double inv = __longlong_as_double((long long)(1023 - lss_frac_bits(a)) << 52);  // 2^-s
    const unsigned long long* acc = a.acc + (size_t)b * XY * a.C;
    long long v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int p = p0 + threadIdx.y + 8 * q, c = c0 + threadIdx.x;
        v[q] = (p < XY && c < a.C) ? (long long)__ldg(acc + (size_t)p * a.C + c) : 0;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) tile[threadIdx.y + 8 * q][threadIdx.x] = __double2float_rn(__ll2double_rn(v[q]) * inv);
    __syncthreads();
    for (int r = threadIdx.y; r < 32; r += 8) {
        const int c = c0 + r, p = p0 + threadIdx.x;
        if (c < a.C && p < XY) a.out[((size_t)b * a.C + c) * XY + p] = tile[threadIdx.x][r];
    }
}

// Backward: one CTA of kLssWarps warps per pixel; warp w takes bins
// k = w, w + kLssWarps, ...; dout is channels-last [B][X*Y][C].
template <int V>
__global__ void __launch_bounds__(kLssWarps * 32) lss_backward_kernel(const LssArgs a) {
    __shared__ float part[kLssWarps][kLssMaxChannels];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long pix = blockIdx.x;
    const int w = (int)(pix % a.Wf);
    const int h = (int)((pix / a.Wf) % a.Hf);
    const long long bn = pix / ((long long)a.Hf * a.Wf);
    const int b = (int)(bn / a.N);
    const float* K = a.K + bn * 9;
    const float* E = a.E + bn * 16;
    const size_t hw = (size_t)a.Hf * a.Wf;
    const size_t poff = (size_t)h * a.Wf + w;
    const float* G = a.dout_cl + (size_t)b * a.X * a.Y * a.C;
    const Ray ray = lss_ray(a, K, h, w);
    float f[V], df[V];
#pragma unroll
    for (int v = 0; v < V; ++v) {
        const int c = lane + 32 * v;
        f[v] = c < a.C ? a.feat[((size_t)bn * a.C + c) * hw + poff] : 0.0f;
        df[v] = 0.0f;
    }
    for (int k0 = warp; k0 < a.D; k0 += 32 * kLssWarps) {
        const int k = k0 + kLssWarps * lane;
        int cell = -1;
        float al = 0.0f;
        if (k < a.D) {
            cell = lss_cell(a, ray, E, k);
            al = a.depth[((size_t)bn * a.D + k) * hw + poff];
        }
        float dd = 0.0f;  // this lane's bin's ddepth
        const int kn = min(32, (a.D - k0 + kLssWarps - 1) / kLssWarps);
        // four bins per step: their dout vectors are loaded before any is used
        for (int kb = 0; kb < kn; kb += 4) {
            int ck[4];
            float ak[4], g[4][V];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int kk = kb + u;
                ck[u] = __shfl_sync(0xffffffffu, cell, kk & 31);
                ak[u] = __shfl_sync(0xffffffffu, al, kk & 31);
                if (kk >= kn) ck[u] = -1;
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    const int c = lane + 32 * v;
                    g[u][v] = (ck[u] >= 0 && c < a.C) ? G[(size_t)ck[u] * a.C + c] : 0.0f;
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (ck[u] < 0) continue;
                float dot = 0.0f;
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    dot = __fmaf_rn(g[u][v], f[v], dot);
                    df[v] = __fmaf_rn(ak[u], g[u][v], df[v]);
                }
                dot = warp_sum(dot);
                if (lane == kb + u) dd = dot;
            }
        }
        if (k < a.D) a.ddepth[((size_t)bn * a.D + k) * hw + poff] = dd;
    }
#pragma unroll
    for (int v = 0; v < V; ++v)
        if (lane + 32 * v < a.C) part[warp][lane + 32 * v] = df[v];
    __syncthreads();
    for (int c = threadIdx.x; c < a.C; c += kLssWarps * 32) {
        float s = part[0][c];
#pragma unroll
        for (int ww = 1; ww < kLssWarps; ++ww) s = __fadd_rn(s, part[ww][c]);
        a.dfeat[((size_t)bn * a.C + c) * hw + poff] = s;
    }
}

// Backward over a block of the feature map: rows h0 .. h0 + kLssRows and
// columns w0 .. w0 + kLssBwdCols of one camera.  Warp w takes column
// w % kLssBwdCols and the bins k of parity w / kLssBwdCols; it holds its
// column's features (one 64-channel chunk at a time, staged channels-last
// with loads along w) and the feature-gradient partials of its rows in
// registers.  Walking the rows of one bin, it reads a pillar's dout vector
// once per run of rows that share the pillar (a camera without pitch or roll
// puts the whole column in one pillar, as in the forward), where the
// per-pixel kernel reads it once per pixel.  The two parities' partials are
// added in a fixed order, and a later channel chunk adds its dot products to
// the depth gradient after the earlier ones, so the result is deterministic.
constexpr int kLssBwdCols = 4, kLssBwdPar = 2;
constexpr int kLssBwdPix = kLssBwdCols * kLssRows;
constexpr int kLssBwdThreads = 32 * kLssBwdCols * kLssBwdPar;

__global__ void __launch_bounds__(kLssBwdThreads) lss_backward_cols_kernel(const LssArgs a) {
    __shared__ float fs[kLssBwdPix * (kLssChunk + 1)];   // [pixel][channel of the chunk]; pixel = r * kLssBwdCols + x
    __shared__ float dfs[kLssBwdPix * (kLssChunk + 1)];  // the odd-bin warps' feature-gradient partials
    __shared__ float rx[kLssBwdPix], ry[kLssBwdPix];
    const int nwb = (a.Wf + kLssBwdCols - 1) / kLssBwdCols;
    const int w0 = (int)(blockIdx.x % nwb) * kLssBwdCols, h0 = (int)(blockIdx.x / nwb) * kLssRows;
    const long long bn = blockIdx.y;
    const int b = (int)(bn / a.N);
    const float* K = a.K + bn * 9;
    const float* E = a.E + bn * 16;
    const size_t hw = (size_t)a.Hf * a.Wf;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int x = warp % kLssBwdCols, kp = warp / kLssBwdCols, w = w0 + x;
    const float* G = a.dout_cl + (size_t)b * a.X * a.Y * a.C;
    if (tid < kLssBwdPix) {
        const int h = h0 + tid / kLssBwdCols, ww = w0 + tid % kLssBwdCols;
        Ray ray = {0.0f, 0.0f};
        if (h < a.Hf && ww < a.Wf) ray = lss_ray(a, K, h, ww);
        rx[tid] = ray.xn;
        ry[tid] = ray.yn;
    }
    for (int c0 = 0; c0 < a.C; c0 += kLssChunk) {
        __syncthreads();  // rays staged; the previous chunk's shared reads done
        for (int t = tid; t < kLssChunk * kLssBwdPix; t += kLssBwdThreads) {
            const int cl = t / kLssBwdPix, pix = t % kLssBwdPix;
            const int h = h0 + pix / kLssBwdCols, ww = w0 + pix % kLssBwdCols, c = c0 + cl;
            fs[pix * (kLssChunk + 1) + cl] =
                (c < a.C && h < a.Hf && ww < a.Wf) ? a.feat[((size_t)bn * a.C + c) * hw + (size_t)h * a.Wf + ww] : 0.0f;
        }
        __syncthreads();
        const bool on0 = c0 + lane < a.C, on1 = c0 + lane + 32 < a.C;
        float f[kLssRows][2], df[kLssRows][2];
#pragma unroll
        for (int r = 0; r < kLssRows; ++r) {
            const float* fp = fs + (r * kLssBwdCols + x) * (kLssChunk + 1) + lane;
            f[r][0] = fp[0];
            f[r][1] = fp[32];
            df[r][0] = df[r][1] = 0.0f;
        }
        const int h = h0 + lane;
        const bool row_ok = lane < kLssRows && h < a.Hf && w < a.Wf;
        const Ray ray = {row_ok ? rx[lane * kLssBwdCols + x] : 0.0f, row_ok ? ry[lane * kLssBwdCols + x] : 0.0f};
        // this lane's row: pillar and depth of the warp's next bin, fetched one
        // bin ahead so that their latency overlaps the current bin's rows
        int cell_n = -1;
        float al_n = 0.0f;
        if (row_ok && kp < a.D) {
            cell_n = lss_cell(a, ray, E, kp);
            al_n = a.depth[((size_t)bn * a.D + kp) * hw + (size_t)h * a.Wf + w];
        }
        for (int k = kp; k < a.D; k += kLssBwdPar) {
            const int cell = cell_n;
            const float al = al_n;
            cell_n = -1;
            al_n = 0.0f;
            if (row_ok && k + kLssBwdPar < a.D) {
                cell_n = lss_cell(a, ray, E, k + kLssBwdPar);
                al_n = a.depth[((size_t)bn * a.D + k + kLssBwdPar) * hw + (size_t)h * a.Wf + w];
            }
            // per lane: its two channels' share of each row's dot product
            float q[kLssRows];
            float g0 = 0.0f, g1 = 0.0f;
            int cur = -1;
#pragma unroll
            for (int r = 0; r < kLssRows; ++r) {
                const int ck = __shfl_sync(0xffffffffu, cell, r);
                const float ak = __shfl_sync(0xffffffffu, al, r);
                q[r] = 0.0f;
                if (ck < 0) continue;
                if (ck != cur) {
                    cur = ck;
                    g0 = on0 ? G[(size_t)ck * a.C + c0 + lane] : 0.0f;
                    g1 = on1 ? G[(size_t)ck * a.C + c0 + lane + 32] : 0.0f;
                }
                q[r] = __fmaf_rn(g1, f[r][1], __fmul_rn(g0, f[r][0]));
                df[r][0] = __fmaf_rn(ak, g0, df[r][0]);
                df[r][1] = __fmaf_rn(ak, g1, df[r][1]);
            }
            // reduce the 16 rows over the 32 lanes at once (recursive halving:
            // at each step a lane keeps half of its rows and adds its partner's
            // share of them); lanes 2r and 2r + 1 end with row r's total
#pragma unroll
            for (int half = kLssRows / 2, o = 16; half >= 1; half >>= 1, o >>= 1) {
                const bool up = (lane & o) != 0;
#pragma unroll
                for (int i = 0; i < half; ++i) {
                    const float send = up ? q[i] : q[i + half];
                    const float keep = up ? q[i + half] : q[i];
                    q[i] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, o));
                }
            }
            const float dd = __fadd_rn(q[0], __shfl_xor_sync(0xffffffffu, q[0], 1));
            const int hr = h0 + (lane >> 1);
            if ((lane & 1) == 0 && hr < a.Hf && w < a.Wf) {
                float* p = a.ddepth + ((size_t)bn * a.D + k) * hw + (size_t)hr * a.Wf + w;
                *p = c0 == 0 ? dd : __fadd_rn(*p, dd);
            }
        }
        if (kp == 1) {
#pragma unroll
            for (int r = 0; r < kLssRows; ++r) {
                float* dp = dfs + (r * kLssBwdCols + x) * (kLssChunk + 1) + lane;
                dp[0] = df[r][0];
                dp[32] = df[r][1];
            }
        }
        __syncthreads();
        if (kp == 0 && w < a.Wf) {
#pragma unroll
            for (int r = 0; r < kLssRows; ++r) {
                if (h0 + r >= a.Hf) break;
                const float* dp = dfs + (r * kLssBwdCols + x) * (kLssChunk + 1) + lane;
                float* out = a.dfeat + ((size_t)bn * a.C + c0 + lane) * hw + (size_t)(h0 + r) * a.Wf + w;
                if (on0) out[0] = __fadd_rn(df[r][0], dp[0]);
                if (on1) out[32 * hw] = __fadd_rn(df[r][1], dp[32]);
            }
        }
    }
}

}  // namespace bev

cudaError_t bev_launch_lss_forward(const bev::LssArgs& a, cudaStream_t st) {
    using namespace bev;
    const size_t nd = (size_t)a.B * a.N * a.D * a.Hf * a.Wf, nf = (size_t)a.B * a.N * a.C * a.Hf * a.Wf;
    const size_t mx = (nd > nf ? nd : nf);
    const int mblocks = (int)((mx / 4 + 255) / 256 < 148 * 4 ? (mx / 4 + 255) / 256 + 1 : 148 * 4);
    lss_maxabs_kernel<<<mblocks, 256, 0, st>>>(a.depth, nd, a.feat, nf, a.maxabs);
    const long long nblk = (long long)((a.Hf + kLssRows - 1) / kLssRows) * ((a.Wf + kLssCols - 1) / kLssCols);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    LssArgs f = a;
    f.bins_per_cta = kLssBins;
    while (f.bins_per_cta > 1 && nblk * a.B * a.N * ((a.D + f.bins_per_cta - 1) / f.bins_per_cta) < 2LL * sms)
        f.bins_per_cta >>= 1;
    const dim3 fgrid((unsigned)nblk, (unsigned)((a.D + f.bins_per_cta - 1) / f.bins_per_cta), (unsigned)(a.B * a.N));
    lss_forward_kernel<<<fgrid, kLssThreads, 0, st>>>(f);
    const int XY = a.X * a.Y;
    const dim3 grid((XY + 31) / 32, (a.C + 31) / 32, a.B);
    lss_convert_kernel<<<grid, dim3(32, 8), 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t bev_launch_lss_backward(const bev::LssArgs& a, cudaStream_t st) {
    using namespace bev;
    // Column blocks when they give at least one CTA per SM; one CTA per pixel
    // otherwise (small maps, where the blocks would leave SMs idle).
    const long long nblk = (long long)((a.Hf + kLssRows - 1) / kLssRows) * ((a.Wf + kLssBwdCols - 1) / kLssBwdCols);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (nblk * a.B * a.N >= sms) {
        lss_backward_cols_kernel<<<dim3((unsigned)nblk, (unsigned)(a.B * a.N)), kLssBwdThreads, 0, st>>>(a);
        return cudaGetLastError();
    }
    const long long npix = (long long)a.B * a.N * a.Hf * a.Wf;
    const int V = (a.C + 31) / 32;
    const dim3 grid((unsigned)npix);
    switch (V) {
        case 1: lss_backward_kernel<1><<<grid, kLssWarps * 32, 0, st>>>(a); break;
        case 2: lss_backward_kernel<2><<<grid, kLssWarps * 32, 0, st>>>(a); break;
        case 3: lss_backward_kernel<3><<<grid, kLssWarps * 32, 0, st>>>(a); break;
        case 4: lss_backward_kernel<4><<<grid, kLssWarps * 32, 0, st>>>(a); break;
        case 5: lss_backward_kernel<5><<<grid, kLssWarps * 32, 0, st>>>(a); break;
        case 6: lss_backward_kernel<6><<<grid, kLssWarps * 32, 0, st>>>(a); break;
        case 7: lss_backward_kernel<7><<<grid, kLssWarps * 32, 0, st>>>(a); break;
        case 8: lss_backward_kernel<8><<<grid, kLssWarps * 32, 0, st>>>(a); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}
