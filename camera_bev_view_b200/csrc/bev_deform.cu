// bev_deform.cu -- deformable aggregation, forward and backward (sm_100a).
//
// SparseDriveV2 notes, "Deformable Aggregation", steps 1-3: a query with
// anchor a and keypoint offsets d_k samples every camera n at the keypoints
// p_k = a + d_k, keeps the samples whose projection is valid (depth > 0.1 and
// inside the image), and sums the bilinear samples with weights w[n, k]:
//   out[b, q, c] = sum_n sum_k [valid] w[b, q, n, k] * bilinear(F[b, n, c], fx, fy)
// The geometry is the pinned fp32 projection of the dense path
// (bev_geometry.cuh), so validity and corners match the oracle bit for bit.
//
// One CTA per query; its kDeformWarps warps split the query's (camera,
// keypoint) pairs, warp w taking every kDeformWarps-th pair from w.  A warp's
// lanes first take one pair each -- keypoint, projection, weight -- 32 pairs
// per pass; the valid pairs of a pass are then visited in turn, each
// broadcast to the warp, whose lanes read the four bilinear corners of their
// channel chunks (16-byte loads from the channels-last features, V chunks
// per lane) and accumulate in fp32, up to two pairs in flight per step.  The
// warps' partial sums meet in shared memory and are added in warp order, so
// the result does not depend on timing.
//
// Backward, per valid pair: the lane-local dot products of the four corners
// with dout are reduced over the warp into the weight gradient (the sample
// itself) and the derivative of the sample in (fx, fy); the owning lane
// carries the latter through the projection to the keypoint offset,
//   d/dp = w R^T (g_x (Wf/W_img) du/dpc + g_y (Hf/H_img) dv/dpc),
//   du/dpc = (K00, K01, K02 - u) / depth, dv/dpc likewise,
// adding into a per-warp shared-memory accumulator in pair order; the warps'
// accumulators are added in warp order at the end (deterministic).  The feature gradient is reduced into an fp32
// channels-last buffer with 16-byte vector reductions.
#include "bev_deform.cuh"
#include "bev_kernels.cuh"

namespace bev {

namespace {

template <bool BF16>
struct DChunk;

template <>
struct DChunk<false> {
    static constexpr int kFloats = 4;
    __device__ __forceinline__ static void unpack(const uint4& d, float (&f)[4]) {
        f[0] = __uint_as_float(d.x);
        f[1] = __uint_as_float(d.y);
        f[2] = __uint_as_float(d.z);
        f[3] = __uint_as_float(d.w);
    }
};

template <>
struct DChunk<true> {
    static constexpr int kFloats = 8;
    // bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32 word.
    __device__ __forceinline__ static void unpack(const uint4& d, float (&f)[8]) {
        const unsigned w[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Calibration of batch item b into shared memory: E rows 0..2, K rows 0..1.
__device__ __forceinline__ void stage_cams(const DeformArgs& a, int b, float* cams) {
    for (int t = threadIdx.x; t < a.N * kCamFloats; t += blockDim.x) {
        const int n = t / kCamFloats, r = t - n * kCamFloats;
        cams[t] = r < 12 ? a.E[((size_t)b * a.N + n) * 16 + r] : a.K[((size_t)b * a.N + n) * 9 + (r - 12)];
    }
}

// One (camera, keypoint) pair of query (b, q), projected by the calling lane.
struct Pair {
    float fx, fy, w;
    int n, k;
    bool ok;
    ProjDetail det;
};

__device__ __forceinline__ Pair project_pair(const DeformArgs& a, const float* cams, int b, int q, int pr,
                                             float ax, float ay, float az) {
    Pair p;
    p.ok = false;
    p.fx = p.fy = p.w = 0.0f;
    p.n = p.k = 0;
    p.det.u = p.det.v = p.det.depth = 0.0f;
    if (pr < a.N * a.Kp) {
        p.n = pr / a.Kp;
        p.k = pr - p.n * a.Kp;
        const float* d = a.offsets + (((size_t)b * a.Q + q) * a.Kp + p.k) * 3;
        const float px = __fadd_rn(ax, d[0]), py = __fadd_rn(ay, d[1]), pz = __fadd_rn(az, d[2]);
        p.ok = project_point(cams + p.n * kCamFloats, px, py, pz, a.g, p.fx, p.fy, p.det);
        p.w = a.weights[((size_t)b * a.Q + q) * a.N * a.Kp + pr];
    }
    return p;
}

// Corner t (0: (y0, x0), 1: (y0, x0+1), 2: (y0+1, x0), 3: (y0+1, x0+1)) of a
// sample: texel offset within the camera's plane and whether it is inside.
__device__ __forceinline__ void corner_texels(const Corners& c, int Hf, int Wf, int (&tex)[4], bool (&in)[4]) {
    const bool cx0 = (unsigned)c.x0 < (unsigned)Wf, cx1 = (unsigned)(c.x0 + 1) < (unsigned)Wf;
    const bool cy0 = (unsigned)c.y0 < (unsigned)Hf, cy1 = (unsigned)(c.y0 + 1) < (unsigned)Hf;
    in[0] = cy0 && cx0;
    in[1] = cy0 && cx1;
    in[2] = cy1 && cx0;
    in[3] = cy1 && cx1;
    const int base = c.y0 * Wf + c.x0;
    tex[0] = base;
    tex[1] = base + 1;
    tex[2] = base + Wf;
    tex[3] = base + Wf + 1;
}

}  // namespace

template <bool BF16, int V>
__global__ void __launch_bounds__(kDeformWarps * 32) deform_forward_kernel(const DeformArgs a) {
    constexpr int NF = DChunk<BF16>::kFloats;
    extern __shared__ __align__(16) float dsmem[];
    float* cams = dsmem;
    const int q = blockIdx.x, b = blockIdx.y;
    stage_cams(a, b, cams);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const GeoParams& g = a.g;
    const float* A = a.anchors + ((size_t)b * a.Q + q) * 3;
    const float ax = A[0], ay = A[1], az = A[2];
    const size_t texels = (size_t)g.Hf * g.Wf;
    const uint4* featb = reinterpret_cast<const uint4*>(a.feat) + (size_t)b * a.N * texels * a.Qtot + lane;
    bool lane_ok[V];
#pragma unroll
    for (int v = 0; v < V; ++v) lane_ok[v] = lane + 32 * v < a.Qtot;

    float acc[V][NF];
#pragma unroll
    for (int v = 0; v < V; ++v)
#pragma unroll
        for (int e = 0; e < NF; ++e) acc[v][e] = 0.0f;

    // valid pairs per step, their loads issued together (as many as the
    // registers allow: 8 x 16-byte loads per lane in flight)
    constexpr int PP = V <= 2 ? 2 : 1;
    const int pairs = a.N * a.Kp;
    for (int p0 = warp; p0 < pairs; p0 += 32 * kDeformWarps) {
        const Pair my = project_pair(a, cams, b, q, p0 + kDeformWarps * lane, ax, ay, az);
        unsigned m = __ballot_sync(0xffffffffu, my.ok);
        while (m) {
            int src[PP];
#pragma unroll
            for (int s = 0; s < PP; ++s) {
                src[s] = m ? __ffs(m) - 1 : -1;
                if (m) m &= m - 1;
            }
            uint4 d[PP][4][V];
            float wt[PP][4];
#pragma unroll
            for (int s = 0; s < PP; ++s) {
                const int sl = src[s] < 0 ? src[0] : src[s];
                const float fx = __shfl_sync(0xffffffffu, my.fx, sl);
                const float fy = __shfl_sync(0xffffffffu, my.fy, sl);
                const float w = src[s] < 0 ? 0.0f : __shfl_sync(0xffffffffu, my.w, sl);
                const int n = __shfl_sync(0xffffffffu, my.n, sl);
                const Corners c = bilinear_corners(fx, fy);
                int tex[4];
                bool in[4];
                corner_texels(c, g.Hf, g.Wf, tex, in);
                const float cw[4] = {c.w00, c.w01, c.w10, c.w11};
                const uint4* Fn = featb + (size_t)n * texels * a.Qtot;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    wt[s][t] = in[t] ? __fmul_rn(w, cw[t]) : 0.0f;
#pragma unroll
                    for (int v = 0; v < V; ++v)
                        d[s][t][v] = (wt[s][t] != 0.0f && lane_ok[v]) ? __ldg(Fn + (size_t)tex[t] * a.Qtot + 32 * v)
                                                                     : make_uint4(0, 0, 0, 0);
                }
            }
#pragma unroll
            for (int s = 0; s < PP; ++s)
#pragma unroll
                for (int t = 0; t < 4; ++t)
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        float f[NF];
                        DChunk<BF16>::unpack(d[s][t][v], f);
#pragma unroll
                        for (int e = 0; e < NF; ++e) acc[v][e] = __fmaf_rn(wt[s][t], f[e], acc[v][e]);
                    }
        }
    }

    // the warps' partial sums, added in warp order
    const int cpad = (a.C > a.Kp * 3 ? a.C : a.Kp * 3) + 3 & ~3;
    float* part = dsmem + (a.N * kCamFloats + 3) / 4 * 4 + warp * cpad;
#pragma unroll
    for (int v = 0; v < V; ++v) {
        const int c0 = (lane + 32 * v) * NF;
        if (!lane_ok[v]) continue;
#pragma unroll
        for (int e = 0; e < NF; ++e)
            if (c0 + e < a.C) part[c0 + e] = acc[v][e];
    }
    __syncthreads();
    const float* part0 = dsmem + (a.N * kCamFloats + 3) / 4 * 4;
    float* o = a.out + ((size_t)b * a.Q + q) * a.C;
    for (int c = threadIdx.x; c < a.C; c += kDeformWarps * 32) {
        float s = part0[c];
#pragma unroll
        for (int ww = 1; ww < kDeformWarps; ++ww) s = __fadd_rn(s, part0[ww * cpad + c]);
        o[c] = s;
    }
}

template <bool BF16, int V>
__global__ void __launch_bounds__(kDeformWarps * 32) deform_backward_kernel(const DeformArgs a) {
    constexpr int NF = DChunk<BF16>::kFloats;
    extern __shared__ __align__(16) float dsmem[];
    float* cams = dsmem;
    const int q = blockIdx.x, b = blockIdx.y;
    stage_cams(a, b, cams);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cpad = (a.C > a.Kp * 3 ? a.C : a.Kp * 3) + 3 & ~3;
    float* doff0 = dsmem + (a.N * kCamFloats + 3) / 4 * 4;
    float* doff = doff0 + warp * cpad;
    for (int t = lane; t < a.Kp * 3; t += 32) doff[t] = 0.0f;
    __syncthreads();
    const GeoParams& g = a.g;
    const float* A = a.anchors + ((size_t)b * a.Q + q) * 3;
    const float ax = A[0], ay = A[1], az = A[2];
    const size_t texels = (size_t)g.Hf * g.Wf;
    const uint4* featb = reinterpret_cast<const uint4*>(a.feat) + (size_t)b * a.N * texels * a.Qtot + lane;
    const int tstride = a.Qtot * NF;  // floats per texel of the gradient buffer
    float* gradb = a.dfeat + (size_t)b * a.N * texels * tstride + (size_t)lane * NF;
    bool lane_ok[V];
    float dg[V][NF];
    const float* go = a.dout + ((size_t)b * a.Q + q) * a.C;
#pragma unroll
    for (int v = 0; v < V; ++v) {
        lane_ok[v] = lane + 32 * v < a.Qtot;
#pragma unroll
        for (int e = 0; e < NF; ++e) {
            const int c = (lane + 32 * v) * NF + e;
            dg[v][e] = (lane_ok[v] && c < a.C) ? go[c] : 0.0f;
        }
    }
    float* dW = a.dweights + ((size_t)b * a.Q + q) * a.N * a.Kp;

    const int pairs = a.N * a.Kp;
    for (int p0 = warp; p0 < pairs; p0 += 32 * kDeformWarps) {
        const int pr = p0 + kDeformWarps * lane;
        const Pair my = project_pair(a, cams, b, q, pr, ax, ay, az);
        if (pr < pairs && !my.ok) dW[pr] = 0.0f;  // no sample, no gradient
        unsigned m = __ballot_sync(0xffffffffu, my.ok);
        while (m) {
            const int src = __ffs(m) - 1;
            m &= m - 1;
            const float fx = __shfl_sync(0xffffffffu, my.fx, src);
            const float fy = __shfl_sync(0xffffffffu, my.fy, src);
            const float w = __shfl_sync(0xffffffffu, my.w, src);
            const int n = __shfl_sync(0xffffffffu, my.n, src);
            const Corners c = bilinear_corners(fx, fy);
            int tex[4];
            bool in[4];
            corner_texels(c, g.Hf, g.Wf, tex, in);
            const float cw[4] = {c.w00, c.w01, c.w10, c.w11};
            const uint4* Fn = featb + (size_t)n * texels * a.Qtot;
            float* Gn = gradb + (size_t)n * texels * tstride;
            // lane-local dot products of each corner with dout
            uint4 dv[4][V];
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int v = 0; v < V; ++v)
                    dv[t][v] = (in[t] && lane_ok[v]) ? __ldg(Fn + (size_t)tex[t] * a.Qtot + 32 * v) : make_uint4(0, 0, 0, 0);
            float dot[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                float s = 0.0f;
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    float f[NF];
                    DChunk<BF16>::unpack(dv[t][v], f);
#pragma unroll
                    for (int e = 0; e < NF; ++e) s = __fmaf_rn(f[e], dg[v][e], s);
                }
                dot[t] = s;
            }
            // feature gradient: w * corner weight * dout into each in-range corner
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float wt = __fmul_rn(w, cw[t]);
                if (!in[t] || wt == 0.0f) continue;
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    if (!lane_ok[v]) continue;
                    float* gp = Gn + (size_t)tex[t] * tstride + (size_t)32 * v * NF;
#pragma unroll
                    for (int e = 0; e < NF; e += 4)
                        red_add_v4(gp + e, wt * dg[v][e], wt * dg[v][e + 1], wt * dg[v][e + 2], wt * dg[v][e + 3]);
                }
            }
            // weight gradient (the sample against dout) and the derivative of
            // the sample in (fx, fy) inside its cell
            const float wx1 = __fsub_rn(fx, floorf(fx)), wy1 = __fsub_rn(fy, floorf(fy));
            const float wx0 = 1.0f - wx1, wy0 = 1.0f - wy1;
            float s = cw[0] * dot[0] + cw[1] * dot[1] + cw[2] * dot[2] + cw[3] * dot[3];
            float gx = wy0 * (dot[1] - dot[0]) + wy1 * (dot[3] - dot[2]);
            float gy = wx0 * (dot[2] - dot[0]) + wx1 * (dot[3] - dot[1]);
            s = warp_sum(s);
            gx = warp_sum(gx);
            gy = warp_sum(gy);
            if (lane == src) {
                dW[pr] = s;
                const float* cam = cams + n * kCamFloats;
                const float rd = 1.0f / my.det.depth;
                const float du[3] = {cam[12] * rd, cam[13] * rd, (cam[14] - my.det.u) * rd};
                const float dv3[3] = {cam[15] * rd, cam[16] * rd, (cam[17] - my.det.v) * rd};
                const float ax_ = gx * g.sW, ay_ = gy * g.sH;
#pragma unroll
                for (int dd = 0; dd < 3; ++dd) {
                    float val = 0.0f;
#pragma unroll
                    for (int r = 0; r < 3; ++r) val += cam[4 * r + dd] * (ax_ * du[r] + ay_ * dv3[r]);
                    doff[my.k * 3 + dd] += w * val;
                }
            }
            __syncwarp();
        }
    }
    __syncthreads();
    float* dO = a.doffsets + ((size_t)b * a.Q + q) * a.Kp * 3;
    for (int t = threadIdx.x; t < a.Kp * 3; t += kDeformWarps * 32) {
        float s = doff0[t];
#pragma unroll
        for (int ww = 1; ww < kDeformWarps; ++ww) s = __fadd_rn(s, doff0[ww * cpad + t]);
        dO[t] = s;
    }
}

namespace {

template <auto K>
cudaError_t launch(const DeformArgs& a, cudaStream_t st) {
    const auto k = K;
    const size_t smem = deform_smem_bytes(a.N, a.C, a.Kp);
    static std::atomic<long long> attrs[kAttrDevices];
    const cudaError_t e = set_smem_attributes(k, smem, -1, attrs);
    if (e != cudaSuccess) return e;
    const dim3 grid(a.Q, a.B);
    k<<<grid, kDeformWarps * 32, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

}  // namespace bev

cudaError_t bev_launch_deform_forward(const bev::DeformArgs& a, bool bf16, int V, cudaStream_t stream) {
    using namespace bev;
    switch ((bf16 ? 16 : 0) + V) {
        case 1: return launch<deform_forward_kernel<false, 1>>(a, stream);
        case 2: return launch<deform_forward_kernel<false, 2>>(a, stream);
        case 3: return launch<deform_forward_kernel<false, 3>>(a, stream);
        case 4: return launch<deform_forward_kernel<false, 4>>(a, stream);
        case 16 + 1: return launch<deform_forward_kernel<true, 1>>(a, stream);
        case 16 + 2: return launch<deform_forward_kernel<true, 2>>(a, stream);
        case 16 + 3: return launch<deform_forward_kernel<true, 3>>(a, stream);
        case 16 + 4: return launch<deform_forward_kernel<true, 4>>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t bev_launch_deform_backward(const bev::DeformArgs& a, bool bf16, int V, cudaStream_t stream) {
    using namespace bev;
    switch ((bf16 ? 16 : 0) + V) {
        case 1: return launch<deform_backward_kernel<false, 1>>(a, stream);
        case 2: return launch<deform_backward_kernel<false, 2>>(a, stream);
        case 3: return launch<deform_backward_kernel<false, 3>>(a, stream);
        case 4: return launch<deform_backward_kernel<false, 4>>(a, stream);
        case 16 + 1: return launch<deform_backward_kernel<true, 1>>(a, stream);
        case 16 + 2: return launch<deform_backward_kernel<true, 2>>(a, stream);
        case 16 + 3: return launch<deform_backward_kernel<true, 3>>(a, stream);
        case 16 + 4: return launch<deform_backward_kernel<true, 4>>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}
