// bev_layout.cu -- layout transforms around the sampling kernels (sm_100a).
//
// to_channels_last: features [BN][C][HW] (or [BN][HW][C]) -> [BN][HW][Cp] with
//   zero padding channels, so that one texel's channel vector is contiguous
//   and 16-byte aligned for the gather kernels.  Pure HBM-bound copies: the
//   NCHW case moves 4x4 blocks (4-byte elements) or 8x8 blocks (2-byte
//   elements) with 16-byte loads and stores when the shapes allow it, else a
//   32x32 shared-memory tiled transpose (coalesced on both sides); the
//   unaligned-NHWC case is a straight strided copy.
// to_nchw: the fp32 channels-last gradient buffer [BN][HW][Cp] -> [BN][C][HW].
//   When HW is a multiple of 4 and the output is 16-byte aligned, each thread
//   moves a 4 texel x 4 channel block with 16-byte loads and 16-byte stores
//   (a register transpose; whole 32-byte sectors on both sides); otherwise a
//   32x32 shared-memory tiled transpose.
#include <stdint.h>

#include "bev_kernels.cuh"

namespace bev {

constexpr int kT = 32;

template <typename T>
__global__ void __launch_bounds__(256) nchw_to_nhwc_kernel(const T* __restrict__ src, int C, int HW,
                                                           int Cp, T* __restrict__ dst) {
    __shared__ T tile[kT][kT + 1];
    const size_t bn = blockIdx.z;
    const int p0 = blockIdx.x * kT, c0 = blockIdx.y * kT;
    const T* s = src + bn * (size_t)C * HW;
    T* d = dst + bn * (size_t)HW * Cp;
    for (int r = threadIdx.y; r < kT; r += 8) {
        const int c = c0 + r, p = p0 + threadIdx.x;
        tile[r][threadIdx.x] = (c < C && p < HW) ? s[(size_t)c * HW + p] : T(0);
    }
    __syncthreads();
    for (int r = threadIdx.y; r < kT; r += 8) {
        const int p = p0 + r, c = c0 + threadIdx.x;
        if (p < HW && c < Cp) d[(size_t)p * Cp + c] = tile[threadIdx.x][r];
    }
}

template <typename T>
__global__ void __launch_bounds__(256) nhwc_pad_kernel(const T* __restrict__ src, int C, size_t rows,
                                                       int Cp, T* __restrict__ dst) {
    const size_t total = rows * (size_t)Cp;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total;
         e += (size_t)gridDim.x * blockDim.x) {
        const size_t r = e / Cp;
        const int c = (int)(e - r * Cp);
        dst[e] = c < C ? src[r * C + c] : T(0);
    }
}

__global__ void __launch_bounds__(256) nhwc_to_nchw_kernel(const float* __restrict__ src, int C, int HW,
                                                           int Cp, float* __restrict__ dst) {
    __shared__ float tile[kT][kT + 1];
    const size_t bn = blockIdx.z;
    const int p0 = blockIdx.x * kT, c0 = blockIdx.y * kT;
    const float* s = src + bn * (size_t)HW * Cp;
    float* d = dst + bn * (size_t)C * HW;
    for (int r = threadIdx.y; r < kT; r += 8) {
        const int p = p0 + r, c = c0 + threadIdx.x;
        tile[r][threadIdx.x] = (p < HW && c < C) ? s[(size_t)p * Cp + c] : 0.0f;
    }
    __syncthreads();
    for (int r = threadIdx.y; r < kT; r += 8) {
        const int c = c0 + r, p = p0 + threadIdx.x;
        if (c < C && p < HW) d[(size_t)c * HW + p] = tile[threadIdx.x][r];
    }
}

// 4x4 register-blocked NCHW -> channels-last copy for 4-byte elements: block
// (16 x 16 threads) covers 64 channels x 64 texels; thread (tx, ty) reads
// channels 4 ty .. 4 ty + 3 at texels 4 tx .. 4 tx + 3 and writes them as four
// texel rows; padding channels (C <= c < Cp) are written as 0.  HW % 4 == 0,
// Cp % 4 == 0, both pointers 16-byte aligned.
__global__ void __launch_bounds__(256) nchw_to_nhwc_v4_kernel(const float* __restrict__ src, int C, int HW,
                                                              int Cp, float* __restrict__ dst) {
    const size_t bn = blockIdx.z;
    const int c = blockIdx.y * 64 + 4 * threadIdx.y;
    const int p = blockIdx.x * 64 + 4 * threadIdx.x;
    if (p >= HW || c >= Cp) return;
    float4 r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        r[i] = c + i < C ? __ldg(reinterpret_cast<const float4*>(src + (bn * C + c + i) * (size_t)HW + p))
                         : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    float* d = dst + (bn * HW + p) * (size_t)Cp + c;
    *reinterpret_cast<float4*>(d) = make_float4(r[0].x, r[1].x, r[2].x, r[3].x);
    *reinterpret_cast<float4*>(d + Cp) = make_float4(r[0].y, r[1].y, r[2].y, r[3].y);
    *reinterpret_cast<float4*>(d + 2 * (size_t)Cp) = make_float4(r[0].z, r[1].z, r[2].z, r[3].z);
    *reinterpret_cast<float4*>(d + 3 * (size_t)Cp) = make_float4(r[0].w, r[1].w, r[2].w, r[3].w);
}

// 8x8 register-blocked NCHW -> channels-last copy for 2-byte elements: block
// (16 x 16 threads) covers 128 channels x 128 texels; thread (tx, ty) reads
// channels 8 ty .. 8 ty + 7 at texels 8 tx .. 8 tx + 7 (eight 16-byte loads)
// and writes eight texel rows of 8 channels (eight 16-byte stores); each
// output word pairs the same texel of two channels (a byte permute).
// Padding channels are written as 0.  HW % 8 == 0, Cp % 8 == 0, both
// pointers 16-byte aligned.
__global__ void __launch_bounds__(256) nchw_to_nhwc_16x8_kernel(const uint16_t* __restrict__ src, int C, int HW,
                                                                int Cp, uint16_t* __restrict__ dst) {
    const size_t bn = blockIdx.z;
    const int c = blockIdx.y * 128 + 8 * threadIdx.y;
    const int p = blockIdx.x * 128 + 8 * threadIdx.x;
    if (p >= HW || c >= Cp) return;
    uint4 r[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        r[i] = c + i < C ? __ldg(reinterpret_cast<const uint4*>(src + (bn * C + c + i) * (size_t)HW + p))
                         : make_uint4(0u, 0u, 0u, 0u);
    uint16_t* d = dst + (bn * HW + p) * (size_t)Cp + c;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        // texel j sits in word j / 2 of every channel row, low half for even j
        const unsigned sel = (j & 1) ? 0x7632u : 0x5410u;
        unsigned w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint4& v = r[i];
            w[i] = (j >> 1) == 0 ? v.x : (j >> 1) == 1 ? v.y : (j >> 1) == 2 ? v.z : v.w;
        }
        const uint4 o = make_uint4(__byte_perm(w[0], w[1], sel), __byte_perm(w[2], w[3], sel),
                                   __byte_perm(w[4], w[5], sel), __byte_perm(w[6], w[7], sel));
        *reinterpret_cast<uint4*>(d + (size_t)j * Cp) = o;
    }
}

// 4x4 register-blocked transpose: block (16 x 16 threads) covers 64 texels x
// 64 channels; thread (tx, ty) reads texels 4 ty .. 4 ty + 3 at channels
// 4 tx .. 4 tx + 3 and writes them back as four channel rows.  HW % 4 == 0,
// Cp % 4 == 0, dst 16-byte aligned.
__global__ void __launch_bounds__(256) nhwc_to_nchw_v4_kernel(const float* __restrict__ src, int C, int HW,
                                                              int Cp, float* __restrict__ dst) {
    const size_t bn = blockIdx.z;
    const int p = blockIdx.x * 64 + 4 * threadIdx.y;
    const int c = blockIdx.y * 64 + 4 * threadIdx.x;
    if (p >= HW || c >= C) return;
    const float* s = src + (bn * HW + p) * (size_t)Cp + c;
    float4 r[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) r[j] = __ldg(reinterpret_cast<const float4*>(s + (size_t)j * Cp));
    float* d = dst + (bn * C + c) * (size_t)HW + p;
    const float col[4][4] = {{r[0].x, r[1].x, r[2].x, r[3].x},
                             {r[0].y, r[1].y, r[2].y, r[3].y},
                             {r[0].z, r[1].z, r[2].z, r[3].z},
                             {r[0].w, r[1].w, r[2].w, r[3].w}};
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (c + i < C)
            *reinterpret_cast<float4*>(d + (size_t)i * HW) = make_float4(col[i][0], col[i][1], col[i][2], col[i][3]);
}

}  // namespace bev

cudaError_t bev_launch_to_channels_last(const void* src, int layout, int esize, int BN, int C, int HW,
                                        int Cp, void* dst, cudaStream_t stream) {
    if (layout == 0 && esize == 4 && HW % 4 == 0 && Cp % 4 == 0 && ((uintptr_t)src % 16) == 0 &&
        ((uintptr_t)dst % 16) == 0) {
        const dim3 grid((HW + 63) / 64, (Cp + 63) / 64, BN);
        bev::nchw_to_nhwc_v4_kernel<<<grid, dim3(16, 16), 0, stream>>>((const float*)src, C, HW, Cp, (float*)dst);
    } else if (layout == 0 && esize == 2 && HW % 8 == 0 && Cp % 8 == 0 && ((uintptr_t)src % 16) == 0 &&
               ((uintptr_t)dst % 16) == 0) {
        const dim3 grid((HW + 127) / 128, (Cp + 127) / 128, BN);
        bev::nchw_to_nhwc_16x8_kernel<<<grid, dim3(16, 16), 0, stream>>>((const uint16_t*)src, C, HW, Cp,
                                                                         (uint16_t*)dst);
    } else if (layout == 0) {  // NCHW
        const dim3 grid((HW + bev::kT - 1) / bev::kT, (Cp + bev::kT - 1) / bev::kT, BN);
        const dim3 block(bev::kT, 8);
        if (esize == 4)
            bev::nchw_to_nhwc_kernel<uint32_t><<<grid, block, 0, stream>>>(
                (const uint32_t*)src, C, HW, Cp, (uint32_t*)dst);
        else
            bev::nchw_to_nhwc_kernel<uint16_t><<<grid, block, 0, stream>>>(
                (const uint16_t*)src, C, HW, Cp, (uint16_t*)dst);
    } else {
        const size_t rows = (size_t)BN * HW;
        const size_t total = rows * Cp;
        const int blocks = (int)((total + 255) / 256 < 148 * 16 ? (total + 255) / 256 : 148 * 16);
        if (esize == 4)
            bev::nhwc_pad_kernel<uint32_t><<<blocks, 256, 0, stream>>>((const uint32_t*)src, C, rows, Cp,
                                                                     (uint32_t*)dst);
        else
            bev::nhwc_pad_kernel<uint16_t><<<blocks, 256, 0, stream>>>((const uint16_t*)src, C, rows, Cp,
                                                                     (uint16_t*)dst);
    }
    return cudaGetLastError();
}

cudaError_t bev_launch_to_nchw(const float* src, int BN, int C, int HW, int Cp, float* dst,
                               cudaStream_t stream) {
    if (HW % 4 == 0 && Cp % 4 == 0 && ((uintptr_t)src % 16) == 0 && ((uintptr_t)dst % 16) == 0) {
        const dim3 grid((HW + 63) / 64, (C + 63) / 64, BN);
        bev::nhwc_to_nchw_v4_kernel<<<grid, dim3(16, 16), 0, stream>>>(src, C, HW, Cp, dst);
        return cudaGetLastError();
    }
    const dim3 grid((HW + bev::kT - 1) / bev::kT, (C + bev::kT - 1) / bev::kT, BN);
    const dim3 block(bev::kT, 8);
    bev::nhwc_to_nchw_kernel<<<grid, block, 0, stream>>>(src, C, HW, Cp, dst);
    return cudaGetLastError();
}
