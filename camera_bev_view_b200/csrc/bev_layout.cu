// bev_layout.cu -- layout transforms around the sampling kernels (sm_100a).
//
// to_channels_last: features [BN][C][HW] (or [BN][HW][C]) -> [BN][HW][Cp] with
//   zero padding channels, so that one texel's channel vector is contiguous
//   and 16-byte aligned for the gather kernels.  Pure HBM-bound copies: the
//   NCHW case is a 32x32 shared-memory tiled transpose (coalesced on both
//   sides); the unaligned-NHWC case is a straight strided copy.
// to_nchw: the fp32 channels-last gradient buffer [BN][HW][Cp] -> [BN][C][HW].
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

}  // namespace bev

cudaError_t bev_launch_to_channels_last(const void* src, int layout, int esize, int BN, int C, int HW,
                                        int Cp, void* dst, cudaStream_t stream) {
    if (layout == 0) {  // NCHW
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
    const dim3 grid((HW + bev::kT - 1) / bev::kT, (C + bev::kT - 1) / bev::kT, BN);
    const dim3 block(bev::kT, 8);
    bev::nhwc_to_nchw_kernel<<<grid, block, 0, stream>>>(src, C, HW, Cp, dst);
    return cudaGetLastError();
}
