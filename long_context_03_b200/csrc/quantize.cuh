// FP8 (E4M3) quantiser for tokens appended to the caches: per row, scale =
// absmax/448 in fp32 (1 for an all-zero row) and code = E4M3(x / scale) by
// round-to-nearest-even, saturating to +-448 ("Lightning Indexer 的计算过程",
// step 2 <2>, FP8 量化, adg.csdn.net/695234...). The divisions are IEEE fp32
// (correctly rounded), the conversion is the hardware's RNE one, so the
// result is bit-identical to the definition. One CTA per row.
#pragma once

#include <cuda_fp8.h>

#include "dsa_common.cuh"

namespace dsa {

constexpr int kQuantThreads = 256;

__global__ void __launch_bounds__(kQuantThreads)
    quantize_e4m3_rows_kernel(const float* __restrict__ x, int n, int d, uint8_t* __restrict__ codes,
                              float* __restrict__ scale) {
  __shared__ float wmax[kQuantThreads / 32];
  for (int r = blockIdx.x; r < n; r += gridDim.x) {
    const float* xr = x + static_cast<size_t>(r) * d;
    float amax = 0.f;
    for (int i = threadIdx.x; i < d; i += kQuantThreads) amax = fmaxf(amax, fabsf(xr[i]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = wmax[0];
#pragma unroll
    for (int w = 1; w < kQuantThreads / 32; ++w) amax = fmaxf(amax, wmax[w]);
    const float sc = (amax > 0.f) ? __fdiv_rn(amax, 448.f) : 1.f;
    if (threadIdx.x == 0) scale[r] = sc;
    uint8_t* cr = codes + static_cast<size_t>(r) * d;
    for (int i = threadIdx.x; i < d; i += kQuantThreads) {
      const float y = fminf(fmaxf(__fdiv_rn(xr[i], sc), -448.f), 448.f);
      cr[i] = static_cast<uint8_t>(__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3));
    }
    __syncthreads();  // wmax is reused by the next row
  }
}

}  // namespace dsa
