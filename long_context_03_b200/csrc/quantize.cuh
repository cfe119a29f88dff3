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

// RoPE, then the same quantiser, for appended indexer queries / keys
// ("Lightning Indexer 的计算过程", step 2 <1> then <2>): the first rope_dim
// dimensions of every head of row r are turned pairwise by pos[r] * theta_i,
// theta_i = base^(-2i / rope_dim) (the rotary encoding of RoFormer), pairs
// (2i, 2i+1) when interleaved, else (i, i + rope_dim/2); the rest of each head
// passes through. Angles, sines and the rotation are float64 (products and
// the difference each rounded once, no fused multiply-add), then the rotated
// value is rounded to fp32: a value therefore differs from the float64
// rotation only by that last rounding, up to the few-ulp float64 differences
// of pow/sincos. The quantiser then reads those fp32 values exactly as
// quantize_e4m3_rows does. One CTA per row; the rotation is evaluated twice
// (absmax pass, encoding pass) by the same code, so both see equal values.
constexpr int kRopeMaxHalf = 64;  // rope_dim <= 128

__device__ __forceinline__ float rope_value(const float* __restrict__ xh, int j, int rope_dim, bool interleaved,
                                            const double* cs_c, const double* cs_s) {
  if (j >= rope_dim) return xh[j];
  const int half = rope_dim >> 1;
  int pi, partner;
  bool first;
  if (interleaved) {
    pi = j >> 1;
    first = (j & 1) == 0;
    partner = j ^ 1;
  } else {
    first = j < half;
    pi = first ? j : j - half;
    partner = first ? j + half : j - half;
  }
  const double a = static_cast<double>(first ? xh[j] : xh[partner]);
  const double b = static_cast<double>(first ? xh[partner] : xh[j]);
  const double c = cs_c[pi], s = cs_s[pi];
  const double v = first ? __dsub_rn(__dmul_rn(a, c), __dmul_rn(b, s)) : __dadd_rn(__dmul_rn(a, s), __dmul_rn(b, c));
  return __double2float_rn(v);
}

__global__ void __launch_bounds__(kQuantThreads)
    rope_quantize_e4m3_rows_kernel(const float* __restrict__ x, const int32_t* __restrict__ pos, int n, int heads,
                                   int d, int rope_dim, double base, int interleaved, uint8_t* __restrict__ codes,
                                   float* __restrict__ scale, float* __restrict__ rotated) {
  __shared__ float wmax[kQuantThreads / 32];
  __shared__ double cs_c[kRopeMaxHalf], cs_s[kRopeMaxHalf];
  const int nd = heads * d;
  const int half = rope_dim >> 1;
  for (int r = blockIdx.x; r < n; r += gridDim.x) {
    const float* xr = x + static_cast<size_t>(r) * nd;
    const double p = static_cast<double>(pos[r]);
    for (int i = threadIdx.x; i < half; i += kQuantThreads) {
      const double theta = pow(base, static_cast<double>(-2 * i) / static_cast<double>(rope_dim));
      double sn, cn;
      sincos(__dmul_rn(p, theta), &sn, &cn);
      cs_c[i] = cn;
      cs_s[i] = sn;
    }
    __syncthreads();
    float amax = 0.f;
    for (int e = threadIdx.x; e < nd; e += kQuantThreads) {
      const int h = e / d;
      const float v = rope_value(xr + static_cast<size_t>(h) * d, e - h * d, rope_dim, interleaved != 0, cs_c, cs_s);
      amax = fmaxf(amax, fabsf(v));
      if (rotated) rotated[static_cast<size_t>(r) * nd + e] = v;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = wmax[0];
#pragma unroll
    for (int w = 1; w < kQuantThreads / 32; ++w) amax = fmaxf(amax, wmax[w]);
    const float sc = (amax > 0.f) ? __fdiv_rn(amax, 448.f) : 1.f;
    if (threadIdx.x == 0) scale[r] = sc;
    uint8_t* cr = codes + static_cast<size_t>(r) * nd;
    for (int e = threadIdx.x; e < nd; e += kQuantThreads) {
      const int h = e / d;
      const float v = rope_value(xr + static_cast<size_t>(h) * d, e - h * d, rope_dim, interleaved != 0, cs_c, cs_s);
      const float y = fminf(fmaxf(__fdiv_rn(v, sc), -448.f), 448.f);
      cr[e] = static_cast<uint8_t>(__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3));
    }
    __syncthreads();  // wmax and the angle table are reused by the next row
  }
}

}  // namespace dsa
