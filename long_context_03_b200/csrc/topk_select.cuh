// Exact top-K selection helpers over 64-bit ranking keys.
//
// A ranking key packs (order-preserving score bits << 32) | ~s, so "larger key"
// is exactly the order (score descending, index ascending) of the fine-grained
// token selection ("Lightning Indexer 的计算过程", step 4 <1>, on
// adg.csdn.net/695234...: keep the index_topk best-scoring tokens), with ties
// going to the lower index. Keys are unique, so the K largest keys are a
// unique set. Key 0 marks an empty slot and is never a valid key.
#pragma once

#include "dsa_common.cuh"

namespace dsa {

// Cooperative radix select over keys held in registers.
//
// `NT` threads (thread index `et`, synchronised with named barrier `bar_id`)
// hold up to MAXPER keys each in v[] (0 = empty). Finds `floor`, the smallest
// key value such that exactly K keys are >= floor (K < number of valid keys),
// by walking 8-bit digits from the first bit where the keys differ.
// scratch: >= 256 + 8 ints of shared memory.
template <int NT, int MAXPER>
__device__ __forceinline__ uint64_t radix_select_floor(const uint64_t (&v)[MAXPER], int K, int* scratch, int et,
                                                       uint32_t bar_id) {
  int* hist = scratch;
  unsigned long long* mm = reinterpret_cast<unsigned long long*>(scratch + 256);  // [0]=min [1]=max... via atomics
  int* misc = scratch + 256 + 4;
  // min / max over valid keys -> common prefix to skip
  unsigned long long kmin = ~0ull, kmax = 0ull;
#pragma unroll
  for (int j = 0; j < MAXPER; ++j) {
    if (v[j] != 0) {
      kmin = v[j] < kmin ? v[j] : kmin;
      kmax = v[j] > kmax ? v[j] : kmax;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    unsigned long long a = __shfl_xor_sync(0xffffffffu, kmin, off);
    unsigned long long b = __shfl_xor_sync(0xffffffffu, kmax, off);
    kmin = a < kmin ? a : kmin;
    kmax = b > kmax ? b : kmax;
  }
  if (et == 0) {
    mm[0] = ~0ull;
    mm[1] = 0ull;
  }
  named_bar_sync(bar_id, NT);
  if ((et & 31) == 0) {
    atomicMin(&mm[0], kmin);
    atomicMax(&mm[1], kmax);
  }
  named_bar_sync(bar_id, NT);
  kmin = mm[0];
  kmax = mm[1];
  const uint64_t diff = kmin ^ kmax;
  const int hi_bit = diff ? 63 - __clzll(static_cast<long long>(diff)) : 0;  // highest differing bit
  int shift = hi_bit & ~7;  // byte-aligned digits; bits above shift+8 are common to all keys
  uint64_t prefix = (shift + 8 >= 64) ? 0ull : (kmax >> (shift + 8)) << (shift + 8);
  int remaining = K;
  while (true) {
    for (int i = et; i < 256; i += NT) hist[i] = 0;
    named_bar_sync(bar_id, NT);
#pragma unroll
    for (int j = 0; j < MAXPER; ++j) {
      const uint64_t x = v[j];
      const bool match = (x != 0) && ((shift + 8 >= 64) || ((x >> (shift + 8)) == (prefix >> (shift + 8))));
      if (match) atomicAdd(&hist[(x >> shift) & 255u], 1);
    }
    named_bar_sync(bar_id, NT);
    if (et < 32) {
      const int l = et;
      int c[8];
      int tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = hist[255 - 8 * l - i];
        tot += c[i];
      }
      int incl = tot;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (l >= off) incl += y;
      }
      const uint32_t ball = __ballot_sync(0xffffffffu, incl >= remaining);
      const int L0 = __ffs(ball) - 1;
      if (l == L0) {
        int cum = incl - tot;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (cum + c[i] >= remaining) {
            misc[0] = 255 - 8 * l - i;
            misc[1] = cum;
            misc[2] = c[i];
            break;
          }
          cum += c[i];
        }
      }
    }
    named_bar_sync(bar_id, NT);
    const int d = misc[0];
    const int above = misc[1];
    const int inb = misc[2];
    remaining -= above;
    prefix |= static_cast<uint64_t>(d) << shift;
    if (inb == remaining || shift == 0) break;
    shift -= 8;
  }
  return prefix;  // bits below `shift` are zero
}

// Compact row `c[0..n)` (global memory, keys) to exactly K keys (K < n) in
// c[0..K), unordered. Returns the floor used (every kept key >= floor).
template <int NT, int MAXPER>
__device__ __forceinline__ uint64_t compact_top_k(uint64_t* c, int n, int K, int* scratch, int et, uint32_t bar_id) {
  uint64_t v[MAXPER];
#pragma unroll
  for (int j = 0; j < MAXPER; ++j) {
    const int i = et + j * NT;
    v[j] = (i < n) ? c[i] : 0ull;
  }
  const uint64_t floor = radix_select_floor<NT, MAXPER>(v, K, scratch, et, bar_id);
  int* wpos = scratch + 256 + 8;
  if (et == 0) *wpos = 0;
  named_bar_sync(bar_id, NT);
#pragma unroll
  for (int j = 0; j < MAXPER; ++j) {
    if (v[j] != 0 && v[j] >= floor) {
      const int pos = atomicAdd(wpos, 1);
      c[pos] = v[j];
    }
  }
  named_bar_sync(bar_id, NT);
  return floor;
}

// One CTA per row: sort the row's K keys descending (bitonic, in shared
// memory) and write the token indices; empty slots (key 0) become -1.
// keys [rows, K] (row r at keys + r*K), idx [rows, K].
template <int P>  // power of two >= K
__global__ void __launch_bounds__(256) rank_sort_kernel(const uint64_t* __restrict__ keys, int32_t* __restrict__ idx,
                                                        int K, int rows) {
  __shared__ uint64_t s[P];
  const int r = blockIdx.x;
  if (r >= rows) return;
  const uint64_t* src = keys + static_cast<size_t>(r) * K;
  for (int i = threadIdx.x; i < P; i += blockDim.x) s[i] = (i < K) ? src[i] : 0ull;
  __syncthreads();
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < P / 2; i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool desc = ((lo & size) == 0);  // final merge (size == P) is descending everywhere
        const uint64_t a = s[lo], b = s[hi];
        if ((a < b) == desc) {
          s[lo] = b;
          s[hi] = a;
        }
      }
      __syncthreads();
    }
  }
  int32_t* dst = idx + static_cast<size_t>(r) * K;
  for (int i = threadIdx.x; i < K; i += blockDim.x) {
    const uint64_t k = s[i];
    dst[i] = (k == 0ull) ? -1 : rank_key_index(k);
  }
}

}  // namespace dsa
