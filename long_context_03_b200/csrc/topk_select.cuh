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
// by walking 8-bit digits from the first bit where the keys differ. Each warp
// counts into its own histogram (no cross-warp atomic contention); the
// histograms are then summed per bin.
// scratch: select_scratch_ints(NT) ints of shared memory.
__host__ __device__ constexpr int select_scratch_ints(int nt) { return (nt / 32) * 256 + 16; }

template <int NT, int MAXPER>
__device__ __forceinline__ uint64_t radix_select_floor(const uint64_t (&v)[MAXPER], int K, int* scratch, int et,
                                                       uint32_t bar_id) {
  constexpr int NW = NT / 32;
  int* hist = scratch;                                   // [NW][256]
  unsigned long long* mm = reinterpret_cast<unsigned long long*>(scratch + NW * 256);  // min, max
  int* misc = scratch + NW * 256 + 4;                    // digit, count above, count in bin
  int* my_hist = hist + (et >> 5) * 256;
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
    for (int i = et; i < NW * 256; i += NT) hist[i] = 0;
    named_bar_sync(bar_id, NT);
#pragma unroll
    for (int j = 0; j < MAXPER; ++j) {
      const uint64_t x = v[j];
      const bool match = (x != 0) && ((shift + 8 >= 64) || ((x >> (shift + 8)) == (prefix >> (shift + 8))));
      if (match) atomicAdd(&my_hist[(x >> shift) & 255u], 1);
    }
    named_bar_sync(bar_id, NT);
    for (int i = et; i < 256; i += NT) {
      int tot = 0;
#pragma unroll
      for (int w = 0; w < NW; ++w) tot += hist[w * 256 + i];
      hist[i] = tot;
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
  int* wpos = scratch + (NT / 32) * 256 + 8;
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

// Exclusive prefix sum of one int per thread over NT threads (named barrier
// bar_id). wsum: NT/32 + 1 ints of shared memory. Returns the prefix;
// *total gets the sum over all threads.
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int x, int* wsum, int et, uint32_t bar_id, int* total) {
  constexpr int NW = NT / 32;
  const int l = et & 31, w = et >> 5;
  int incl = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (l >= off) incl += y;
  }
  named_bar_sync(bar_id, NT);  // wsum may still be read by a previous scan
  if (l == 31) wsum[w] = incl;
  named_bar_sync(bar_id, NT);
  int base = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < NW; ++i) {
    const int v = wsum[i];
    base += (i < w) ? v : 0;
    tot += v;
  }
  *total = tot;
  return base + incl - x;
}

// ---------------------------------------------------------------------------
// Candidate lists split in four quarter sub-lists (one writer warp each).
// ---------------------------------------------------------------------------
// Scratch layout (ints) for the cut below: [0, 2048) histogram, then 8 warp
// sums, then small fields.
__host__ __device__ constexpr int cut_scratch_ints() { return 2048 + 64; }  // wsum needs NT/32 <= 16 ints

// Count of each 11-bit digit of the valid keys (from the highest bit where the
// keys differ), then find the digit bin holding the K-th largest key.
// Returns the bin's lower edge `floor`; *above = keys in higher bins,
// *inb = keys in that bin (so keys >= floor number *above + *inb >= K).
template <int NT, int M>
__device__ __forceinline__ uint64_t histogram_cut(const uint64_t (&v)[M], int K, int* scratch, int et,
                                                  uint32_t bar_id, int* above_out, int* inb_out) {
  constexpr int NW = NT / 32;
  static_assert(NT == 256 || NT == 512, "the 2048-bin scan takes 256 or 512 threads");
  constexpr int BPT = 2048 / NT;  // bins per thread
  int* hist = scratch;
  int* wsum = scratch + 2048;
  unsigned long long* mm = reinterpret_cast<unsigned long long*>(scratch + 2048 + 16);
  int* res = scratch + 2048 + 24;
  unsigned long long kmin = ~0ull, kmax = 0ull;
#pragma unroll
  for (int j = 0; j < M; ++j) {
    if (v[j] != 0) {
      kmin = v[j] < kmin ? v[j] : kmin;
      kmax = v[j] > kmax ? v[j] : kmax;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const unsigned long long a = __shfl_xor_sync(0xffffffffu, kmin, off);
    const unsigned long long b = __shfl_xor_sync(0xffffffffu, kmax, off);
    kmin = a < kmin ? a : kmin;
    kmax = b > kmax ? b : kmax;
  }
  if (et == 0) {
    mm[0] = ~0ull;
    mm[1] = 0ull;
  }
  for (int i = et; i < 2048; i += NT) hist[i] = 0;
  named_bar_sync(bar_id, NT);
  if ((et & 31) == 0) {
    atomicMin(&mm[0], kmin);
    atomicMax(&mm[1], kmax);
  }
  named_bar_sync(bar_id, NT);
  kmin = mm[0];
  kmax = mm[1];
  const uint64_t diff = kmin ^ kmax;
  const int hi_bit = diff ? 63 - __clzll(static_cast<long long>(diff)) : 0;
  const int shift = hi_bit >= 10 ? hi_bit - 10 : 0;
  const uint64_t prefix = (shift + 11 >= 64) ? 0ull : (kmax >> (shift + 11)) << (shift + 11);
#pragma unroll
  for (int j = 0; j < M; ++j)
    if (v[j] != 0) atomicAdd(&hist[(v[j] >> shift) & 2047u], 1);
  named_bar_sync(bar_id, NT);
  // descending scan: thread et owns bins 2047-BPT*et .. 2048-BPT*(et+1)
  int c[BPT];
  int tot = 0;
#pragma unroll
  for (int i = 0; i < BPT; ++i) {
    c[i] = hist[2047 - BPT * et - i];
    tot += c[i];
  }
  const int l = et & 31, w = et >> 5;
  int incl = tot;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (l >= off) incl += y;
  }
  if (l == 31) wsum[w] = incl;
  named_bar_sync(bar_id, NT);
  int wbase = 0;
#pragma unroll
  for (int i = 0; i < NW; ++i) wbase += (i < w) ? wsum[i] : 0;
  const int excl = wbase + incl - tot;
  if (excl < K && excl + tot >= K) {
    int cum = excl;
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
      if (cum + c[i] >= K) {
        res[0] = 2047 - BPT * et - i;
        res[1] = cum;
        res[2] = c[i];
        break;
      }
      cum += c[i];
    }
  }
  named_bar_sync(bar_id, NT);
  *above_out = res[1];
  *inb_out = res[2];
  return prefix | (static_cast<uint64_t>(res[0]) << shift);
}

// Load a row's four quarter sub-lists (counts cnt[0..3], capacity capq each)
// into registers: v[q*MQ + j] = sub-list q entry et + j*NT (0 if absent).
template <int NT, int MQ>
__device__ __forceinline__ void load_sublists(const uint64_t* row, int capq, const int* cnt, int et,
                                              uint64_t (&v)[4 * MQ]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int n = cnt[q];
#pragma unroll
    for (int j = 0; j < MQ; ++j) {
      const int i = et + j * NT;
      v[q * MQ + j] = (i < n) ? row[static_cast<size_t>(q) * capq + i] : 0ull;
    }
  }
}

// Write every key >= floor back, spread round-robin over the four sub-lists,
// and set their counts. Positions come from a block-wide prefix sum of the
// per-thread survivor counts (no atomics). Returns the number kept.
template <int NT, int MQ>
__device__ __forceinline__ int store_sublists(uint64_t* row, int capq, int* cnt, const uint64_t (&v)[4 * MQ],
                                              uint64_t floor, int* wsum, int et, uint32_t bar_id) {
  int mine = 0;
#pragma unroll
  for (int j = 0; j < 4 * MQ; ++j) mine += (v[j] != 0 && v[j] >= floor) ? 1 : 0;
  int kept = 0;
  int pos = block_exclusive_scan<NT>(mine, wsum, et, bar_id, &kept);
#pragma unroll
  for (int j = 0; j < 4 * MQ; ++j) {
    if (v[j] != 0 && v[j] >= floor) {
      row[static_cast<size_t>(pos & 3) * capq + (pos >> 2)] = v[j];
      ++pos;
    }
  }
  if (et < 4) cnt[et] = (kept + 3 - et) / 4;
  return kept;
}

// One CTA per row (small K): sort the row's K keys descending (bitonic, in
// shared memory) and write the token indices; empty slots (key 0) become -1.
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

// Compare-exchange of the in-thread pairs (a, a | S), a & S == 0, of a
// thread's 8 consecutive elements 8i..8i+7 within bitonic blocks of `size`.
template <int S>
__device__ __forceinline__ void bitonic_reg_step(uint64_t (&v)[8], int i, int size) {
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    if ((a & S) == 0) {
      const int b = a | S;
      const bool desc = ((8 * i + a) & size) == 0;
      const uint64_t mx = v[a] > v[b] ? v[a] : v[b], mn = v[a] > v[b] ? v[b] : v[a];
      v[a] = desc ? mx : mn;
      v[b] = desc ? mn : mx;
    }
  }
}

// One CTA of P/8 threads per row, 8 keys per thread in registers: a bitonic
// sort into descending key order (= score descending, index ascending).
// Strides below 8 stay inside a thread, strides 8..128 go through warp
// shuffles, larger strides through shared memory. Writes the token indices;
// empty slots (key 0) become -1.
template <int P>
__global__ void __launch_bounds__(P / 8) rank_sort_reg_kernel(const uint64_t* __restrict__ keys,
                                                               int32_t* __restrict__ idx, int K, int rows) {
  static_assert(P >= 256 && P <= 2048, "8 keys per thread, at least one warp");
  __shared__ uint64_t sm[P];
  const int r = blockIdx.x;
  if (r >= rows) return;
  const int i = threadIdx.x;
  const uint64_t* src = keys + static_cast<size_t>(r) * K;
  uint64_t v[8];
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int e = 8 * i + a;
    v[a] = (e < K) ? src[e] : 0ull;
  }
#pragma unroll 1
  for (int size = 2; size <= P; size <<= 1) {
#pragma unroll 1
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride >= 256) {
        __syncthreads();
#pragma unroll
        for (int a = 0; a < 8; ++a) sm[8 * i + a] = v[a];
        __syncthreads();
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          const int e = 8 * i + a;
          const uint64_t o = sm[e ^ stride];
          const bool lower = (e & stride) == 0;
          const bool desc = (e & size) == 0;
          const uint64_t mx = v[a] > o ? v[a] : o, mn = v[a] > o ? o : v[a];
          v[a] = (lower == desc) ? mx : mn;
        }
      } else if (stride >= 8) {
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          const int e = 8 * i + a;
          const uint64_t o = __shfl_xor_sync(0xffffffffu, v[a], stride >> 3);
          const bool lower = (e & stride) == 0;
          const bool desc = (e & size) == 0;
          const uint64_t mx = v[a] > o ? v[a] : o, mn = v[a] > o ? o : v[a];
          v[a] = (lower == desc) ? mx : mn;
        }
      } else if (stride == 4) {
        bitonic_reg_step<4>(v, i, size);
      } else if (stride == 2) {
        bitonic_reg_step<2>(v, i, size);
      } else {
        bitonic_reg_step<1>(v, i, size);
      }
    }
  }
  int32_t* dst = idx + static_cast<size_t>(r) * K;
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int e = 8 * i + a;
    if (e < K) dst[e] = (v[a] == 0ull) ? -1 : rank_key_index(v[a]);
  }
}

}  // namespace dsa
