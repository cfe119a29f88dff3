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
// `NT` threads (thread index `et`, synchronised with the group barrier `bar`)
// hold up to MAXPER keys each in v[] (0 = empty). Finds `floor`, the smallest
// key value such that exactly K keys are >= floor (K < number of valid keys),
// by walking 8-bit digits from the first bit where the keys differ. Each warp
// counts into its own histogram (no cross-warp atomic contention); the
// histograms are then summed per bin.
// scratch: select_scratch_ints(NT) ints of shared memory.
__host__ __device__ constexpr int select_scratch_ints(int nt) { return (nt / 32) * 256 + 16; }

template <int NT, int MAXPER>
__device__ __forceinline__ uint64_t radix_select_floor(const uint64_t (&v)[MAXPER], int K, int* scratch, int et,
                                                       const GroupBar& bar) {
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
  bar.sync();
  if ((et & 31) == 0) {
    atomicMin(&mm[0], kmin);
    atomicMax(&mm[1], kmax);
  }
  bar.sync();
  kmin = mm[0];
  kmax = mm[1];
  const uint64_t diff = kmin ^ kmax;
  const int hi_bit = diff ? 63 - __clzll(static_cast<long long>(diff)) : 0;  // highest differing bit
  int shift = hi_bit & ~7;  // byte-aligned digits; bits above shift+8 are common to all keys
  uint64_t prefix = (shift + 8 >= 64) ? 0ull : (kmax >> (shift + 8)) << (shift + 8);
  int remaining = K;
  while (true) {
    for (int i = et; i < NW * 256; i += NT) hist[i] = 0;
    bar.sync();
#pragma unroll
    for (int j = 0; j < MAXPER; ++j) {
      const uint64_t x = v[j];
      const bool match = (x != 0) && ((shift + 8 >= 64) || ((x >> (shift + 8)) == (prefix >> (shift + 8))));
      if (match) atomicAdd(&my_hist[(x >> shift) & 255u], 1);
    }
    bar.sync();
    for (int i = et; i < 256; i += NT) {
      int tot = 0;
#pragma unroll
      for (int w = 0; w < NW; ++w) tot += hist[w * 256 + i];
      hist[i] = tot;
    }
    bar.sync();
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
    bar.sync();
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

// Exclusive prefix sum of one int per thread over NT threads (named barrier
// bar). wsum: NT/32 + 1 ints of shared memory. Returns the prefix;
// *total gets the sum over all threads.
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int x, int* wsum, int et, const GroupBar& bar, int* total) {
  constexpr int NW = NT / 32;
  const int l = et & 31, w = et >> 5;
  int incl = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (l >= off) incl += y;
  }
  bar.sync();  // wsum may still be read by a previous scan
  if (l == 31) wsum[w] = incl;
  bar.sync();
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
                                                  const GroupBar& bar, int* above_out, int* inb_out) {
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
  bar.sync();
  if ((et & 31) == 0) {
    atomicMin(&mm[0], kmin);
    atomicMax(&mm[1], kmax);
  }
  bar.sync();
  kmin = mm[0];
  kmax = mm[1];
  const uint64_t diff = kmin ^ kmax;
  const int hi_bit = diff ? 63 - __clzll(static_cast<long long>(diff)) : 0;
  const int shift = hi_bit >= 10 ? hi_bit - 10 : 0;
  const uint64_t prefix = (shift + 11 >= 64) ? 0ull : (kmax >> (shift + 11)) << (shift + 11);
#pragma unroll
  for (int j = 0; j < M; ++j)
    if (v[j] != 0) atomicAdd(&hist[(v[j] >> shift) & 2047u], 1);
  bar.sync();
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
  bar.sync();
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
  bar.sync();
  *above_out = res[1];
  *inb_out = res[2];
  return prefix | (static_cast<uint64_t>(res[0]) << shift);
}

// Exact top-K of one row, ranked, in one histogram pass. The NT threads hold
// the row's keys in v[] (0 = empty). Every key's 11-bit digit below the
// keys' common prefix puts it in one of 2048 bins; bins are ordered like the
// keys, so a descending prefix sum over the bin counts gives each bin's first
// rank, and a key's rank is that plus the number of larger keys in its own
// bin. The K-th largest key lies in bin b*: keys in higher bins all rank below
// K, keys of b* are kept by their rank, lower bins are dropped. The keys of
// bins >= b* go to buf (at most bufn) grouped by bin; dst[0..K) gets the
// token indices in rank order, -1 past the row's valid keys.
// Returns false, with nothing written, when a bin >= b* holds more than cmax
// keys or more than bufn keys lie in bins >= b*: the caller then ranks with
// the exact select and the bitonic sort. Scratch (ints, shared): hist[2048],
// start[2048], small[64].
template <int NT, int M>
__device__ __forceinline__ bool topk_rank_by_bins(const uint64_t (&v)[M], int K, int* hist, int* start, int* small,
                                                  uint64_t* buf, int bufn, int cmax, int et, const GroupBar& bar,
                                                  int32_t* __restrict__ dst) {
  constexpr int NW = NT / 32;
  static_assert(NT == 512 || NT == 1024, "two or four bins per thread");
  constexpr int BPT = 2048 / NT;
  int* wsum = small;                                                        // [NW]
  unsigned long long* mm = reinterpret_cast<unsigned long long*>(small + 32);  // min, max
  int* res = small + 40;  // b*, keys above b*, keys in b*, largest bin count, valid keys
  bar.sync();  // every thread is done with the previous row's hist, start and buf
  unsigned long long kmin = ~0ull, kmax = 0ull;
  int nv = 0;
#pragma unroll
  for (int j = 0; j < M; ++j) {
    if (v[j] != 0) {
      kmin = v[j] < kmin ? v[j] : kmin;
      kmax = v[j] > kmax ? v[j] : kmax;
      ++nv;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const unsigned long long a = __shfl_xor_sync(0xffffffffu, kmin, off);
    const unsigned long long b = __shfl_xor_sync(0xffffffffu, kmax, off);
    kmin = a < kmin ? a : kmin;
    kmax = b > kmax ? b : kmax;
    nv += __shfl_xor_sync(0xffffffffu, nv, off);
  }
  if (et == 0) {
    mm[0] = ~0ull;
    mm[1] = 0ull;
    res[0] = 0;
    res[1] = 0;
    res[2] = 0;
    res[3] = 0;
    res[4] = 0;
  }
  for (int i = et; i < 2048; i += NT) hist[i] = 0;
  bar.sync();
  if ((et & 31) == 0) {
    atomicMin(&mm[0], kmin);
    atomicMax(&mm[1], kmax);
    atomicAdd(&res[4], nv);
  }
  bar.sync();
  kmin = mm[0];
  kmax = mm[1];
  const int n = res[4];
  const uint64_t diff = kmin ^ kmax;
  const int hi_bit = diff ? 63 - __clzll(static_cast<long long>(diff)) : 0;
  const int shift = hi_bit >= 10 ? hi_bit - 10 : 0;
#pragma unroll
  for (int j = 0; j < M; ++j)
    if (v[j] != 0) atomicAdd(&hist[(v[j] >> shift) & 2047u], 1);
  bar.sync();
  // descending scan: thread et owns bins 2047 - BPT*et - i, i < BPT
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
  bar.sync();
  int wbase = 0;
#pragma unroll
  for (int i = 0; i < NW; ++i) wbase += (i < w) ? wsum[i] : 0;
  const int excl = wbase + incl - tot;
  const int keff = K < n ? K : n;  // the K-th largest, or the smallest valid key
  {
    int cum = excl;
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
      start[2047 - BPT * et - i] = cum;
      if (keff > 0 && cum < keff && cum + c[i] >= keff) {
        res[0] = 2047 - BPT * et - i;
        res[1] = cum;
        res[2] = c[i];
      }
      cum += c[i];
    }
  }
  bar.sync();
  const int bstar = res[0];
  const int total = res[1] + res[2];  // keys in bins >= b*
  int cm = 0;
#pragma unroll
  for (int i = 0; i < BPT; ++i)
    if (2047 - BPT * et - i >= bstar) cm = c[i] > cm ? c[i] : cm;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const int y = __shfl_xor_sync(0xffffffffu, cm, off);
    cm = y > cm ? y : cm;
  }
  if (l == 0 && cm > 0) atomicMax(&res[3], cm);
  bar.sync();
  if (res[3] > cmax || total > bufn) return false;  // the same answer on every thread
  // group the keys of bins >= b* by bin (start[] then points past each bin)
#pragma unroll
  for (int j = 0; j < M; ++j) {
    if (v[j] != 0) {
      const int b = static_cast<int>((v[j] >> shift) & 2047u);
      if (b >= bstar) {
        const int p = atomicAdd(&start[b], 1);
        if (p < bufn) buf[p] = v[j];
      }
    }
  }
  bar.sync();
  for (int i = et; i < total; i += NT) {
    const uint64_t key = buf[i];
    const int b = static_cast<int>((key >> shift) & 2047u);
    const int cb = hist[b];
    const int s0 = start[b] - cb;
    int r = s0;
    for (int q = s0; q < s0 + cb; ++q) r += (buf[q] > key) ? 1 : 0;
    if (r < K) __stcs(dst + r, rank_key_index(key));  // streaming store: the index rows are not read back here
  }
  for (int i = (total > 0 ? total : 0) + et; i < K; i += NT) __stcs(dst + i, -1);
  return true;
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
                                              uint64_t floor, int* wsum, int et, const GroupBar& bar) {
  int mine = 0;
#pragma unroll
  for (int j = 0; j < 4 * MQ; ++j) mine += (v[j] != 0 && v[j] >= floor) ? 1 : 0;
  int kept = 0;
  int pos = block_exclusive_scan<NT>(mine, wsum, et, bar, &kept);
#pragma unroll
  for (int j = 0; j < 4 * MQ; ++j) {
    if (v[j] != 0 && v[j] >= floor) {
      if (pos < 4 * capq) row[static_cast<size_t>(pos & 3) * capq + (pos >> 2)] = v[j];
      ++pos;
    }
  }
  kept = min(kept, 4 * capq);
  if (et < 4) cnt[et] = (kept + 3 - et) / 4;
  return kept;
}

// Rank the selected keys of one row and write its token indices, inside the
// kernel that selected them: the keys v[i] != 0 && v[i] >= floor (at most K
// over the NT cooperating threads) are compacted into `srt` (shared memory,
// P = the power of two >= K keys), padded with empty keys (0) and sorted into
// descending 64-bit order (score descending, then index ascending) by a
// bitonic network; dst[0..K) gets their token indices and -1 past them.
// With P == 4 * NT each thread keeps four consecutive keys in registers:
// strides 1 and 2 stay in the thread, strides 4..64 are warp shuffles and
// only strides >= 128 go through shared memory. Group barrier `bar` over the
// NT threads; wsum as for block_exclusive_scan. Writes stay inside srt and
// dst even if the group aborted and the positions are stale.
template <int NT, int M>
__device__ __forceinline__ void sort_selected_to_idx(const uint64_t (&v)[M], uint64_t floor, uint64_t* srt, int* wsum,
                                                     int et, const GroupBar& bar, int K, int32_t* __restrict__ dst) {
  int mine = 0;
#pragma unroll
  for (int i = 0; i < M; ++i) mine += (v[i] != 0 && v[i] >= floor) ? 1 : 0;
  int kept = 0;
  int pos = block_exclusive_scan<NT>(mine, wsum, et, bar, &kept);
#pragma unroll
  int P = 1;
  while (P < K) P <<= 1;
#pragma unroll
  for (int i = 0; i < M; ++i)
    if (v[i] != 0 && v[i] >= floor) {
      if (pos < P) srt[pos] = v[i];
      ++pos;
    }
  for (int i = max(kept, 0) + et; i < P; i += NT) srt[i] = 0ull;
  bar.sync();
  if (P == 4 * NT) {
    uint64_t a[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) a[u] = srt[4 * et + u];
#pragma unroll 1
    for (int k = 2; k <= P; k <<= 1) {
#pragma unroll 1
      for (int j = k >> 1; j > 0; j >>= 1) {
        if (j >= 128) {  // the partner sits in another warp
          bar.sync();  // every thread has read what the last exchange wrote
#pragma unroll
          for (int u = 0; u < 4; ++u) srt[4 * et + u] = a[u];
          bar.sync();
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int e = 4 * et + u;
            const uint64_t b = srt[e ^ j];
            const bool keep_max = ((e & j) == 0) == ((e & k) == 0);
            a[u] = keep_max ? (a[u] > b ? a[u] : b) : (a[u] > b ? b : a[u]);
          }
        } else if (j >= 4) {  // the partner is lane (et ^ j/4) of this warp
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int e = 4 * et + u;
            const uint64_t b = __shfl_xor_sync(0xffffffffu, a[u], j >> 2);
            const bool keep_max = ((e & j) == 0) == ((e & k) == 0);
            a[u] = keep_max ? (a[u] > b ? a[u] : b) : (a[u] > b ? b : a[u]);
          }
        } else {  // both keys are this thread's
          // for k >= 4 the direction bit (e & k) is the same for the four keys
          // 4et..4et+3; for k = 2 the pairs (0,1) and (2,3) run opposite ways
          const bool desc = ((4 * et) & k) == 0;
          auto cx = [&](uint64_t& lo, uint64_t& hi, bool d) {
            const uint64_t mx = lo > hi ? lo : hi, mn = lo > hi ? hi : lo;
            lo = d ? mx : mn;
            hi = d ? mn : mx;
          };
          if (j == 2) {
            cx(a[0], a[2], desc);
            cx(a[1], a[3], desc);
          } else if (k == 2) {
            cx(a[0], a[1], true);
            cx(a[2], a[3], false);
          } else {
            cx(a[0], a[1], desc);
            cx(a[2], a[3], desc);
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = 4 * et + u;
      if (e < K) dst[e] = (a[u] == 0ull) ? -1 : rank_key_index(a[u]);
    }
  } else {
#pragma unroll 1
    for (int k = 2; k <= P; k <<= 1) {
#pragma unroll 1
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int i = et; i < P / 2; i += NT) {
          const int lo = 2 * i - (i & (j - 1));
          const int hi = lo + j;
          const bool desc = (lo & k) == 0;
          const uint64_t a = srt[lo], b = srt[hi];
          if ((a < b) == desc) {
            srt[lo] = b;
            srt[hi] = a;
          }
        }
        bar.sync();
      }
    }
    for (int i = et; i < K; i += NT) dst[i] = (srt[i] == 0ull) ? -1 : rank_key_index(srt[i]);
  }
}

}  // namespace dsa
