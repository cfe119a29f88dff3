// Decode lightning indexer: B sequences, one new query token each, scored
// against that sequence's cached FP8 keys, then an exact per-sequence top-k.
//
// Same score as the prefill indexer ("Lightning Indexer 的计算过程", step 3,
// adg.csdn.net/695234...), for the single row t = lens[b]-1:
//     I[b,s] = q_scale[b] * k_scale[b,s] * sum_j w[b,j] * ReLU(q8[b,j,:] . k8[b,s,:]),  s < lens[b].
// The decode cost curve of "DeepSeek-V3.2-Exp" (adg.csdn.net/695234..., figure
// (b) Decoding) is the regime here: one query per sequence, so the work is a
// single pass over the key cache and HBM bandwidth is the bound.
//
// Scoring kernel: persistent CTAs (two per SM) walk contiguous ranges of
// (sequence, 1024-key chunk) items. For each item the query is loaded once,
// its 8 key tiles stream through a 4-stage TMA ring, each tile is multiplied
// against the [H_I x d_I] query on the tensor core (M = 128 keys, N = H_I
// heads) and the epilogue reduces the heads per key, writing one fp32 score
// per key and counting its 11-bit bin in a shared histogram that is added to
// the sequence's global histogram when the CTA moves to another sequence.
//
// Selection kernel: one CTA per sequence runs an exact radix select over the
// 64-bit ranking keys (score, then lower index) of its scores, then ranks the
// selected keys in shared memory and writes the sequence's index row.
#pragma once

#include "dsa_common.cuh"
#include "topk_select.cuh"

namespace dsa {

template <int HI, int DI>
struct IdxDecodeCfg {
  static constexpr int BM = 128;
  static constexpr int CHUNK = 1024;           // keys per CTA
  static constexpr int NKT = CHUNK / BM;
  static constexpr int KST = 4;
  static constexpr int NACC = 2;
  static constexpr int QBYTES = HI * DI;
  static constexpr int KTILE_BYTES = BM * DI;
  static constexpr int NTHREADS = 6 * 32;      // producer, MMA, 4 epilogue warps
  static constexpr SwizzleMode SW = (DI == 128) ? kSw128 : kSw64;
  static constexpr uint32_t SBO = 8 * DI;
  static constexpr uint32_t IDESC = instr_desc(kFmtE4M3, 128, HI, false, false);
  static constexpr int KSTEPS = DI / 32;
  static constexpr int TMEM_COLS = 128;        // 2 x HI (<= 128) rounded to a power of two >= 32
  static constexpr int OFF_K = 0;
  static constexpr int OFF_Q = OFF_K + KST * KTILE_BYTES;
  static constexpr int QPAD = ((QBYTES + 1023) / 1024) * 1024;
  static constexpr int OFF_W = OFF_Q + 2 * QPAD;  // two query buffers: the next item's loads early
  static constexpr int OFF_HIST = OFF_W + HI * 4;         // u32 [2048] per-CTA histogram
  static constexpr int OFF_BAR = OFF_HIST + 2048 * 4;
  static constexpr int NBAR = 4 + 2 * KST + 2 * NACC;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int MAX_ITEM_PAGES = CHUNK / 16;  // pages one item touches at the smallest page size
  static constexpr int OFF_PG = OFF_MISC + 16;       // i32 [MAX_ITEM_PAGES]: paged producer's staged pages
  static constexpr int SMEM_BYTES = OFF_PG + MAX_ITEM_PAGES * 4 + 1024;
  static_assert(HI % 16 == 0 && HI <= 64, "decode indexer: H_I must be 16, 32, 48 or 64");
};

struct IdxDecodeParams {
  const float* q_scale;  // [B]
  const float* w;        // [B, HI]
  const float* k_scale;  // [B, L_max]
  const int32_t* lens;   // [B]
  int L_max;
  int B;
  float* scores;         // [B, L_max]; entries s >= lens[b] untouched
  uint32_t* hist;        // [B, 2048] counts of the top 11 bits of each ranking key, or null
  // paged key cache (paged instance only): key s of sequence b is pool row
  // block_table[b * bt_stride + (s >> page_shift)] * page + (s & (page - 1));
  // k_scale is then indexed by pool row; the pool holds pool_pages pages
  const int32_t* block_table;
  int bt_stride, page_shift, pool_pages;
};

// Pool row of key s of sequence b in a paged cache, or -1 when its page entry
// lies outside the pool.
__device__ __forceinline__ int paged_key_row(const IdxDecodeParams& p, int b, int s) {
  const int page = p.block_table[static_cast<long long>(b) * p.bt_stride + (s >> p.page_shift)];
  if (page < 0 || page >= p.pool_pages) return -1;
  return (page << p.page_shift) + (s & ((1 << p.page_shift) - 1));
}

// Bin of a ranking key in the 2048-bin histogram: its top 11 bits (sign,
// exponent and the top two mantissa bits of the score).
__device__ __forceinline__ uint32_t key_bin11(uint64_t key) { return static_cast<uint32_t>(key >> 53); }

template <int HI, int DI, bool kPaged>
__global__ void __launch_bounds__(IdxDecodeCfg<HI, DI>::NTHREADS, 2)
    indexer_decode_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const IdxDecodeParams p) {
  using C = IdxDecodeCfg<HI, DI>;
  griddep_launch_dependents();  // the selection may be scheduled now; it waits for this grid
  // Persistent: work item i is chunk i % nch of sequence i / nch; each CTA
  // takes a contiguous range of items (so its sequence rarely changes) and
  // keeps its barriers, TMEM and ring phases from one item to the next.
  const int nch = (p.L_max + C::CHUNK - 1) / C::CHUNK;
  const int total = p.B * nch;
  const int per = (total + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
  const int it0 = static_cast<int>(blockIdx.x) * per;
  const int it1 = min(total, it0 + per);
  if (it0 >= it1) return;  // whole CTA, before any barrier or TMEM allocation

  // 1024-byte aligned base, derived from the shared array by an offset so
  // the compiler keeps every access in the shared address space
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* k_s = smem + C::OFF_K;
  uint8_t* q_s = smem + C::OFF_Q;
  float* w_s = reinterpret_cast<float*>(smem + C::OFF_W);
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + C::OFF_HIST);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;      // [2]
  uint64_t* q_empty = bars + 2;  // [2]
  uint64_t* k_full = bars + 4;
  uint64_t* k_empty = bars + 4 + C::KST;
  uint64_t* acc_full = bars + 4 + 2 * C::KST;
  uint64_t* acc_empty = bars + 4 + 2 * C::KST + C::NACC;
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  int* abort_s = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);
  const AbortFlag ab{abort_s};
  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();

  if (threadIdx.x == 0) {
    *abort_s = 0;
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full + i, 1);
      mbar_init(q_empty + i, 1);
    }
    for (int i = 0; i < C::KST; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 1);
    }
    for (int i = 0; i < C::NACC; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, 4);
    }
    fence_mbar_init();
  }
  if (p.hist)
    for (int i = threadIdx.x; i < 2048; i += blockDim.x) hist_s[i] = 0;
  if (warp == 1) tmem_alloc(tmem_base_s, C::TMEM_COLS);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_s;

  // sequence, first key, key tiles and length of item `it`; false when the
  // chunk starts past the sequence's length (the same answer on every role)
  auto item = [&](int it, int& b, int& s0, int& nkt, int& n) {
    b = it / nch;
    s0 = (it % nch) * C::CHUNK;
    n = min(p.lens[b], p.L_max);
    if (s0 >= n) return false;
    nkt = min(C::NKT, (n - s0 + C::BM - 1) / C::BM);
    return true;
  };

  if (warp == 0) {
    // the keys stream through once: let them leave L2 first, so the scores
    // this kernel writes are still there for the selection that reads them
    const uint64_t kpol = l2_evict_first();
    if constexpr (kPaged) {
      // Paged producer: the whole warp first stages the pool row of the first
      // key of every page the item touches (one round trip for all of them),
      // then lane 0 issues the boxes: R = min(page, BM) rows per box. A box past
      // the sequence or behind a bad page entry starts outside the pool and
      // lands as zeros (its bytes still count).
      int* pg_s = reinterpret_cast<int*>(smem + C::OFF_PG);
      const int shift = p.page_shift;
      const int R = min(1 << shift, C::BM);
      const int oob = p.pool_pages << shift;
      int g = 0;   // key tiles issued so far (ring position and phase)
      int qn = 0;  // query loads issued so far
      bool ok = true;
      for (int it = it0; it < it1 && ok; ++it) {
        int b, s0, nkt, n;
        if (!item(it, b, s0, nkt, n)) continue;
        const int fp = s0 >> shift;                                     // first page of the item
        const int npg = ((min(s0 + nkt * C::BM, n) - 1) >> shift) - fp + 1;  // <= MAX_ITEM_PAGES
        __syncwarp();  // lane 0 is done with the previous item's entries
        for (int j = static_cast<int>(lane); j < npg; j += 32) {
          const int page = p.block_table[static_cast<long long>(b) * p.bt_stride + fp + j];
          const bool bad = page < 0 || page >= p.pool_pages;
          if (bad) set_device_error(kErrBadIndex, 2);
          pg_s[j] = bad ? -1 : (page << shift);
        }
        __syncwarp();
        if (lane == 0) {
          const int qb = qn & 1;
          if (!mbar_wait(q_empty + qb, ((qn >> 1) & 1) ^ 1, ab, 10)) ok = false;
          if (ok) {
            mbar_arrive_expect_tx(q_full + qb, C::QBYTES);
            tma_load_2d(q_s + qb * C::QPAD, &tmQ, q_full + qb, 0, b * HI);
            ++qn;
          }
          for (int kt = 0; kt < nkt && ok; ++kt, ++g) {
            const int slot = g % C::KST;
            if (!mbar_wait(k_empty + slot, ((g / C::KST) & 1) ^ 1, ab, 11)) { ok = false; break; }
            mbar_arrive_expect_tx(k_full + slot, C::KTILE_BYTES);
            for (int i = 0; i < C::BM; i += R) {
              const int sk = s0 + kt * C::BM + i;
              int prow = oob;
              if (sk < n) {
                const int base = pg_s[(sk >> shift) - fp];
                if (base >= 0) prow = base + (sk & ((1 << shift) - 1));
              }
              tma_load_2d_hint(k_s + slot * C::KTILE_BYTES + i * DI, &tmK, k_full + slot, 0, prow, kpol);
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      }
      // wait until the MMA has consumed every issued tile (copies landed)
      if (lane == 0)
        for (int gg = max(0, g - C::KST); gg < g && !ab.raised(); ++gg)
          mbar_wait(k_empty + gg % C::KST, (gg / C::KST) & 1, ab, 12);
    } else if (lane == 0) {
      int g = 0;   // key tiles issued so far (ring position and phase)
      int qn = 0;  // query loads issued so far
      for (int it = it0; it < it1; ++it) {
        int b, s0, nkt, n;
        if (!item(it, b, s0, nkt, n)) continue;
        // query buffer qn & 1: the MMA has finished with the item two back
        const int qb = qn & 1;
        if (!mbar_wait(q_empty + qb, ((qn >> 1) & 1) ^ 1, ab, 10)) break;
        mbar_arrive_expect_tx(q_full + qb, C::QBYTES);
        tma_load_2d(q_s + qb * C::QPAD, &tmQ, q_full + qb, 0, b * HI);
        ++qn;
        const int row0 = b * p.L_max + s0;  // B * L_max < 2^31 (checked on the host)
        bool ok = true;
        for (int kt = 0; kt < nkt; ++kt, ++g) {
          const int slot = g % C::KST;
          if (!mbar_wait(k_empty + slot, ((g / C::KST) & 1) ^ 1, ab, 11)) { ok = false; break; }
          mbar_arrive_expect_tx(k_full + slot, C::KTILE_BYTES);
          tma_load_2d_hint(k_s + slot * C::KTILE_BYTES, &tmK, k_full + slot, 0, row0 + kt * C::BM, kpol);
        }
        if (!ok) break;
      }
      // wait until the MMA has consumed every issued tile (copies landed)
      for (int gg = max(0, g - C::KST); gg < g && !ab.raised(); ++gg)
        mbar_wait(k_empty + gg % C::KST, (gg / C::KST) & 1, ab, 12);
    }
  } else if (warp == 1) {
    // the warp waits converged; one elected lane issues and commits
    int g = 0;
    int qn = 0;
    bool ok = true;
    for (int it = it0; it < it1 && ok; ++it) {
      int b, s0, nkt, n;
      if (!item(it, b, s0, nkt, n)) continue;
      const int qb = qn & 1;
      if (!mbar_wait_warp(q_full + qb, (qn >> 1) & 1, ab, 13)) break;
      ++qn;
      const uint32_t q_addr = smem_u32(q_s + qb * C::QPAD);
      for (int kt = 0; kt < nkt; ++kt, ++g) {
        const int slot = g % C::KST;
        const int buf = g % C::NACC;
        if (!mbar_wait_warp(k_full + slot, (g / C::KST) & 1, ab, 14)) { ok = false; break; }
        if (!mbar_wait_warp(acc_empty + buf, ((g / C::NACC) & 1) ^ 1, ab, 15)) { ok = false; break; }
        tc_fence_after();
        if (elect_one()) {
          const uint32_t a_addr = smem_u32(k_s + slot * C::KTILE_BYTES);
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk) {
            const uint64_t ad = smem_desc(a_addr + kk * 32, 16, C::SBO, C::SW);
            const uint64_t bd = smem_desc(q_addr + kk * 32, 16, C::SBO, C::SW);
            mma_f8(tmem + buf * HI, ad, bd, C::IDESC, kk > 0 ? 1u : 0u);
          }
          tc_commit(acc_full + buf);
          tc_commit(k_empty + slot);
          if (kt == nkt - 1) tc_commit(q_empty + qb);  // this item's query buffer may be reused
        }
        __syncwarp();
      }
    }
  } else {
    const int quarter = static_cast<int>(warp & 3);
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const int et = static_cast<int>(threadIdx.x) - 64;  // 0..127
    // add this CTA's counts of sequence bq to the global histogram, zeroing them
    auto flush_hist = [&](int bq) {
      for (int i = et; i < 2048; i += 128) {
        const uint32_t c = hist_s[i];
        if (c) {
          atomicAdd(p.hist + static_cast<size_t>(bq) * 2048 + i, c);
          hist_s[i] = 0;
        }
      }
    };
    int g = 0;
    int cur_b = -1;
    bool ok = true;
    const GroupBar bar{1, 128, ab};  // the four epilogue warps (abort-safe: see GroupBar)
    // Per-key scales of an item's tiles (this thread's key in each), loaded one
    // item ahead so their DRAM latency hides behind a whole item.
    auto load_scales = [&](int it, float (&ks)[C::NKT]) {
      int b, s0, nkt, n;
      const bool v = it < it1 && item(it, b, s0, nkt, n);
#pragma unroll
      for (int kt = 0; kt < C::NKT; ++kt) {
        ks[kt] = 0.f;
        if (v && kt < nkt) {
          const int s = s0 + kt * C::BM + quarter * 32 + static_cast<int>(lane);
          if constexpr (kPaged) {
            const int r = (s < n) ? paged_key_row(p, b, s) : -1;
            if (r >= 0) ks[kt] = __ldg(p.k_scale + r);
          } else {
            if (s < n) ks[kt] = __ldg(p.k_scale + static_cast<size_t>(b) * p.L_max + s);
          }
        }
      }
    };
    float ks_cur[C::NKT], ks_nxt[C::NKT];
    load_scales(it0, ks_nxt);
    for (int it = it0; it < it1 && ok; ++it) {
#pragma unroll
      for (int kt = 0; kt < C::NKT; ++kt) ks_cur[kt] = ks_nxt[kt];
      load_scales(it + 1, ks_nxt);
      int b, s0, nkt, n;
      if (!item(it, b, s0, nkt, n)) continue;
      if (b != cur_b) {
        if (!bar.sync()) { ok = false; break; }  // the previous sequence's weights and counts are done with
        if (p.hist && cur_b >= 0) flush_hist(cur_b);
        for (int i = et; i < HI; i += 128) w_s[i] = p.w[static_cast<size_t>(b) * HI + i];
        if (!bar.sync()) { ok = false; break; }
        cur_b = b;
      }
      const float qs = p.q_scale[b];
#pragma unroll 1
      for (int kt = 0; kt < nkt; ++kt, ++g) {
        const int buf = g % C::NACC;
        const int s = s0 + kt * C::BM + quarter * 32 + static_cast<int>(lane);
        float ks = ks_cur[0];
#pragma unroll
        for (int u = 1; u < C::NKT; ++u) ks = (kt == u) ? ks_cur[u] : ks;  // no dynamic register indexing
        if (!mbar_wait(acc_full + buf, (g / C::NACC) & 1, ab, 16)) { ok = false; break; }
        tc_fence_after();
        // eight independent partial sums (head j to sum j % 8), added in a
        // fixed order: a single running sum would be a 64-deep dependent chain
        float part[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if constexpr (HI % 32 == 0) {
#pragma unroll
          for (int h = 0; h < HI / 32; ++h) {
            uint32_t r[32];
            tmem_ld32(tmem + lane_addr + buf * HI + h * 32, r);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              part[j & 7] = __fmaf_rn(w_s[h * 32 + j], fmaxf(__uint_as_float(r[j]), 0.f), part[j & 7]);
          }
        } else {
          uint32_t r[16];
          tmem_ld16(tmem + lane_addr + buf * HI, r);
#pragma unroll
          for (int j = 0; j < 16; ++j)
            part[j & 7] = __fmaf_rn(w_s[j], fmaxf(__uint_as_float(r[j]), 0.f), part[j & 7]);
        }
        const float acc = ((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7]));
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty + buf);
        if (s < n) {
          const float score = __fmul_rn(__fmul_rn(acc, qs), ks);
          p.scores[static_cast<size_t>(b) * p.L_max + s] = score;
          if (p.hist) atomicAdd(hist_s + key_bin11(rank_key(score, static_cast<uint32_t>(s))), 1u);
        }
      }
    }
    if (ok && p.hist && cur_b >= 0 && bar.sync()) flush_hist(cur_b);
    if (bar.aborted()) bar.leave();  // count this warp in at the barrier the others may wait at
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Exact top-k of one sequence's scores (one CTA of kThreads per sequence).
// With the scoring kernel's 2048-bin histogram of ranking keys (top 11 bits),
// the bin holding the k-th largest key is known before reading any score:
// one pass writes every key above that bin straight to the output and keeps
// the bin's own keys in shared memory, where an exact radix select picks the
// rest. Without a histogram (or if the bin overflows the shared buffer) the
// kernel counts the histogram itself / falls back to multi-pass selection
// over global memory. Writes the k best keys of sequence b (unordered, 0
// where lens[b] < k) to sel_keys[b, 0..k).
constexpr int kDecodeSelThreads = 1024;
constexpr int kDecodeSelBinCap = 16384;  // boundary-bin keys kept in shared memory (128 KB)

__device__ __forceinline__ void decode_select_body(const float* __restrict__ scores, const int32_t* __restrict__ lens,
                                                   int L_max, int K, const uint32_t* __restrict__ hist_in,
                                                   uint64_t* __restrict__ sel_keys, int b) {
  constexpr int NT = kDecodeSelThreads;
  extern __shared__ __align__(16) uint8_t dsmem[];
  uint64_t* bin_keys = reinterpret_cast<uint64_t*>(dsmem);                          // [kDecodeSelBinCap]
  int* hist = reinterpret_cast<int*>(dsmem + kDecodeSelBinCap * 8);                 // [2048]
  int* scr = hist + 2048;                                                            // select scratch
  __shared__ int wsum[32];
  __shared__ int res[4];
  __shared__ int wpos, bpos;
  const int n = min(lens[b], L_max);
  const float* sc = scores + static_cast<size_t>(b) * L_max;
  uint64_t* dst = sel_keys + static_cast<size_t>(b) * K;
  const int tid = threadIdx.x;
  if (n <= K) {
    for (int i = tid; i < K; i += NT) dst[i] = (i < n) ? rank_key(sc[i], static_cast<uint32_t>(i)) : 0ull;
    return;
  }
  // 1. the 2048-bin histogram
  if (hist_in) {
    for (int i = tid; i < 2048; i += NT) hist[i] = static_cast<int>(hist_in[static_cast<size_t>(b) * 2048 + i]);
  } else {
    for (int i = tid; i < 2048; i += NT) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += NT) atomicAdd(hist + key_bin11(rank_key(sc[i], static_cast<uint32_t>(i))), 1);
  }
  if (tid == 0) {
    wpos = 0;
    bpos = 0;
  }
  __syncthreads();
  // 2. bin of the K-th largest key: descending scan, 2 bins per thread
  {
    const int c0 = hist[2047 - 2 * tid], c1 = hist[2046 - 2 * tid];
    const int tot = c0 + c1;
    const int l = tid & 31, w = tid >> 5;
    int incl = tot;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (l >= off) incl += y;
    }
    if (l == 31) wsum[w] = incl;
    __syncthreads();
    int wbase = 0;
    for (int i = 0; i < w; ++i) wbase += wsum[i];
    const int excl = wbase + incl - tot;
    if (excl < K && excl + tot >= K) {
      if (excl + c0 >= K) {
        res[0] = 2047 - 2 * tid; res[1] = excl; res[2] = c0;
      } else {
        res[0] = 2046 - 2 * tid; res[1] = excl + c0; res[2] = c1;
      }
    }
    __syncthreads();
  }
  const uint32_t dbin = static_cast<uint32_t>(res[0]);
  const int above = res[1], inb = res[2];
  const int need = K - above;  // keys to take from the boundary bin (1..inb)
  // 3. one pass: keys above the bin go out; the bin's keys are kept
  const bool fits = inb <= kDecodeSelBinCap;
  // Each thread takes 4 consecutive keys per round (one 16-byte load when
  // the rows are 16-byte aligned); a warp scan of the per-thread counts
  // gives every thread its write positions, one shared atomic per warp and
  // destination.
  const int lane = tid & 31;
  const bool vec = ((L_max & 3) == 0) && ((reinterpret_cast<uintptr_t>(scores) & 15) == 0);
  const int nround = (n + 4 * NT - 1) / (4 * NT);  // same trip count on every lane
  for (int rd = 0; rd < nround; ++rd) {
    const int i0 = 4 * (rd * NT + tid);
    float f[4];
    if (vec && i0 + 3 < n) {
      const float4 x = *reinterpret_cast<const float4*>(sc + i0);
      f[0] = x.x; f[1] = x.y; f[2] = x.z; f[3] = x.w;
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) f[u] = (i0 + u < n) ? sc[i0 + u] : 0.f;
    }
    uint64_t key[4];
    uint32_t hi = 0, eq = 0;  // bit u: key u goes out / is kept for the bin
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      key[u] = rank_key(f[u], static_cast<uint32_t>(i0 + u));
      const uint32_t bin = key_bin11(key[u]);
      const bool in = i0 + u < n;
      hi |= (in && bin > dbin) ? (1u << u) : 0u;
      eq |= (in && bin == dbin && fits) ? (1u << u) : 0u;
    }
    // counts packed as (eq << 16) | hi; inclusive warp scan
    const int mine = __popc(hi) | (__popc(eq) << 16);
    int incl = mine;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    int base = 0;
    if (lane == 31 && incl != 0) {
      const int th = incl & 0xffff, te = incl >> 16;
      base = (th ? atomicAdd(&wpos, th) : 0) | ((te ? atomicAdd(&bpos, te) : 0) << 16);
    }
    base = __shfl_sync(0xffffffffu, base, 31);
    int ph = (base & 0xffff) + ((incl - mine) & 0xffff);
    int pe = (base >> 16) + ((incl - mine) >> 16);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if ((hi >> u) & 1u) dst[ph++] = key[u];
      if ((eq >> u) & 1u) bin_keys[pe++] = key[u];
    }
  }
  __syncthreads();
  // 4. exact choice of `need` keys inside the boundary bin
  if (fits) {
    uint64_t v[kDecodeSelBinCap / NT];
#pragma unroll
    for (int j = 0; j < kDecodeSelBinCap / NT; ++j) {
      const int i = tid + j * NT;
      v[j] = (i < inb) ? bin_keys[i] : 0ull;
    }
    uint64_t floor = 1ull;
    // no bounded waits in this kernel: the group barrier never sees an abort
    __shared__ int never_aborts;
    if (tid == 0) never_aborts = 0;
    __syncthreads();
    const GroupBar bar{1, NT, AbortFlag{&never_aborts}};
    if (need < inb) floor = radix_select_floor<NT, kDecodeSelBinCap / NT>(v, need, scr, tid, bar);
#pragma unroll
    for (int j = 0; j < kDecodeSelBinCap / NT; ++j)
      if (v[j] != 0 && v[j] >= floor) dst[atomicAdd(&wpos, 1)] = v[j];
    return;
  }
  // the boundary bin is too large for shared memory: radix select over the
  // bin's keys in global memory, 8-bit digits below the 11-bit bin, then 5
  uint64_t prefix = static_cast<uint64_t>(dbin) << 53;
  int remaining = need;
  for (int shift = 45; shift >= 0; shift = (shift >= 13) ? shift - 8 : (shift == 5 ? 0 : -1)) {
    const int width = (shift == 0) ? 5 : 8;
    for (int i = tid; i < 256; i += NT) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += NT) {
      const uint64_t x = rank_key(sc[i], static_cast<uint32_t>(i));
      if ((x >> (shift + width)) == (prefix >> (shift + width)))
        atomicAdd(&hist[(x >> shift) & ((1u << width) - 1u)], 1);
    }
    __syncthreads();
    if (tid < 32) {
      int c[8];
      int tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = hist[255 - 8 * tid - i];
        tot += c[i];
      }
      int incl = tot;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (tid >= off) incl += y;
      }
      const uint32_t ball = __ballot_sync(0xffffffffu, incl >= remaining);
      if (tid == __ffs(ball) - 1) {
        int cum = incl - tot;
        for (int i = 0; i < 8; ++i) {
          if (cum + c[i] >= remaining) {
            res[0] = 255 - 8 * tid - i;
            res[1] = cum;
            res[2] = c[i];
            break;
          }
          cum += c[i];
        }
      }
    }
    __syncthreads();
    const int d = res[0], ab = res[1], ib = res[2];
    remaining -= ab;
    prefix |= static_cast<uint64_t>(d) << shift;
    __syncthreads();
    if (ib == remaining) break;
  }
  // keys of the bin that are >= prefix
  for (int i = tid; i < n; i += NT) {
    const uint64_t x = rank_key(sc[i], static_cast<uint32_t>(i));
    if (key_bin11(x) == dbin && x >= prefix) dst[atomicAdd(&wpos, 1)] = x;
  }
}

// The k selected keys of one sequence in ranked order: a bitonic sort of the
// keys (padded with 0 to a power of two <= 2048) in shared memory into
// descending 64-bit order (score descending, then index ascending), written
// as token indices, -1 for padding keys.
template <int NT>
__device__ __forceinline__ void sort_keys_to_idx(uint64_t* s, const uint64_t* src, int K, int32_t* out) {
  const int tid = threadIdx.x;
  int P = 1;
  while (P < K) P <<= 1;
  for (int i = tid; i < P; i += NT) s[i] = (i < K) ? src[i] : 0ull;
  __syncthreads();
  for (int k = 2; k <= P; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < P; i += NT) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint64_t a = s[i], c = s[ixj];
          // blocks with (i & k) == 0 run descending; the last stage (k = P) is all descending
          if (((i & k) == 0) ? (a < c) : (a > c)) {
            s[i] = c;
            s[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < K; i += NT) out[i] = (s[i] == 0ull) ? -1 : rank_key_index(s[i]);
}

// Largest histogram bin the decode ranking scans key by key.
constexpr int kDecodeBinRankMax = 256;

// The fast path of the decode selection: the candidates (keys in bins above
// the boundary bin of the scoring kernel's 11-bit histogram, plus the
// boundary bin's own keys) are gathered in shared memory and ranked by one
// finer histogram pass (topk_rank_by_bins), which writes the sequence's
// index row. False when the boundary bin is too large for shared memory or a
// finer bin is too crowded; nothing is written to idx then.
//
// kPair: the two CTAs of a cluster share the sequence (blockIdx.x / 2, the
// scoring kernel's histogram required): each takes half of the pass over
// the scores and appends its candidates to CTA 0's shared memory (cluster
// atomics and stores), and CTA 0 ranks. Both CTAs reach the same decisions
// (same histogram), so they leave before the cluster barriers together when
// the fast path does not apply; CTA 1 returns true without writing anything
// (CTA 0 writes the row).
template <bool kPair>
__device__ __forceinline__ bool decode_rank_fast(const float* __restrict__ scores, const int32_t* __restrict__ lens,
                                                 int L_max, int K, const uint32_t* __restrict__ hist_in,
                                                 int32_t* __restrict__ idx) {
  constexpr int NT = kDecodeSelThreads;
  constexpr int NV = (2048 + kDecodeSelBinCap) / NT;  // candidate slots per thread
  extern __shared__ __align__(16) uint8_t dsmem[];
  uint64_t* bin_keys = reinterpret_cast<uint64_t*>(dsmem);  // [kDecodeSelBinCap]; the ranking buffer afterwards
  uint64_t* abv = bin_keys + kDecodeSelBinCap;              // [2048] keys above the boundary bin
  int* hist = reinterpret_cast<int*>(abv + 2048);           // [2048]
  int* start = hist + 2048;                                 // [2048]
  int* small = start + 2048;                                // [64]
  __shared__ int wsum[32];
  __shared__ int res[4];
  __shared__ int npos;  // slots taken: keys above the bin (low 16 bits), the bin's keys (high 16)
  __shared__ int never_aborts;  // no bounded waits in this kernel
  const int b = kPair ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const uint32_t crank = kPair ? cluster_ctarank() : 0u;
  const int n = min(lens[b], L_max);
  const float* sc = scores + static_cast<size_t>(b) * L_max;
  int32_t* out = idx + static_cast<size_t>(b) * K;
  const int tid = threadIdx.x;
  if (tid == 0) {
    never_aborts = 0;
    npos = 0;
  }
  const GroupBar bar{1, NT, AbortFlag{&never_aborts}};
  if (n <= K) {  // every key is selected: rank them all (K <= 2048 = 2 per thread)
    if (kPair && crank != 0) return true;
    uint64_t v[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int i = tid + j * NT;
      v[j] = (i < n) ? rank_key(sc[i], static_cast<uint32_t>(i)) : 0ull;
    }
    __syncthreads();
    return topk_rank_by_bins<NT, 2>(v, K, hist, start, small, bin_keys, kDecodeSelBinCap, kDecodeBinRankMax, tid,
                                    bar, out);
  }
  // 1. the scoring kernel's 2048-bin histogram of the top 11 key bits
  if (hist_in) {
    for (int i = tid; i < 2048; i += NT) hist[i] = static_cast<int>(hist_in[static_cast<size_t>(b) * 2048 + i]);
  } else {
    for (int i = tid; i < 2048; i += NT) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += NT) atomicAdd(hist + key_bin11(rank_key(sc[i], static_cast<uint32_t>(i))), 1);
  }
  __syncthreads();
  // 2. the bin of the K-th largest key: descending scan, 2 bins per thread
  {
    const int c0 = hist[2047 - 2 * tid], c1 = hist[2046 - 2 * tid];
    const int tot = c0 + c1;
    const int l = tid & 31, w = tid >> 5;
    int incl = tot;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (l >= off) incl += y;
    }
    if (l == 31) wsum[w] = incl;
    __syncthreads();
    int wbase = 0;
    for (int i = 0; i < w; ++i) wbase += wsum[i];
    const int excl = wbase + incl - tot;
    if (excl < K && excl + tot >= K) {
      if (excl + c0 >= K) {
        res[0] = 2047 - 2 * tid; res[1] = excl; res[2] = c0;
      } else {
        res[0] = 2046 - 2 * tid; res[1] = excl + c0; res[2] = c1;
      }
    }
    __syncthreads();
  }
  const uint32_t dbin = static_cast<uint32_t>(res[0]);
  const int above = res[1], inb = res[2];
  if (inb > kDecodeSelBinCap || above > 2048) return false;
  // a pair appends into CTA 0's buffers (addresses mapped where used) once
  // its counter is set up
  if constexpr (kPair) cluster_sync_all();
  // 3. one pass over the scores: keys above the bin and the bin's keys to
  //    shared memory (4 keys per thread per round). The loads of PF rounds
  //    are issued together so their latencies overlap, and a warp reserves
  //    space for all PF rounds with one shared atomic: keys above the bin
  //    count in the low 16 bits of `pos`, the bin's keys in the high 16
  //    (above <= 2048 and inb <= kDecodeSelBinCap were checked, so neither
  //    field overflows).
  const int lane = tid & 31;
  const bool vec = ((L_max & 3) == 0) && ((reinterpret_cast<uintptr_t>(scores) & 15) == 0);
  const int nround = (n + 4 * NT - 1) / (4 * NT);
  // a pair: CTA 0 takes rounds [0, h), CTA 1 rounds [h, nround)
  const int rhalf = (nround + 1) / 2;
  const int rbeg = (kPair && crank != 0) ? rhalf : 0;
  const int rend = kPair ? (crank != 0 ? nround : rhalf) : nround;
  // rounds past rend read nothing (their i0 is pushed past n)
  auto first_key = [&](int rd) { return rd < rend ? 4 * (rd * NT + tid) : n; };
  constexpr int PF = 4;
  for (int rd0 = rbeg; rd0 < rend; rd0 += PF) {
    float f[PF][4];
#pragma unroll
    for (int q = 0; q < PF; ++q) {
      const int i0 = first_key(rd0 + q);
      if (vec && i0 + 3 < n) {
        const float4 x = *reinterpret_cast<const float4*>(sc + i0);
        f[q][0] = x.x; f[q][1] = x.y; f[q][2] = x.z; f[q][3] = x.w;
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) f[q][u] = (i0 + u < n) ? sc[i0 + u] : 0.f;
      }
    }
    uint32_t hi[PF], eq[PF];
    int excl[PF];  // this lane's first slot of round q within the warp's batch (both fields)
    int wtot = 0;  // the warp's keys of the batch (both fields)
#pragma unroll
    for (int q = 0; q < PF; ++q) {
      const int i0 = first_key(rd0 + q);
      hi[q] = 0;
      eq[q] = 0;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t bin = key_bin11(rank_key(f[q][u], static_cast<uint32_t>(i0 + u)));
        const bool in = i0 + u < n;
        hi[q] |= (in && bin > dbin) ? (1u << u) : 0u;
        eq[q] |= (in && bin == dbin) ? (1u << u) : 0u;
      }
      const int mine = __popc(hi[q]) | (__popc(eq[q]) << 16);
      int incl = mine;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      excl[q] = wtot + incl - mine;
      wtot += __shfl_sync(0xffffffffu, incl, 31);
    }
    int base = 0;
    if (lane == 0 && wtot != 0) base = kPair ? atom_add_cluster(map_to_peer(smem_u32(&npos), 0), wtot) : atomicAdd(&npos, wtot);
    base = __shfl_sync(0xffffffffu, base, 0);
#pragma unroll
    for (int q = 0; q < PF; ++q) {
      const int i0 = first_key(rd0 + q);
      int ph = (base & 0xffff) + (excl[q] & 0xffff);
      int pe = (base >> 16) + (excl[q] >> 16);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (((hi[q] | eq[q]) >> u) & 1u) {
          const uint64_t key = rank_key(f[q][u], static_cast<uint32_t>(i0 + u));
          if ((hi[q] >> u) & 1u) {
            if (ph < 2048) {
              if (kPair) st_cluster_u64(map_to_peer(smem_u32(abv + ph), 0), key);
              else abv[ph] = key;
            }
            ++ph;
          } else {
            if (pe < kDecodeSelBinCap) {
              if (kPair) st_cluster_u64(map_to_peer(smem_u32(bin_keys + pe), 0), key);
              else bin_keys[pe] = key;
            }
            ++pe;
          }
        }
      }
    }
  }
  if constexpr (kPair) {
    cluster_sync_all();  // CTA 1's candidates have landed in CTA 0
    if (crank != 0) return true;
  }
  __syncthreads();
  // 4. rank the candidates (the ranking buffer reuses the bin keys' space
  //    once every thread holds its candidates)
  uint64_t v[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int i = tid + j * NT;
    v[j] = (i < above) ? abv[i] : ((i - above < inb) ? bin_keys[i - above] : 0ull);
  }
  return topk_rank_by_bins<NT, NV>(v, K, hist, start, small, bin_keys, kDecodeSelBinCap, kDecodeBinRankMax, tid,
                                   bar, out);
}

// Exact top-k of sequence blockIdx.x, ranked, as its index row idx[b, 0..K):
// the fast path above, else (a crowded bin) the exact select into sel_keys
// and a bitonic ranking of those keys.
__global__ void __launch_bounds__(kDecodeSelThreads)
    decode_select_kernel(const float* __restrict__ scores, const int32_t* __restrict__ lens, int L_max, int K,
                         const uint32_t* __restrict__ hist_in, uint64_t* __restrict__ sel_keys,
                         int32_t* __restrict__ idx) {
  griddep_wait();               // launched as a programmatic dependent of the scoring kernel
  griddep_launch_dependents();  // the attention may be scheduled now; it waits for this grid
  if (decode_rank_fast<false>(scores, lens, L_max, K, hist_in, idx)) return;  // the same answer on every thread
  __syncthreads();
  decode_select_body(scores, lens, L_max, K, hist_in, sel_keys, static_cast<int>(blockIdx.x));
  extern __shared__ __align__(16) uint8_t dsmem[];
  __syncthreads();  // the selected keys (global, this CTA's writes) are complete; the bin buffer is free
  const size_t row = static_cast<size_t>(blockIdx.x) * K;
  sort_keys_to_idx<kDecodeSelThreads>(reinterpret_cast<uint64_t*>(dsmem), sel_keys + row, K, idx + row);
}

// The same selection with two CTAs per sequence (a cluster; the scoring
// kernel's histogram required): the pass over the scores is split between
// them (decode_rank_fast<true>); when the fast path does not apply, CTA 0
// runs the single-CTA selection for the sequence alone.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kDecodeSelThreads)
    decode_select_pair_kernel(const float* __restrict__ scores, const int32_t* __restrict__ lens, int L_max, int K,
                              const uint32_t* __restrict__ hist_in, uint64_t* __restrict__ sel_keys,
                              int32_t* __restrict__ idx) {
  griddep_wait();               // launched as a programmatic dependent of the scoring kernel
  griddep_launch_dependents();  // the attention may be scheduled now; it waits for this grid
  if (decode_rank_fast<true>(scores, lens, L_max, K, hist_in, idx)) return;  // the same answer on every thread
  if (cluster_ctarank() != 0) return;
  __syncthreads();
  const int b = static_cast<int>(blockIdx.x >> 1);
  decode_select_body(scores, lens, L_max, K, hist_in, sel_keys, b);
  extern __shared__ __align__(16) uint8_t dsmem[];
  __syncthreads();  // the selected keys (global, this CTA's writes) are complete; the bin buffer is free
  const size_t row = static_cast<size_t>(b) * K;
  sort_keys_to_idx<kDecodeSelThreads>(reinterpret_cast<uint64_t*>(dsmem), sel_keys + row, K, idx + row);
}

}  // namespace dsa
