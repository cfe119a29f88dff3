// Prefill lightning indexer with the top-k selection streamed into its
// epilogue, for one causal sequence of L tokens.
//
// The score ("Lightning Indexer 的计算过程", step 3 <1>-<2>, adg.csdn.net/695234...;
// "DeepSeek-V3.2-Exp解析" section 一.1, dtcms.com):
//     I[t,s] = q_scale[t] * k_scale[s] * sum_j w[t,j] * ReLU(q8[t,j,:] . k8[s,:]),  s <= t.
// Scales are positive, so they are applied after the ReLU (equal in real
// arithmetic to dequantising first). The FP8 products are exact and summed in
// fp32 by the tensor core.
//
// Mapping onto tcgen05 (kind::f8f6f4, fp32 accumulator in TMEM):
//   D[key, (token, head)] = K_tile[128 keys x d_I] * Q_half[(token, head) x d_I]^T
// i.e. keys in M (128 TMEM lanes) and (token, head) in N (128 columns, two
// tokens of 64 heads). Four such accumulator buffers fill the 512 TMEM
// columns; each is drained by its own four epilogue warps (one per TMEM lane
// quarter), so the tensor core fills one buffer while the others drain. Each
// epilogue thread owns one key (one TMEM lane) and reduces the H_I heads of a
// token inside its own registers: no shuffles.
//
// A CTA is persistent and owns "row blocks" of RB = 4 * 128 / H_I consecutive
// query tokens (8 at H_I = 64), taken longest-first. For a row block it
// streams every key tile up to the block's last token (TMA, 4-stage ring), so
// each key tile is reused by RB tokens from shared memory.
//
// Selection (same page, step 4 <1>; deepseek.csdn.net section 2.2): each row
// keeps a candidate list in the workspace, admitting a key only if its 64-bit
// ranking key beats the row's threshold. When a list nears capacity it is cut
// to exactly topk keys by a cooperative radix select and the threshold rises
// to the cut. Nothing that could still rank in the top-k is ever dropped, and
// the L x L score matrix never exists anywhere. At the end of a row block each
// row's exact top-k keys are ranked in shared memory (a histogram of the
// keys' high bits, then ranks inside each bin) and written as token indices.
#pragma once

#include <type_traits>

#include "dsa_common.cuh"
#include "topk_select.cuh"

namespace dsa {

template <int HI, int DI>
struct IdxPrefillCfg {
  static constexpr int BM = 128;               // keys per tile (MMA M, TMEM lanes)
  static constexpr int NCOL = 128;             // accumulator columns per buffer (MMA N)
  static constexpr int NACC = 4;               // accumulator buffers: all 512 TMEM columns
  static constexpr int TB = NCOL / HI;         // tokens per accumulator buffer
  static constexpr int RB = TB * NACC;         // tokens per row block
  static constexpr int KST = 4;                // key-tile ring depth
  static constexpr int QROWS = RB * HI;        // (token, head) query rows of a row block
  static constexpr int QBOX = 256;             // query rows per TMA box
  static constexpr int QBYTES = QROWS * DI;
  static constexpr int KTILE_BYTES = BM * DI;
  static constexpr int NEPI = 16;              // epilogue warps: 4 per buffer, one per TMEM lane quarter
  static constexpr int NTHREADS = (2 + NEPI) * 32;
  static constexpr int NET = NEPI * 32;        // epilogue threads
  static constexpr int TOK_PER_WARP = TB;      // an epilogue warp scores every token of its buffer
  static constexpr int TPH = 64 / HI;          // tokens per 64-column half of a buffer
  static constexpr int CHECK_EVERY = 16;       // key tiles between list-capacity checks
  static constexpr int NSAMPLE = 8;            // key tiles scored first to set a row's starting threshold
  static constexpr SwizzleMode SW = (DI == 128) ? kSw128 : kSw64;
  static constexpr uint32_t SBO = 8 * DI;      // bytes between 8-row core groups
  static constexpr uint32_t IDESC = instr_desc(kFmtE4M3, 128, NCOL, false, false);
  static constexpr int KSTEPS = DI / 32;       // MMA K = 32 for 8-bit inputs

  // shared memory carve-up (offsets from a 1024-byte aligned base)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QBYTES;
  static constexpr int OFF_W = OFF_K + KST * KTILE_BYTES;  // f32 [RB][HI]
  static constexpr int OFF_QS = OFF_W + RB * HI * 4;       // f32 [RB]
  static constexpr int OFF_THR = OFF_QS + RB * 4;          // u64 [RB]
  static constexpr int OFF_CNT = OFF_THR + RB * 8;         // i32 [RB][4] sub-list counts
  static constexpr int OFF_SCR = OFF_CNT + RB * 16;        // i32 select scratch
  // select scratch: [0, 2048) bin counts, [2048, 2112) the cuts' small fields,
  // [2112, 4160) bin starts and [4160, 4224) small fields of the final ranking;
  // the radix select's per-warp histograms overlay [0, 4112)
  static constexpr int SCR_START = cut_scratch_ints();
  static constexpr int SCR_SMALL = SCR_START + 2048;
  static constexpr int SCR_INTS = SCR_SMALL + 64;
  static_assert(SCR_INTS >= select_scratch_ints(NEPI * 32), "radix select scratch");
  static constexpr int SRT_N = 4096;                                       // keys of the final ranking buffer
  static constexpr int OFF_SRT = (OFF_SCR + SCR_INTS * 4 + 15) / 16 * 16;  // u64 [SRT_N]
  static constexpr int OFF_BAR = OFF_SRT + SRT_N * 8;
  static constexpr int NBAR = 2 + 2 * KST + 2 * NACC;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;      // tmem base, abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack

  static_assert(HI * TB == NCOL && HI <= 64, "heads must divide a buffer's 128 columns");
  static_assert(QROWS % QBOX == 0, "whole query boxes per row block");
  static_assert(RB <= 64, "one bit per row in the 64-bit cut mask");
  static_assert(NACC * NCOL == 512, "the buffers fill TMEM");
};

struct IdxPrefillParams {
  const float* q_scale;  // [L]
  const float* w;        // [L, HI]
  const float* k_scale;  // [L]
  int L;                 // keys in the cache (positions 0..L-1)
  int q0, Tq;            // query row r sits at position q0 + r, r < Tq (q0 + Tq <= L)
  int topk;
  int rb_begin, rb_end;  // row blocks [rb_begin, rb_end) of RB query rows
  // selection mode
  uint64_t* cand;        // [gridDim.x][RB][cap] candidate lists
  int cap;
  int32_t* idx;          // [Tq][topk] token indices per row, ranked, -1 padded
  // Sampled starting thresholds: row blocks with t0 >= spec_min_t (0: never)
  // first score NSAMPLE evenly spread key tiles and start from the sample's
  // r-th largest score (r ~ 2 * topk * sampled keys / (t+1)). A row that
  // ends with fewer than topk keys at or above that start is re-run: its row
  // block index goes to redo_list[atomicAdd(redo_count, 1)].
  int spec_min_t;
  int* redo_count;
  int* redo_list;
  // Re-run mode: when rb_list is set, process row blocks rb_list[0 .. *list_count)
  // (plain streaming, no sampling) instead of [rb_begin, rb_end).
  const int* rb_list;
  const int* list_count;
  // Packed batch: when blk_seq is set, row block id covers local block
  // blk_lrb[id] of sequence blk_seq[id]; sequence b owns query rows
  // [seq_cuq[b], seq_cuq[b+1]) at positions from seq_q0[b] and keys
  // [seq_cuk[b], seq_cuk[b+1]) (local positions 0..). Ids are in longest-first order.
  const int* blk_seq;
  const int* blk_lrb;
  const int* seq_cuq;
  const int* seq_cuk;
  const int* seq_q0;
  // score mode (test hook)
  float* scores;         // [nrows][L]; rows t in [row0, row0 + nrows)
  int row0, nrows;
  // Paged key cache (the kernel's paged instance, one sequence): key s is pool
  // row block_table[s >> page_shift] * page + (s & (page - 1)) of the FP8 keys
  // and of k_scale; the pool holds pool_pages pages.
  const int32_t* block_table;
  int page_shift, pool_pages;
};

// sum_j w[j] * ReLU(x_j) over the H_I accumulator values of one token
// (registers loaded from TMEM), in eight partial sums held as four float pairs
// and accumulated with the packed two-lane FMA: head j of each group of eight
// goes to partial sum j. In a group the first six ReLUs are max(x, 0) (ALU
// pipe) and the last two x + |x| = 2 ReLU(x) (FMA pipe), so both pipes carry
// part of the work; that last pair accumulates exactly twice the plain sums
// (scaling by two is exact in binary floating point) and is halved at the
// end, so the result is bit-identical to using max(x, 0) throughout. A token
// whose heads all ReLU to zero gets exactly 0. The weights come from shared
// memory as 16-byte vectors. Shared by both modes, so scores are identical.
template <int HI>
__device__ __forceinline__ float head_sum(const uint32_t* x, const float* __restrict__ w) {
  static_assert(HI % 8 == 0, "groups of eight heads");
  float2 acc[4];
#pragma unroll
  for (int a = 0; a < 4; ++a) acc[a] = make_float2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < HI; j += 8) {
    const float4 w0 = *reinterpret_cast<const float4*>(w + j);
    const float4 w1 = *reinterpret_cast<const float4*>(w + j + 4);
    float r[8];
#pragma unroll
    for (int a = 0; a < 6; ++a) r[a] = fmaxf(__uint_as_float(x[j + a]), 0.f);
#pragma unroll
    for (int a = 6; a < 8; ++a) {
      const float v = __uint_as_float(x[j + a]);
      r[a] = __fadd_rn(v, fabsf(v));
    }
    acc[0] = __ffma2_rn(make_float2(w0.x, w0.y), make_float2(r[0], r[1]), acc[0]);
    acc[1] = __ffma2_rn(make_float2(w0.z, w0.w), make_float2(r[2], r[3]), acc[1]);
    acc[2] = __ffma2_rn(make_float2(w1.x, w1.y), make_float2(r[4], r[5]), acc[2]);
    acc[3] = __ffma2_rn(make_float2(w1.z, w1.w), make_float2(r[6], r[7]), acc[3]);
  }
  return ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) + ((acc[2].x + acc[2].y) + 0.5f * (acc[3].x + acc[3].y));
}

// Threshold of a row as a float: a score s can pass only if s >= this value
// (the score part of the 64-bit threshold; -inf for the empty threshold 0).
__device__ __forceinline__ float thr_score(uint64_t thr) {
  const uint32_t hi = static_cast<uint32_t>(thr >> 32);
  return hi == 0 ? -INFINITY : order_key_float(hi);
}

// Largest bin the final ranking scans key by key (more: the exact select and
// the bitonic ranking take over).
constexpr int kBinRankMax = 96;

// Key tile of step i of a row block's sequence: with sampling, steps
// 0..NSAMPLE-1 are tiles at the middles of NSAMPLE equal strata of the
// block's nkt tiles, then every tile 0..nkt-1 follows in order.
template <int NS>
__device__ __forceinline__ int tile_at(int i, int nkt, bool spec) {
  if (!spec) return i;
  if (i < NS) return ((2 * i + 1) * nkt) / (2 * NS);
  return i - NS;
}
// Rank r of the sampled key whose score starts a row's threshold: twice the
// row's share of topk among the sampled keys, so that the expected count of
// keys at or above it is ~2 * topk; at least 1, at most n.
__device__ __forceinline__ int sample_rank(int topk, int sampled_keys, int t, int n) {
  const long long num = 2ll * topk * sampled_keys;
  const long long den = static_cast<long long>(t + 1);
  long long r = (num + den - 1) / den;
  if (r > n) r = n;
  if (r < 1) r = 1;
  return static_cast<int>(r);
}

// Paged key cache: the page-table entry of key s (-1 past the cache), and the
// pool row a box starting at key s reads (the pool's end, which TMA fills
// with zeros, past the cache or behind a bad entry).
__device__ __forceinline__ int prefill_page_entry(const IdxPrefillParams& p, int s, int L) {
  return (s < L) ? __ldg(p.block_table + (s >> p.page_shift)) : -1;
}
__device__ __forceinline__ int prefill_pool_row(const IdxPrefillParams& p, int s, int L, int page) {
  if (s >= L) return p.pool_pages << p.page_shift;
  if (page < 0 || page >= p.pool_pages) {
    set_device_error(kErrBadIndex, 3);
    return p.pool_pages << p.page_shift;
  }
  return (page << p.page_shift) + (s & ((1 << p.page_shift) - 1));
}

template <int HI, int DI, bool kSelect, int MQ, bool kPaged = false>
__global__ void __launch_bounds__(IdxPrefillCfg<HI, DI>::NTHREADS, 1)
    indexer_prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const IdxPrefillParams p) {
  using C = IdxPrefillCfg<HI, DI>;
  // 1024-byte aligned base, derived from the shared array by an offset so
  // the compiler keeps every access in the shared address space
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* q_s = smem + C::OFF_Q;
  uint8_t* k_s = smem + C::OFF_K;
  float* w_s = reinterpret_cast<float*>(smem + C::OFF_W);
  float* qs_s = reinterpret_cast<float*>(smem + C::OFF_QS);
  uint64_t* thr_s = reinterpret_cast<uint64_t*>(smem + C::OFF_THR);
  int* cnt_s = reinterpret_cast<int*>(smem + C::OFF_CNT);
  int* scr_s = reinterpret_cast<int*>(smem + C::OFF_SCR);
  uint64_t* srt_s = reinterpret_cast<uint64_t*>(smem + C::OFF_SRT);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = bars + 2 + C::KST;
  uint64_t* acc_full = bars + 2 + 2 * C::KST;
  uint64_t* acc_empty = bars + 2 + 2 * C::KST + C::NACC;
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  int* abort_s = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);
  // bit tl: a sub-list of row tl may overflow before the next check (set by
  // the appending warp, read at the capacity checks)
  unsigned long long* cutmask_s = reinterpret_cast<unsigned long long*>(smem + C::OFF_MISC + 8);
  const AbortFlag ab{abort_s};

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();

  if (threadIdx.x == 0) {
    *abort_s = 0;
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < C::KST; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 1);
    }
    for (int i = 0; i < C::NACC; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, C::NEPI / C::NACC);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
  }
  if (warp == 1) tmem_alloc(tmem_base_s, 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_s;

  const bool list_mode = p.rb_list != nullptr;
  const int nrb = list_mode ? *p.list_count : (p.rb_end - p.rb_begin);
  const int G = gridDim.x;
  // row block of step j and whether it samples first (the same on every role)
  auto block_of = [&](int j) { return list_mode ? p.rb_list[j] : (p.blk_seq ? j : p.rb_end - 1 - j); };
  // where row block `id` lives: first query row, end of its sequence's rows,
  // position of its first row, its sequence's key count and first key row
  struct Blk {
    int r0, rend, t0, L, kbase;
  };
  auto blk = [&](int id) {
    Blk k;
    if (p.blk_seq) {
      const int sq = p.blk_seq[id], lrb = p.blk_lrb[id];
      k.r0 = p.seq_cuq[sq] + lrb * C::RB;
      k.rend = p.seq_cuq[sq + 1];
      k.t0 = p.seq_q0[sq] + lrb * C::RB;
      k.kbase = p.seq_cuk[sq];
      k.L = p.seq_cuk[sq + 1] - k.kbase;
    } else {
      k.r0 = id * C::RB;
      k.rend = p.Tq;
      k.t0 = p.q0 + k.r0;
      k.kbase = 0;
      k.L = p.L;
    }
    return k;
  };
  auto samples = [&](int t0, int nkt) {
    return kSelect && !list_mode && p.spec_min_t > 0 && t0 >= p.spec_min_t && nkt >= 4 * C::NSAMPLE;
  };

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t qe_phase = 1;
      int kslot = 0;
      uint32_t ke_phase = 1;
      for (int j = blockIdx.x; j < nrb; j += G) {
        const Blk bk = blk(block_of(j));
        const int r0 = bk.r0;
        const int t0 = bk.t0;
        const int tlast = t0 + min(C::RB, bk.rend - r0) - 1;
        const int nkt = tlast / C::BM + 1;
        const bool spec = samples(t0, nkt);
        const int nsteps = nkt + (spec ? C::NSAMPLE : 0);
        if (!mbar_wait(q_empty, qe_phase, ab, 1)) break;
        qe_phase ^= 1;
        mbar_arrive_expect_tx(q_full, C::QBYTES);
        for (int b = 0; b < C::QROWS / C::QBOX; ++b)
          // the query rows are read once: evict-first keeps L2 for the key
          // tiles (read by every row block) and the candidate lists
          tma_load_2d_hint(q_s + b * C::QBOX * DI, &tmQ, q_full, 0, r0 * HI + b * C::QBOX, l2_evict_first());
        bool ok = true;
        // paged: one box of R = min(page, BM) rows per page of the tile; the
        // next tile's page entries load before the wait for this tile's slot
        constexpr int MAXB = C::BM / 16;
        [[maybe_unused]] const int R = kPaged ? min(1 << p.page_shift, C::BM) : C::BM;
        [[maybe_unused]] int nxt[MAXB];
        if constexpr (kPaged) {
#pragma unroll
          for (int q = 0; q < MAXB; ++q)
            nxt[q] = (q * R < C::BM) ? prefill_page_entry(p, tile_at<C::NSAMPLE>(0, nkt, spec) * C::BM + q * R, bk.L)
                                     : -1;
        }
        for (int i = 0; i < nsteps; ++i) {
          [[maybe_unused]] int cur[MAXB];
          if constexpr (kPaged) {
#pragma unroll
            for (int q = 0; q < MAXB; ++q) cur[q] = nxt[q];
            if (i + 1 < nsteps) {
              const int sn = tile_at<C::NSAMPLE>(i + 1, nkt, spec) * C::BM;
#pragma unroll
              for (int q = 0; q < MAXB; ++q) nxt[q] = (q * R < C::BM) ? prefill_page_entry(p, sn + q * R, bk.L) : -1;
            }
          }
          if (!mbar_wait(k_empty + kslot, ke_phase, ab, 2)) { ok = false; break; }
          mbar_arrive_expect_tx(k_full + kslot, C::KTILE_BYTES);
          if constexpr (kPaged) {
            const int sc = tile_at<C::NSAMPLE>(i, nkt, spec) * C::BM;
#pragma unroll
            for (int q = 0; q < MAXB; ++q)
              if (q * R < C::BM)
                tma_load_2d(k_s + kslot * C::KTILE_BYTES + q * R * DI, &tmK, k_full + kslot, 0,
                            prefill_pool_row(p, sc + q * R, bk.L, cur[q]));
          } else {
            tma_load_2d(k_s + kslot * C::KTILE_BYTES, &tmK, k_full + kslot, 0,
                        bk.kbase + tile_at<C::NSAMPLE>(i, nkt, spec) * C::BM);
          }
          if (++kslot == C::KST) { kslot = 0; ke_phase ^= 1; }
        }
        if (!ok) break;
      }
      // Drain: do not leave the CTA while a copy may still land in its
      // shared memory (bounded, like every wait here).
      for (int i = 0; i < C::KST; ++i) {
        if (ab.raised()) break;
        mbar_wait(k_empty + kslot, ke_phase, ab, 3);
        if (++kslot == C::KST) { kslot = 0; ke_phase ^= 1; }
      }
      if (!ab.raised()) mbar_wait(q_empty, qe_phase, ab, 4);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: the warp waits converged, one elected lane issues ----------------
    // Per key tile: one accumulator buffer after the other (tokens b * TB ..
    // b * TB + TB - 1 into buffer b), each as soon as its four epilogue warps
    // have released it.
    {
      uint32_t qf_phase = 0;
      int kslot = 0;
      uint32_t kf_phase = 0;
      uint32_t ae_bits = (1u << C::NACC) - 1u;  // bit b: parity of buffer b's next release
      const uint32_t q_base = smem_u32(q_s);
      const uint32_t k_base = smem_u32(k_s);
      for (int j = blockIdx.x; j < nrb; j += G) {
        const Blk bk = blk(block_of(j));
        const int t0 = bk.t0;
        const int tlast = t0 + min(C::RB, bk.rend - bk.r0) - 1;
        const int nkt = tlast / C::BM + 1;
        const int nsteps = nkt + (samples(t0, nkt) ? C::NSAMPLE : 0);
        if (!mbar_wait_warp(q_full, qf_phase, ab, 5)) break;
        qf_phase ^= 1;
        bool ok = true;
        for (int kt = 0; kt < nsteps && ok; ++kt) {
          if (!mbar_wait_warp(k_full + kslot, kf_phase, ab, 6)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = k_base + kslot * C::KTILE_BYTES;
#pragma unroll
          for (int b = 0; b < C::NACC; ++b) {
            if (ok && !mbar_wait_warp(acc_empty + b, (ae_bits >> b) & 1u, ab, 7)) ok = false;
            if (ok) {
              ae_bits ^= 1u << b;
              tc_fence_after();
              if (elect_one()) {
                const uint32_t b_addr = q_base + b * C::NCOL * DI;
#pragma unroll
                for (int kk = 0; kk < C::KSTEPS; ++kk) {
                  const uint64_t ad = smem_desc(a_addr + kk * 32, 16, C::SBO, C::SW);
                  const uint64_t bd = smem_desc(b_addr + kk * 32, 16, C::SBO, C::SW);
                  mma_f8(tmem + b * C::NCOL, ad, bd, C::IDESC, kk > 0 ? 1u : 0u);
                }
                tc_commit(acc_full + b);
                if (b == C::NACC - 1) {
                  tc_commit(k_empty + kslot);
                  if (kt == nsteps - 1) tc_commit(q_empty);
                }
              }
              __syncwarp();
            }
          }
          if (!ok) break;
          if (++kslot == C::KST) { kslot = 0; kf_phase ^= 1; }
        }
        if (!ok) break;
      }
    }
  } else {
    // ---------------- epilogue: scores, threshold filter, selection ----------------
    const int e = static_cast<int>(warp) - 2;          // 0..NEPI-1
    const int et = e * 32 + static_cast<int>(lane);    // 0..NET-1
    const int quarter = static_cast<int>(warp & 3);    // TMEM lane quarter this warp may access
    const int grp = e / 4;                             // the accumulator buffer this warp drains
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t lanemask_lt = (1u << lane) - 1u;
    constexpr int TPW = C::TOK_PER_WARP;
    constexpr int NR = TPW;  // rows this warp scores: the tokens of its buffer
    const GroupBar bar{1, C::NET, ab};
    uint32_t af_phase = 0;  // parity of this warp's buffer's next completed fill
    // Row tl's list is four quarter sub-lists of capq keys; sub-list q only
    // receives keys from TMEM lane quarter q, so exactly one warp appends to
    // it: its count lives in that warp's registers between cuts.
    const int capq = p.cap / 4;
    uint64_t* my_cand = p.cand + static_cast<size_t>(blockIdx.x) * C::RB * p.cap;
    int* pos_s = scr_s + cut_scratch_ints() - 16;  // 16 ints: warp sums of the block scan
    auto row_of = [&](int r) { return grp * C::TB + r; };
    // this warp's sub-list of each of its rows in the CTA's candidate lists
    uint64_t* row_ptr[TPW];
#pragma unroll
    for (int r = 0; r < TPW; ++r)
      row_ptr[r] = my_cand + static_cast<size_t>(row_of(r)) * p.cap + static_cast<size_t>(quarter) * capq;

    for (int j = blockIdx.x; j < nrb; j += G) {
      const int rb = block_of(j);
      const Blk bk = blk(rb);
      const int r0 = bk.r0;
      const int t0 = bk.t0;  // position of the block's first query row
      const int tlast = t0 + min(C::RB, bk.rend - r0) - 1;
      const int nkt = tlast / C::BM + 1;
      const bool spec = samples(t0, nkt);
      const int nsteps = nkt + (spec ? C::NSAMPLE : 0);
      const bool ragged = r0 + C::RB > bk.rend;  // the block runs past its sequence's last query row
      // per-row-block state
      for (int i = et; i < C::RB * HI; i += C::NET) {
        const int r = r0 + i / HI;
        w_s[i] = (r < bk.rend) ? p.w[static_cast<size_t>(r) * HI + (i % HI)] : 0.f;
      }
      for (int i = et; i < C::RB; i += C::NET) {
        const int r = r0 + i;
        qs_s[i] = (r < bk.rend) ? p.q_scale[r] : 0.f;
        thr_s[i] = 0ull;
      }
      for (int i = et; i < 4 * C::RB; i += C::NET) cnt_s[i] = 0;
      if (et == 0) *cutmask_s = 0;
      if (!bar.sync()) break;
      // this warp's rows in registers: query scale, threshold (exact and as a
      // score), and its sub-list's count
      float qs_r[NR], thf_r[NR];
      uint64_t th_r[NR];
      int cnt_r[NR];
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        qs_r[r] = qs_s[row_of(r)];
        th_r[r] = 0ull;
        thf_r[r] = -INFINITY;
        cnt_r[r] = 0;
      }
      // cuts happen in shared memory: publish the counts before, reload after
      auto publish_counts = [&]() {
        if (lane == 0) {
#pragma unroll
          for (int r = 0; r < NR; ++r) cnt_s[row_of(r) * 4 + quarter] = cnt_r[r];
        }
      };
      auto reload_rows = [&]() {
#pragma unroll
        for (int r = 0; r < NR; ++r) {
          th_r[r] = thr_s[row_of(r)];
          thf_r[r] = thr_score(th_r[r]);
          cnt_r[r] = cnt_s[row_of(r) * 4 + quarter];
        }
      };
      bool ok = true;
      float ks_next = 0.f;
      [[maybe_unused]] int pg_next = -1;
      {
        const int s0 = tile_at<C::NSAMPLE>(0, nkt, spec) * C::BM + quarter * 32 + static_cast<int>(lane);
        if constexpr (kPaged) {
          const int r = prefill_pool_row(p, s0, bk.L, prefill_page_entry(p, s0, bk.L));
          ks_next = (s0 < bk.L && r < (p.pool_pages << p.page_shift)) ? __ldg(p.k_scale + r) : 0.f;
          if (1 < nsteps)
            pg_next = prefill_page_entry(
                p, tile_at<C::NSAMPLE>(1, nkt, spec) * C::BM + quarter * 32 + static_cast<int>(lane), bk.L);
        } else {
          ks_next = (s0 < bk.L) ? __ldg(p.k_scale + bk.kbase + s0) : 0.f;
        }
      }
      // One key tile (step i of the block's sequence) for this warp: wait for
      // its buffer, reduce the heads of its tokens, release the buffer, then
      // filter and append. kMasked: the tile reaches past the block's first
      // position (the causal diagonal or past the cache) or the block is ragged.
      auto tile_step = [&](int i, auto masked_c) -> bool {
        constexpr bool kMasked = decltype(masked_c)::value;
        const int kt = tile_at<C::NSAMPLE>(i, nkt, spec);
        const int s = kt * C::BM + quarter * 32 + static_cast<int>(lane);
        const float ks = ks_next;
        if (i + 1 < nsteps) {
          const int sn = tile_at<C::NSAMPLE>(i + 1, nkt, spec) * C::BM + quarter * 32 + static_cast<int>(lane);
          if constexpr (kPaged) {
            const int r = prefill_pool_row(p, sn, bk.L, pg_next);
            ks_next = (sn < bk.L && r < (p.pool_pages << p.page_shift)) ? __ldg(p.k_scale + r) : 0.f;
            if (i + 2 < nsteps)
              pg_next = prefill_page_entry(
                  p, tile_at<C::NSAMPLE>(i + 2, nkt, spec) * C::BM + quarter * 32 + static_cast<int>(lane), bk.L);
          } else {
            ks_next = (sn < bk.L) ? __ldg(p.k_scale + bk.kbase + sn) : 0.f;
          }
        }
        if (!mbar_wait(acc_full + grp, af_phase, ab, 8)) return false;
        af_phase ^= 1u;
        tc_fence_after();
        // this warp's 128 columns of the buffer (TPW tokens of HI heads) in
        // two halves of 64
        float raw[TPW];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t x[64];
          tmem_ld64(tmem + lane_addr + grp * C::NCOL + hh * 64, x);
#pragma unroll
          for (int q = 0; q < C::TPH; ++q)
            raw[hh * C::TPH + q] = head_sum<HI>(x + q * HI, w_s + row_of(hh * C::TPH + q) * HI);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty + grp);  // the tensor core may refill this buffer now
#pragma unroll
        for (int r = 0; r < TPW; ++r) {
          const int tl = row_of(r);
          const float score = __fmul_rn(__fmul_rn(raw[r], qs_r[r]), ks);
          if constexpr (kSelect) {
            // a key can only pass if its score reaches the threshold's score
            bool pass = score >= thf_r[r];
            if constexpr (kMasked) pass = pass && (r0 + tl < bk.rend) && (s <= t0 + tl);
            if (__any_sync(0xffffffffu, pass)) {
              const uint64_t key = (static_cast<uint64_t>(float_order_key(score)) << 32) |
                                   static_cast<uint64_t>(~static_cast<uint32_t>(s));
              const bool pred = pass && key > th_r[r];
              const uint32_t m = __ballot_sync(0xffffffffu, pred);
              if (pred) row_ptr[r][cnt_r[r] + __popc(m & lanemask_lt)] = key;
              cnt_r[r] += __popc(m);
            }
          } else {
            const int t = t0 + tl;
            if ((r0 + tl < bk.rend) && (s <= t) && t >= p.row0 && t < p.row0 + p.nrows)
              p.scores[static_cast<size_t>(t - p.row0) * p.L + s] = score;
          }
        }
        return true;
      };
      // After step i: the end of the sample, or a capacity checkpoint.
      auto after_step = [&](int i) -> bool {
        if constexpr (kSelect) {
          if (spec && i == C::NSAMPLE - 1) {
            // End of the sample: each row's threshold starts at the score of
            // the lower edge of the histogram bin holding its r-th largest
            // sampled key (keys scoring at least that pass; index bits cleared
            // so equal scores are kept), and the list is emptied: the sampled
            // tiles come round again in order.
            publish_counts();
            if (!bar.sync()) return false;
            for (int tl = 0; tl < C::RB; ++tl) {
              const int t = t0 + tl;
              if (r0 + tl >= bk.rend) break;
              const int* cn = cnt_s + tl * 4;
              const int n = cn[0] + cn[1] + cn[2] + cn[3];
              if (n == 0) continue;
              const int r = sample_rank(p.topk, C::NSAMPLE * C::BM, t, n);
              uint64_t* row = my_cand + static_cast<size_t>(tl) * p.cap;
              uint64_t v[4 * MQ];
              load_sublists<C::NET, MQ>(row, capq, cn, et, v);
              // the lower edge of the bin holding the r-th largest sampled key:
              // at most a bin's width below that key, so no fewer keys pass
              int above = 0, inb = 0;
              const uint64_t floor = histogram_cut<C::NET, 4 * MQ>(v, r, scr_s, et, bar, &above, &inb);
              if (et == 0) {
                const uint64_t hi = floor >> 32;
                thr_s[tl] = (hi == 0) ? 0ull : (hi << 32) - 1;
              }
              if (!bar.sync()) break;
            }
            if (et < 4 * C::RB) cnt_s[et] = 0;
            if (!bar.sync()) return false;
            reload_rows();
            return true;
          }
          // Every CHECK_EVERY tiles, cut any list whose sub-list could
          // overflow before the next check (at most 32 appends per sub-list
          // and tile): one histogram pass keeps every key in or above the bin
          // of the k-th largest; if that keeps too many, an exact select
          // keeps exactly k.
          if ((i % C::CHECK_EVERY) != C::CHECK_EVERY - 1) return true;
          unsigned long long near = 0;  // rows of this warp whose sub-list is near capacity
#pragma unroll
          for (int r = 0; r < NR; ++r)
            if (cnt_r[r] > capq - 32 * C::CHECK_EVERY) near |= 1ull << row_of(r);
          if (lane == 0 && near) atomicOr(cutmask_s, near);
          publish_counts();
          if (!bar.sync()) return false;
          const unsigned long long cmask = *cutmask_s;
          if (cmask == 0) return true;
          for (int tl = 0; tl < C::RB; ++tl) {
            const int* cn = cnt_s + tl * 4;
            if ((cmask >> tl) & 1ull) {
              uint64_t* row = my_cand + static_cast<size_t>(tl) * p.cap;
              const int n = cn[0] + cn[1] + cn[2] + cn[3];
              uint64_t v[4 * MQ];
              load_sublists<C::NET, MQ>(row, capq, cn, et, v);
              uint64_t floor = 1ull;  // fewer than topk keys: only rebalance the sub-lists
              if (n > p.topk) {
                int above = 0, inb = 0;
                floor = histogram_cut<C::NET, 4 * MQ>(v, p.topk, scr_s, et, bar, &above, &inb);
                if (above + inb > p.cap / 2) {
                  // keys below the boundary bin can go now; exact select on the rest
#pragma unroll
                  for (int q = 0; q < 4 * MQ; ++q) v[q] = (v[q] >= floor) ? v[q] : 0ull;
                  floor = radix_select_floor<C::NET, 4 * MQ>(v, p.topk, scr_s, et, bar);
                }
              }
              store_sublists<C::NET, MQ>(row, capq, cnt_s + tl * 4, v, floor, pos_s, et, bar);
              if (et == 0 && floor - 1 > thr_s[tl]) thr_s[tl] = floor - 1;
              if (!bar.sync()) break;
            }
          }
          // every flagged row was cut; all threads read the mask before the cuts' barriers
          if (et == 0) *cutmask_s = 0;
          if (!bar.sync()) return false;
          reload_rows();
        }
        return true;
      };
      // the sampled tiles, then the tiles wholly at or before the block's
      // first position (no masking), then the masked tail
      const int ns = spec ? C::NSAMPLE : 0;
      const int kt_m = ragged ? 0 : min(nkt, (t0 + 1) / C::BM);
      for (int i = 0; i < ns && ok; ++i) ok = tile_step(i, std::true_type{}) && after_step(i);
      // (unrolled by four: about 3.5% faster than by one, two, three or eight)
#pragma unroll 4
      for (int i = ns; i < ns + kt_m && ok; ++i) ok = tile_step(i, std::false_type{}) && after_step(i);
      for (int i = ns + kt_m; i < nsteps && ok; ++i) ok = tile_step(i, std::true_type{}) && after_step(i);
      if (!ok) break;
      if constexpr (kSelect) {
        // exact top-k of each row: the histogram pass finds the boundary bin,
        // a radix select over that bin's keys alone finds the exact cut; the
        // row's keys are then ranked in shared memory and its indices written
        publish_counts();
        if (!bar.sync()) break;
        bool redo = false;
        for (int tl = 0; tl < C::RB; ++tl) {
          const int t = t0 + tl;
          if (r0 + tl >= bk.rend) break;
          const int* cn = cnt_s + tl * 4;
          const int n = cn[0] + cn[1] + cn[2] + cn[3];
          // a sampled start above the row's k-th largest score left too few keys
          if (spec && n < min(p.topk, t + 1)) redo = true;
          uint64_t* row = my_cand + static_cast<size_t>(tl) * p.cap;
          uint64_t v[4 * MQ];
          load_sublists<C::NET, MQ>(row, capq, cn, et, v);
          int32_t* dst = p.idx + static_cast<size_t>(r0 + tl) * p.topk;
          if (!topk_rank_by_bins<C::NET, 4 * MQ>(v, p.topk, scr_s, scr_s + C::SCR_START, scr_s + C::SCR_SMALL, srt_s,
                                                 C::SRT_N, kBinRankMax, et, bar, dst)) {
            // a crowded bin: exact select, then the bitonic ranking
            uint64_t floor = 1ull;  // keep every valid key
            if (n > p.topk) {
              int above = 0, inb = 0;
              floor = histogram_cut<C::NET, 4 * MQ>(v, p.topk, scr_s, et, bar, &above, &inb);
              if (above + inb > p.topk) {
#pragma unroll
                for (int q = 0; q < 4 * MQ; ++q) v[q] = (v[q] >= floor) ? v[q] : 0ull;
                floor = radix_select_floor<C::NET, 4 * MQ>(v, p.topk, scr_s, et, bar);
              }
            }
            sort_selected_to_idx<C::NET, 4 * MQ>(v, floor, srt_s, pos_s, et, bar, p.topk, dst);
          }
          if (bar.aborted()) break;
        }
        if (bar.aborted()) break;
        if (redo && et == 0) p.redo_list[atomicAdd(p.redo_count, 1)] = rb;
      }
      if (!bar.sync()) break;
    }
    // a warp that stopped on the abort flag counts itself in at the barrier
    // the others may be waiting at
    if (bar.aborted()) bar.leave();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace dsa
