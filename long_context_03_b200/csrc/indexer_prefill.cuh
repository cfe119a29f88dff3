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
// i.e. keys in M (128 TMEM lanes) and (token, head) in N (256 columns). Each
// epilogue thread owns one key (one TMEM lane) and reduces the H_I heads of a
// token inside its own registers: no shuffles. Two 256-column accumulators
// alternate so the tensor core fills one while the epilogue drains the other.
//
// A CTA is persistent and owns "row blocks" of RB = 2 * 256 / H_I consecutive
// query tokens, taken longest-first. For a row block it streams every key tile
// up to the block's last token (TMA, 4-stage ring), so each key tile is reused
// by RB tokens from shared memory.
//
// Selection (same page, step 4 <1>; deepseek.csdn.net section 2.2): each row
// keeps a candidate list in the workspace, admitting a key only if its 64-bit
// ranking key beats the row's threshold. When a list nears capacity it is cut
// to exactly topk keys by a cooperative radix select and the threshold rises
// to the cut. Nothing that could still rank in the top-k is ever dropped, and
// the L x L score matrix never exists anywhere. At the end of a row block each
// row's exact top-k keys go to `sel_keys` (unordered); rank_sort_kernel then
// orders them.
#pragma once

#include "dsa_common.cuh"
#include "topk_select.cuh"

namespace dsa {

template <int HI, int DI>
struct IdxPrefillCfg {
  static constexpr int BM = 128;               // keys per tile (MMA M, TMEM lanes)
  static constexpr int NCOL = 256;             // accumulator columns per buffer (MMA N)
  static constexpr int TB = NCOL / HI;         // tokens per accumulator buffer
  static constexpr int NACC = 2;               // accumulator buffers
  static constexpr int RB = TB * NACC;         // tokens per row block
  static constexpr int KST = 4;                // key-tile ring depth
  static constexpr int QBUF_BYTES = NCOL * DI; // one Q half: 256 (token, head) rows x d_I bytes
  static constexpr int KTILE_BYTES = BM * DI;
  static constexpr int NEPI = 16;              // epilogue warps (4 per TMEM lane quarter)
  static constexpr int NTHREADS = (2 + NEPI) * 32;
  static constexpr int NET = NEPI * 32;        // epilogue threads
  static constexpr int TOK_PER_WARP = TB / 4;  // tokens of a buffer per epilogue warp (64 columns)
  static constexpr int CHECK_EVERY = 4;        // key tiles between list-capacity checks
  static constexpr int NSAMPLE = 8;            // key tiles scored first to set a row's starting threshold
  static constexpr SwizzleMode SW = (DI == 128) ? kSw128 : kSw64;
  static constexpr uint32_t SBO = 8 * DI;      // bytes between 8-row core groups
  static constexpr uint32_t IDESC = instr_desc(kFmtE4M3, 128, NCOL, false, false);
  static constexpr int KSTEPS = DI / 32;       // MMA K = 32 for 8-bit inputs

  // shared memory carve-up (offsets from a 1024-byte aligned base)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NACC * QBUF_BYTES;
  static constexpr int OFF_W = OFF_K + KST * KTILE_BYTES;  // f32 [RB][HI]
  static constexpr int OFF_QS = OFF_W + RB * HI * 4;       // f32 [RB]
  static constexpr int OFF_THR = OFF_QS + RB * 4;          // u64 [RB]
  static constexpr int OFF_CNT = OFF_THR + RB * 8;         // i32 [RB][4] sub-list counts
  static constexpr int OFF_SCR = OFF_CNT + RB * 16;        // i32 select scratch
  static constexpr int SCR_INTS = (select_scratch_ints(NEPI * 32) > cut_scratch_ints()) ? select_scratch_ints(NEPI * 32)
                                                                                        : cut_scratch_ints();
  static constexpr int OFF_BAR = (OFF_SCR + SCR_INTS * 4 + 7) / 8 * 8;
  static constexpr int NBAR = 2 + 2 * KST + 2 * NACC;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;      // tmem base, abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack

  static_assert(HI * TB == NCOL, "heads must divide 256");
  static_assert(TB % 4 == 0, "four epilogue warps per lane quarter split a buffer's tokens");
  static_assert(TOK_PER_WARP * HI == 64, "one 64-column slice per warp and buffer");
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
  uint64_t* sel_keys;    // [L][topk] exact top-k keys per row, unordered, 0-padded
  // Sampled starting thresholds: row blocks with t0 >= spec_min_t (0: never)
  // first score NSAMPLE evenly spread key tiles and start from the sample's
  // r-th largest score (r ~ 2.5 * topk * sampled keys / (t+1)). A row that
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

// sum_j w[j] * max(x_j, 0) over the H_I accumulator values of one token
// (registers loaded from TMEM), written as (sum_j w[j]*x_j + sum_j w[j]*|x_j|)/2
// so that both sums run on the FMA pipe: acc[0..3] take w*x as two packed
// float pairs (fma.rn.f32x2 on register pairs straight from the TMEM load),
// acc[4..7] take w*|x| with the absolute value folded into the scalar FMA.
// The halves cancel exactly where every head is negative (an exact zero stays
// zero). Shared by both modes so their scores are bit-identical.
template <int HI>
__device__ __forceinline__ void relu_weighted_acc(float (&acc)[8], const uint32_t* x, const float* __restrict__ w) {
  static_assert(HI % 4 == 0, "a multiple of 4 heads");
#pragma unroll
  for (int j = 0; j < HI; j += 4) {
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      uint64_t d, wa, xa, ca;
      asm("mov.b64 %0, {%1, %2};" : "=l"(wa) : "f"(w[j + 2 * pr]), "f"(w[j + 2 * pr + 1]));
      asm("mov.b64 %0, {%1, %2};" : "=l"(xa) : "r"(x[j + 2 * pr]), "r"(x[j + 2 * pr + 1]));
      asm("mov.b64 %0, {%1, %2};" : "=l"(ca) : "f"(acc[2 * pr]), "f"(acc[2 * pr + 1]));
      asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(wa), "l"(xa), "l"(ca));
      asm("mov.b64 {%0, %1}, %2;" : "=f"(acc[2 * pr]), "=f"(acc[2 * pr + 1]) : "l"(d));
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) acc[4 + a] = __fmaf_rn(w[j + a], fabsf(__uint_as_float(x[j + a])), acc[4 + a]);
  }
}
__device__ __forceinline__ float relu_weighted_finish(const float (&acc)[8]) {
  return 0.5f * (((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7])));
}

// Key tile of step i of a row block's sequence: with sampling, steps
// 0..NSAMPLE-1 are tiles at the middles of NSAMPLE equal strata of the
// block's nkt tiles, then every tile 0..nkt-1 follows in order.
template <int NS>
__device__ __forceinline__ int tile_at(int i, int nkt, bool spec) {
  if (!spec) return i;
  if (i < NS) return ((2 * i + 1) * nkt) / (2 * NS);
  return i - NS;
}
// Rank r of the sampled key whose score starts a row's threshold: about 2.5
// times the row's share of topk among the sampled keys, so that the expected
// count of keys at or above it is ~2.5 * topk; at least 1, at most n.
__device__ __forceinline__ int sample_rank(int topk, int sampled_keys, int t, int n) {
  const long long num = 5ll * topk * sampled_keys;
  const long long den = 2ll * (t + 1);
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
  int* cutmask_s = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);
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
      mbar_init(acc_empty + i, C::NEPI);
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
        mbar_arrive_expect_tx(q_full, C::NACC * C::QBUF_BYTES);
        for (int b = 0; b < C::NACC; ++b)
          tma_load_2d(q_s + b * C::QBUF_BYTES, &tmQ, q_full, 0, (r0 + b * C::TB) * HI);
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
    {
      uint32_t qf_phase = 0;
      int kslot = 0;
      uint32_t kf_phase = 0;
      uint32_t ae_phase[C::NACC];
      for (int b = 0; b < C::NACC; ++b) ae_phase[b] = 1;
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
          for (int b = 0; b < C::NACC; ++b) {
            if (!mbar_wait_warp(acc_empty + b, ae_phase[b], ab, 7)) { ok = false; break; }
            ae_phase[b] ^= 1;
            tc_fence_after();
            if (elect_one()) {
              const uint32_t b_addr = q_base + b * C::QBUF_BYTES;
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
    const int half = e / 4;                            // which quarter of a buffer's tokens
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t lanemask_lt = (1u << lane) - 1u;
    uint32_t af_phase[C::NACC];
    for (int b = 0; b < C::NACC; ++b) af_phase[b] = 0;
    // Row tl's list is four quarter sub-lists of capq keys; sub-list q only
    // receives keys from TMEM lane quarter q, so exactly one warp appends to
    // it and its count needs no atomics.
    const int capq = p.cap / 4;
    uint64_t* my_cand = p.cand + static_cast<size_t>(blockIdx.x) * C::RB * p.cap;
    int* pos_s = scr_s + cut_scratch_ints() - 16;  // 9 ints: warp sums of the block scan

    for (int j = blockIdx.x; j < nrb; j += G) {
      const int rb = block_of(j);
      const Blk bk = blk(rb);
      const int r0 = bk.r0;
      const int t0 = bk.t0;  // position of the block's first query row
      const int tlast = t0 + min(C::RB, bk.rend - r0) - 1;
      const int nkt = tlast / C::BM + 1;
      const bool spec = samples(t0, nkt);
      const int nsteps = nkt + (spec ? C::NSAMPLE : 0);
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
      named_bar_sync(1, C::NET);
      bool ok = true;
      float ks_next = 0.f;
      // paged: page entry of the key two steps ahead, its scale one step ahead
      // (no dependent load waits inside a step)
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
      for (int i = 0; i < nsteps && ok; ++i) {
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
        for (int b = 0; b < C::NACC; ++b) {
          if (!mbar_wait(acc_full + b, af_phase[b], ab, 8)) { ok = false; break; }
          af_phase[b] ^= 1;
          tc_fence_after();
          // this warp's tokens are 128 consecutive accumulator columns
          // this warp's 64 columns in two halves: the second half loads while
          // the first is reduced
          const uint32_t cbase = tmem + lane_addr + b * C::NCOL + half * 64;
          uint32_t xa[32], xb[32];
          tmem_ld32_nowait(cbase, xa);
          tmem_ld_wait_fence(xa);
          tmem_ld32_nowait(cbase + 32, xb);
          // row state first (its loads overlap the arithmetic), every token's
          // score next (independent chains), then the filter
          uint64_t thr_r[C::TOK_PER_WARP];
          int base_r[C::TOK_PER_WARP];
          if constexpr (kSelect) {
#pragma unroll
            for (int q = 0; q < C::TOK_PER_WARP; ++q) {
              const int tl = b * C::TB + half * C::TOK_PER_WARP + q;
              thr_r[q] = thr_s[tl];
              base_r[q] = cnt_s[tl * 4 + quarter];
            }
          }
          float score[C::TOK_PER_WARP];
          {
            // columns [0,32) then [32,64) of the slice; a token spans HI columns
            constexpr int TPH = (HI >= 32) ? 1 : 32 / HI;  // tokens per 32-column half
            float acc[C::TOK_PER_WARP][8];
#pragma unroll
            for (int q = 0; q < C::TOK_PER_WARP; ++q)
#pragma unroll
              for (int a = 0; a < 8; ++a) acc[q][a] = 0.f;
            const int tl0 = b * C::TB + half * C::TOK_PER_WARP;
            if constexpr (HI >= 32) {
              relu_weighted_acc<32>(acc[0], xa, w_s + tl0 * HI);
              tmem_ld_wait_fence(xb);
              relu_weighted_acc<32>(acc[0], xb, w_s + tl0 * HI + 32);
            } else {
#pragma unroll
              for (int q = 0; q < TPH; ++q) relu_weighted_acc<HI>(acc[q], xa + q * HI, w_s + (tl0 + q) * HI);
              tmem_ld_wait_fence(xb);
#pragma unroll
              for (int q = 0; q < TPH; ++q)
                relu_weighted_acc<HI>(acc[TPH + q], xb + q * HI, w_s + (tl0 + TPH + q) * HI);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty + b);  // the tensor core may refill this buffer now
#pragma unroll
            for (int q = 0; q < C::TOK_PER_WARP; ++q)
              score[q] = __fmul_rn(__fmul_rn(relu_weighted_finish(acc[q]), qs_s[tl0 + q]), ks);
          }
#pragma unroll
          for (int q = 0; q < C::TOK_PER_WARP; ++q) {
            const int tl = b * C::TB + half * C::TOK_PER_WARP + q;
            const int t = t0 + tl;
            const bool valid = (r0 + tl < bk.rend) && (s <= t);
            if constexpr (kSelect) {
              // a key can only pass if its score reaches the threshold's score
              const uint32_t sk = float_order_key(score[q]);
              const bool maybe = valid && sk >= static_cast<uint32_t>(thr_r[q] >> 32);
              if (__any_sync(0xffffffffu, maybe)) {
                int* cnt = cnt_s + tl * 4 + quarter;
                const int base = base_r[q];
                const uint64_t key = (static_cast<uint64_t>(sk) << 32) | static_cast<uint64_t>(~static_cast<uint32_t>(s));
                const bool pred = maybe && key > thr_r[q];
                const uint32_t m = __ballot_sync(0xffffffffu, pred);
                if (pred)
                  my_cand[static_cast<size_t>(tl) * p.cap + static_cast<size_t>(quarter) * capq + base +
                          __popc(m & lanemask_lt)] = key;
                __syncwarp();
                if (lane == 0 && m) {
                  *cnt = base + __popc(m);
                  if (base + __popc(m) > capq - 32 * C::CHECK_EVERY) atomicOr(cutmask_s, 1 << tl);
                }
              }
            } else {
              if (valid && t >= p.row0 && t < p.row0 + p.nrows)
                p.scores[static_cast<size_t>(t - p.row0) * p.L + s] = score[q];
            }
          }
        }
        if constexpr (kSelect) {
          // Every CHECK_EVERY tiles, cut any list whose sub-list could
          // overflow before the next check (at most 32 appends per sub-list
          // and tile): one histogram pass keeps every key in or above the bin
          // of the k-th largest; if that keeps too many, an exact select
          // keeps exactly k.
          if (spec && i == C::NSAMPLE - 1) {
            // End of the sample: each row's threshold starts at the score of
            // its r-th largest sampled key (keys scoring at least that pass;
            // index bits cleared so equal scores are kept), and the list is
            // emptied: the sampled tiles come round again in order.
            named_bar_sync(1, C::NET);
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
              int above = 0, inb = 0;
              uint64_t floor = histogram_cut<C::NET, 4 * MQ>(v, r, scr_s, et, 1, &above, &inb);
              if (above + inb > r) {
#pragma unroll
                for (int q = 0; q < 4 * MQ; ++q) v[q] = (v[q] >= floor) ? v[q] : 0ull;
                floor = radix_select_floor<C::NET, 4 * MQ>(v, r, scr_s, et, 1);
              }
              if (et == 0) {
                const uint64_t hi = floor >> 32;
                thr_s[tl] = (hi == 0) ? 0ull : (hi << 32) - 1;
              }
              named_bar_sync(1, C::NET);
            }
            if (et < 4 * C::RB) cnt_s[et] = 0;
            if (et == 0) *cutmask_s = 0;
            named_bar_sync(1, C::NET);
            continue;
          }
          if ((i % C::CHECK_EVERY) != C::CHECK_EVERY - 1) continue;
          named_bar_sync(1, C::NET);
          const uint32_t cmask = static_cast<uint32_t>(*cutmask_s);
          if (cmask == 0) continue;
          for (int tl = 0; tl < C::RB; ++tl) {
            const int* cn = cnt_s + tl * 4;
            if ((cmask >> tl) & 1u) {
              uint64_t* row = my_cand + static_cast<size_t>(tl) * p.cap;
              const int n = cn[0] + cn[1] + cn[2] + cn[3];
              uint64_t v[4 * MQ];
              load_sublists<C::NET, MQ>(row, capq, cn, et, v);
              uint64_t floor = 1ull;  // fewer than topk keys: only rebalance the sub-lists
              if (n > p.topk) {
                int above = 0, inb = 0;
                floor = histogram_cut<C::NET, 4 * MQ>(v, p.topk, scr_s, et, 1, &above, &inb);
                if (above + inb > p.cap / 2) {
                  // keys below the boundary bin can go now; exact select on the rest
#pragma unroll
                  for (int i = 0; i < 4 * MQ; ++i) v[i] = (v[i] >= floor) ? v[i] : 0ull;
                  floor = radix_select_floor<C::NET, 4 * MQ>(v, p.topk, scr_s, et, 1);
                }
              }
              store_sublists<C::NET, MQ>(row, capq, cnt_s + tl * 4, v, floor, pos_s, et, 1);
              if (et == 0 && floor - 1 > thr_s[tl]) thr_s[tl] = floor - 1;
              named_bar_sync(1, C::NET);
            }
          }
          // every flagged row was cut; all threads read the mask before the cuts' barriers
          if (et == 0) *cutmask_s = 0;
          named_bar_sync(1, C::NET);
        }
      }
      if (!ok) break;
      if constexpr (kSelect) {
        // exact top-k of each row: the histogram pass finds the boundary bin,
        // a radix select over that bin's keys alone finds the exact cut
        named_bar_sync(1, C::NET);
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
          uint64_t floor = 1ull;  // keep every valid key
          if (n > p.topk) {
            int above = 0, inb = 0;
            floor = histogram_cut<C::NET, 4 * MQ>(v, p.topk, scr_s, et, 1, &above, &inb);
            if (above + inb > p.topk) {
              // the k-th largest lies in the boundary bin: exact select among keys >= its lower edge
#pragma unroll
              for (int i = 0; i < 4 * MQ; ++i) v[i] = (v[i] >= floor) ? v[i] : 0ull;
              floor = radix_select_floor<C::NET, 4 * MQ>(v, p.topk, scr_s, et, 1);
            }
          }
          // write the row's selected keys (unordered) and zero-pad to topk
          uint64_t* dst = p.sel_keys + static_cast<size_t>(r0 + tl) * p.topk;  // row r0 + tl of the output
          int mine = 0;
#pragma unroll
          for (int i = 0; i < 4 * MQ; ++i) mine += (v[i] != 0 && v[i] >= floor) ? 1 : 0;
          int kept = 0;
          int pos = block_exclusive_scan<C::NET>(mine, pos_s, et, 1, &kept);
#pragma unroll
          for (int i = 0; i < 4 * MQ; ++i)
            if (v[i] != 0 && v[i] >= floor) dst[pos++] = v[i];
          for (int i = kept + et; i < p.topk; i += C::NET) dst[i] = 0ull;
        }
        if (redo && et == 0) p.redo_list[atomicAdd(p.redo_count, 1)] = rb;
      }
      named_bar_sync(1, C::NET);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace dsa
