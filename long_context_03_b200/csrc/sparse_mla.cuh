// Sparse MQA attention over the selected rows of the MLA latent cache.
//
// For a query token t with heads h and selected rows S_t ("细粒度词元选择",
// deepseek.csdn.net section 2.2: attention only over the top-k entries {c_s},
// shared by every head; the 576-value latent row of yudonglee.me
// "DeepSeek-V3.2 explained" section 2.4):
//     z[h,s] = scale * Q[t,h,0:576] . C[s,0:576],   s in S_t
//     u[t,h,:] = sum_s softmax_s(z[h,:]) * C[s, 0:512]
// with fp32 softmax and accumulation, bf16 tensor-core inputs and a bf16 output.
//
// The fp32 output tile of one token (128 heads x 512 values) needs all 512
// TMEM columns of an SM, so each token runs on a 2-CTA cluster:
//   CTA 0 (score CTA) keeps all of Q[t] in TMEM (288 columns of bf16 pairs,
//     the A operand of TMEM-sourced MMAs; Q arrives as nine TMA tiles through
//     the same ring as the gathered rows and the MMA warp copies each into
//     TMEM with tcgen05.cp) and computes S = Q C^T for chunks
//     of 128 selected rows (M = 128 heads, N = 128 rows: a full-rate tcgen05
//     shape) into a single 128-column S buffer. The rows are gathered slab by
//     slab (64 values = 128 bytes of each row, 16 KB per slab tile) through a
//     ring, so the 576-wide chunk never has to be resident at once. Its
//     softmax warps (one thread per head) copy their 128 scores of the chunk
//     into registers and hand the S buffer back at once, so the next chunk's
//     QK^T overlaps this chunk's softmax with one buffer. They turn S into
//     bf16 probabilities P with a running
//     reference max that only moves when a chunk exceeds it by more than 2^8
//     (so P <= 256 and the accumulator is rarely rescaled), and ship P, the
//     per-head rescale factors and, after the last chunk, the row sums and
//     maxima to CTA 1 with a bulk shared-memory copy across the cluster.
//   CTA 1 (value CTA) gathers the value part (first 512 values) of the same
//     rows in 32-row sub-tiles, rescales O when told to, and runs O += P V
//     (M = 128 heads, N = 2 x 256 values, K = 16 rows per instruction) into
//     its whole TMEM. Its MMA commit tells CTA 0 directly (multicast commit)
//     that a P buffer is free. After the last chunk it writes u = O / l in
//     bf16 and the log-sum-exp.
// Per 128-row chunk the score CTA issues 36 MMAs of 128x128x16 and the value
// CTA 16 MMAs of 128x256x16: balanced work, both at the tensor core's full
// per-instruction rate. A cluster is persistent over tokens.
//
// Entries idx < 0 are skipped (probability 0). Entries >= the row bound are
// also skipped and reported through the device error word.
#pragma once

#include <type_traits>

#include "dsa_common.cuh"

namespace dsa {

struct MlaCfg {
  static constexpr int D = 576;               // QK dims
  static constexpr int DV = 512;              // value dims
  static constexpr int NK = 128;              // selected rows per chunk (QK^T N)
  static constexpr int M = 128;               // heads per MMA (rows >= Hq are zero)
  static constexpr int NSLAB_QK = D / 64;     // 9 slabs of 64 values (128 B)
  static constexpr int NSLAB_V = DV / 64;     // 8
  static constexpr int SLAB_TILE = NK * 128;  // one slab of a chunk: 128 rows x 128 B = 16 KB
  static constexpr int NSST = 8;              // slab-tile ring depth (score CTA)
  static constexpr int VROWS = 32;            // rows per value sub-tile
  static constexpr int VSLAB = VROWS * 128;   // one slab of a value sub-tile: 4 KB
  static constexpr int V_TILE = NSLAB_V * VSLAB;  // 32 KB
  static constexpr int NVST = 4;              // value sub-tile ring depth (value CTA)
  static constexpr int NSB = 1;               // S buffer in TMEM (the softmax copies it to registers at once)
  static constexpr int NPB = 2;               // P message buffers
  static constexpr int KMAX = 2048;           // largest selection (index row staged in smem)
  static constexpr int P_BYTES = M * NK * 2;  // 32 KB: two 128-byte-swizzled K slabs of 64 rows
  static constexpr int MSG_ALPHA = P_BYTES;           // f32 [128]
  static constexpr int MSG_CTRL = MSG_ALPHA + M * 4;  // u32 [4]: any_rescale
  static constexpr int MSG_L = MSG_CTRL + 16;         // f32 [128] (last chunk only)
  static constexpr int MSG_M = MSG_L + M * 4;         // f32 [128] (last chunk only)
  static constexpr int MSG_BYTES_MID = MSG_L;
  static constexpr int MSG_BYTES_LAST = MSG_M + M * 4;
  static constexpr int MSG_STRIDE = (MSG_BYTES_LAST + 1023) / 1024 * 1024;
  static constexpr int NPROD = 4;             // producer warps
  static constexpr int W_MMA = 4;
  static constexpr int W_SM0 = 5;             // first softmax / epilogue warp
  static constexpr int NTHREADS = 9 * 32;
  static constexpr int Q_COL = 0;             // Q dims 0..575: columns [0, 288)
  static constexpr int S_COL = 288;           // S: columns [288, 416)
  static constexpr uint32_t IDESC_QK = instr_desc(kFmtBF16, M, NK, false, false);
  static constexpr uint32_t IDESC_PV = instr_desc(kFmtBF16, M, 256, false, true);
  // shared memory (offsets from a 1024-aligned base); both CTAs use the same
  // layout so barrier offsets match across the cluster
  static constexpr int OFF_RING = 0;          // score CTA: NSST slab tiles; value CTA: NVST value sub-tiles
  static constexpr int RING_BYTES = (NSST * SLAB_TILE > NVST * V_TILE) ? NSST * SLAB_TILE : NVST * V_TILE;
  static constexpr int OFF_MSG = OFF_RING + RING_BYTES;    // NPB x MSG_STRIDE (staging / receive)
  static constexpr int OFF_IDX = OFF_MSG + NPB * MSG_STRIDE;  // int32 [KMAX]: the token's index row
  static constexpr int OFF_VMASK = OFF_IDX + KMAX * 4;       // score CTA: u32 [2][KMAX/32] validity bits per token
  // value CTA: output staging for the bulk tensor stores, two 2 KB tiles
  // (32 rows x 64 bytes, 64-byte swizzled) per epilogue warp
  static constexpr int EPI_TILE = 2048;
  static constexpr int OFF_EPI = (OFF_VMASK + 2 * (KMAX / 32) * 4 + 1023) / 1024 * 1024;
  static constexpr int OFF_BAR = OFF_EPI + 4 * 2 * EPI_TILE;
  // barriers
  static constexpr int NRING = (NSST > NVST) ? NSST : NVST;
  static constexpr int B_RING_FULL = 0;                     // [NRING]
  static constexpr int B_RING_EMPTY = B_RING_FULL + NRING;  // [NRING]
  static constexpr int B_S_FULL = B_RING_EMPTY + NRING;     // [NSB]  (score CTA)
  static constexpr int B_S_EMPTY = B_S_FULL + NSB;          // [NSB]  (score CTA)
  static constexpr int B_Q_READY = B_S_EMPTY + NSB;         // score CTA (unused: Q arrives through the ring)
  static constexpr int B_Q_FREE = B_Q_READY + 1;            // score CTA
  static constexpr int B_P_FREE = B_Q_FREE + 1;             // [NPB] score CTA, arrived by the value CTA's MMA
  static constexpr int B_P_FULL = B_P_FREE + NPB;           // [NPB] value CTA, completed by the bulk copy
  static constexpr int B_O_READY = B_P_FULL + NPB;          // [NPB] value CTA: correction done
  static constexpr int B_PV_DONE = B_O_READY + NPB;         // value CTA: a token's last PV is done
  static constexpr int B_STAGE = B_PV_DONE + 1;             // score CTA: softmax warps wrote the staging buffer
  static constexpr int B_QUIESCE = B_STAGE + 1;             // value CTA: all PV issued so far complete
  static constexpr int B_MASK_FULL = B_QUIESCE + 1;         // [2] score CTA: producers wrote a token's masks
  static constexpr int B_MASK_FREE = B_MASK_FULL + 2;       // [2] score CTA: softmax is done with them
  static constexpr int B_PSTAGE = B_MASK_FREE + 2;          // both CTAs: the producers' index-row staging
  static constexpr int NBAR = B_PSTAGE + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 32;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(KMAX % NK == 0, "chunks tile the largest selection");
};

struct MlaParams {
  const __nv_bfloat16* q;    // [T, Hq, 576]
  const __nv_bfloat16* kv;   // latent rows; token i reads kv + i*kv_token_stride
  const int32_t* idx;        // [T, K], or null: dense causal, token i takes rows 0..causal_q0 + i
  __nv_bfloat16* out;        // [T, Hq, 512]
  float* lse;                // [T, Hq] or null
  long long kv_token_stride; // elements between consecutive tokens' caches (0: one shared cache)
  int rows;                  // valid row bound of a token's cache
  int T, Hq, K;
  int causal_q0;             // position of token 0 when idx is null
  // Paged latent cache (the kernel's paged instance): logical row r of token i is
  // physical row block_table[i * bt_stride + (r >> page_shift)] * page + (r & (page - 1))
  // of kv (a pool of pool_rows rows); bt_stride 0 shares one table row.
  const int32_t* block_table;
  int bt_stride, page_shift, pool_rows;
  // Packed batch (cu_seqlens, device arrays): when seq_cu_q is set, token i
  // belongs to the sequence b with seq_cu_q[b] <= i < seq_cu_q[b+1] and reads
  // kv rows seq_cu_k[b] .. seq_cu_k[b+1]-1 (its indices are local to the
  // sequence); rows then holds the packed cache's row count, and every
  // sequence's rows are clamped into it.
  const int32_t* seq_cu_q;
  const int32_t* seq_cu_k;
  int nseq;
  float scale_log2;          // softmax scale * log2(e)
  // Split selections (flash-decoding): when part is set, the T x nchunk
  // (token, 128-entry chunk) units are cut into one contiguous range per
  // cluster, so a token's chunks may be spread over several clusters. A
  // cluster that holds only part of a token writes that part's unnormalised
  // fp32 output and its softmax statistics to a partial slot (see
  // mla_part_slot) instead of `out`; mla_combine_kernel merges the parts.
  float* part;
};

// A partial slot: O[128 heads][512] f32 (softmax numerators, scaled by
// 2^-m), then m[128] (reference maxima, log2 units) and l[128] (row sums).
constexpr int kMlaPartFloats = 128 * 512 + 2 * 128;

// First unit of cluster g when U units are cut into G contiguous ranges.
__host__ __device__ __forceinline__ long long mla_unit_start(int g, long long U, int G) {
  return (static_cast<long long>(g) * U) / G;
}
// The cluster whose range holds unit u.
__host__ __device__ __forceinline__ int mla_unit_owner(long long u, long long U, int G) {
  return static_cast<int>(((u + 1) * G - 1) / U);
}

// One piece of work of a cluster: token tk, chunks [c0, c1). slot < 0: the
// cluster holds the whole token and writes its output; else the partial slot
// it writes: 2g for its first piece, 2g + 1 for its last.
struct MlaSeg {
  int tk, c0, c1, slot;
};
// The pieces of cluster g in order. Whole tokens g, g + G, ... without
// splitting; the range [start(g), start(g + 1)) of (token, chunk) units with it.
struct MlaSegIter {
  int u, u0, u1;  // units (T * nchunk < 2^31, checked by the host)
  int g, G, nchunk, T;
  bool split;
  __device__ __forceinline__ MlaSegIter(const MlaParams& p, int g_, int G_, int nchunk_)
      : g(g_), G(G_), nchunk(nchunk_), T(p.T), split(p.part != nullptr) {
    if (split) {
      const long long U = static_cast<long long>(p.T) * nchunk;
      u0 = static_cast<int>(mla_unit_start(g, U, G));
      u1 = static_cast<int>(mla_unit_start(g + 1, U, G));
      u = u0;
    } else {
      u = g;
      u0 = u1 = 0;
    }
  }
  __device__ __forceinline__ bool next(MlaSeg& s) {
    if (split) {
      if (u >= u1) return false;
      s.tk = u / nchunk;
      s.c0 = u - s.tk * nchunk;
      s.c1 = min(nchunk, s.c0 + (u1 - u));
      s.slot = (s.c0 == 0 && s.c1 == nchunk) ? -1 : (u == u0 ? 2 * g : 2 * g + 1);
      u += s.c1 - s.c0;
      return true;
    }
    if (u >= T) return false;
    s.tk = u;
    s.c0 = 0;
    s.c1 = nchunk;
    s.slot = -1;
    u += G;
    return true;
  }
  // token of the piece next() returns next, or -1 at the end
  __device__ __forceinline__ int next_token() const {
    if (split) return u < u1 ? u / nchunk : -1;
    return u < T ? u : -1;
  }
  // P messages (one per chunk) this cluster sends, and whether message i
  // is the last chunk of its piece (it then carries the row sums and maxima)
  __device__ __forceinline__ int messages() const {
    return split ? u1 - u0 : (g < T ? ((T - 1 - g) / G + 1) * nchunk : 0);
  }
  __device__ __forceinline__ bool last_of_piece(int i) const {
    if (!split) return (i % nchunk) == nchunk - 1;
    const int uu = u0 + i;
    return (uu % nchunk) == nchunk - 1 || uu == u1 - 1;
  }
};

// First row and row count of token tk's cache.
__device__ __forceinline__ void token_cache(const MlaParams& p, int tk, const __nv_bfloat16*& kv_tok, int& rows) {
  if (p.seq_cu_q) {
    int lo = 0, hi = p.nseq - 1;  // the last sequence whose first query is at or before tk
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(p.seq_cu_q + mid) <= tk) lo = mid;
      else hi = mid - 1;
    }
    const int k0 = min(max(__ldg(p.seq_cu_k + lo), 0), p.rows);
    const int k1 = min(max(__ldg(p.seq_cu_k + lo + 1), k0), p.rows);
    kv_tok = p.kv + static_cast<long long>(k0) * MlaCfg::D;
    rows = k1 - k0;
  } else {
    kv_tok = p.kv + tk * p.kv_token_stride;
    rows = p.rows;
  }
}

// Bulk copy local shared memory -> a cluster peer's shared memory, completing
// (complete_tx) on the peer's mbarrier. Addresses 16-byte aligned, size % 16 == 0.
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst_cluster, uint32_t src_cta, uint32_t bytes,
                                                  uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst_cluster),
      "r"(src_cta), "r"(bytes), "r"(bar_cluster)
      : "memory");
}
// Commit that arrives on the barrier at the same offset in each CTA of `mask`.
__device__ __forceinline__ void tc_commit_mc(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}

// 2^x with the hardware approximation (relative error a few ulp; P is
// rounded to bf16 afterwards). ex2 of -inf is +0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Row index of selection entry e, or -1 when absent / outside the cache.
__device__ __forceinline__ int checked_row(const int32_t* idx_s, int e, int K, int rows) {
  int row = (e < K) ? idx_s[e] : -1;
  if (row >= rows) {
    set_device_error(kErrBadIndex, 0);
    row = -1;
  }
  return row;
}

// Score CTA: the 8 rows (r = ptid/8 + 16k) this thread copies for chunk j,
// as byte pointers to the rows (absent rows point at row 0 and copy zeros).
// Paged cache: address of the latent row a token's (checked) logical row
// points to through the token's page table; null when the row is absent or
// the page leads outside the pool (reported as a bad index).
__device__ __forceinline__ const char* paged_row(const MlaParams& p, int tk, int row) {
  if (row < 0) return nullptr;
  const int page = p.block_table[static_cast<long long>(tk) * p.bt_stride + (row >> p.page_shift)];
  const long long phys = (static_cast<long long>(page) << p.page_shift) + (row & ((1 << p.page_shift) - 1));
  if (page < 0 || phys >= p.pool_rows) {
    set_device_error(kErrBadIndex, 1);
    return nullptr;
  }
  return reinterpret_cast<const char*>(p.kv + phys * MlaCfg::D);
}

struct ChunkRows {
  const char* src[8];
  uint32_t valid;  // bit k: row k present
};
template <bool kPaged>
__device__ __forceinline__ ChunkRows chunk_rows(const MlaParams& p, const __nv_bfloat16* __restrict__ kv_tok, int tk,
                                                const int32_t* idx_s, int j,
                                                int K, int rows, int ptid) {
  ChunkRows cr;
  cr.valid = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int r = (ptid >> 3) + 16 * k;
    const int row = checked_row(idx_s, j * MlaCfg::NK + r, K, rows);
    if constexpr (kPaged) {
      const char* src = paged_row(p, tk, row);
      // absent rows copy zeros (source size 0); any valid address serves
      cr.src[k] = (src ? src : reinterpret_cast<const char*>(p.kv)) + (ptid & 7) * 16;
      cr.valid |= (src ? 1u : 0u) << k;
    } else {
      cr.src[k] = reinterpret_cast<const char*>(kv_tok + static_cast<long long>(row >= 0 ? row : 0) * MlaCfg::D) +
                  (ptid & 7) * 16;
      cr.valid |= (row >= 0 ? 1u : 0u) << k;
    }
  }
  return cr;
}
// Slab s (values 64s..64s+63) of the chunk's 128 rows into a 16 KB
// 128-byte-swizzled tile: row r at r*128, 16-byte chunk c at c ^ (r & 7).
// Eight consecutive threads copy one row's 128 bytes, so each warp-wide copy
// covers four whole row segments.
__device__ __forceinline__ void gather_slab_tile(uint32_t tile, const ChunkRows& cr, int s, int ptid) {
  const int c = ptid & 7;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int r = (ptid >> 3) + 16 * k;
    cp_async_16_zfill(tile + r * 128 + ((c ^ (r & 7)) << 4), cr.src[k] + s * 128, (cr.valid >> k) & 1u);
  }
}

// Value CTA: rows [j*128 + u*32, +32) of the selection, first 512 values, into
// a 32 KB sub-tile: slab s at s*4096, row r at r*128, chunk c at c ^ (r & 7).
// Eight consecutive threads copy one (row, slab) segment of 128 bytes; each
// group of eight handles rows g and g+16 across all eight slabs, so a thread
// looks up two row indices per sub-tile.
template <bool kPaged>
__device__ __forceinline__ void gather_value_tile(uint32_t tile, const MlaParams& p,
                                                  const __nv_bfloat16* __restrict__ kv_tok, int tk,
                                                  const int32_t* idx_s, int j, int u, int K, int rows, int ptid) {
  const int c = ptid & 7;
  const int g = ptid >> 3;  // 0..15
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = g + 16 * half;
    const int row = checked_row(idx_s, j * MlaCfg::NK + u * MlaCfg::VROWS + r, K, rows);
    const char* src;
    bool present;
    if constexpr (kPaged) {
      const char* rp = paged_row(p, tk, row);
      present = rp != nullptr;
      src = (rp ? rp : reinterpret_cast<const char*>(p.kv)) + c * 16;
    } else {
      present = row >= 0;
      src = reinterpret_cast<const char*>(kv_tok + static_cast<long long>(row >= 0 ? row : 0) * MlaCfg::D) + c * 16;
    }
#pragma unroll
    for (int sl = 0; sl < 8; ++sl)
      cp_async_16_zfill(tile + sl * MlaCfg::VSLAB + r * 128 + ((c ^ (r & 7)) << 4), src + sl * 128, present);
  }
}

// The producer warps copy a token's index row into shared memory once. The
// 128 producer threads of a CTA meet twice per token on the mbarrier
// `stage` (everyone is done with the previous row; the new row is written),
// with bounded waits, so a producer that gives up never leaves the others
// waiting. Without an index row (dense causal mode) entry e is row e for
// e <= pos, else absent. False once the CTA aborted.
__device__ __forceinline__ bool stage_index_row(int32_t* idx_s, const int32_t* __restrict__ idx_tok, int K, int ptid,
                                                int pos, uint64_t* stage, uint32_t& phase, AbortFlag ab) {
  mbar_arrive(stage);
  if (!mbar_wait(stage, phase, ab, 26)) return false;  // everyone is done with the previous row
  phase ^= 1u;
  if (idx_tok == nullptr) {
    for (int i = ptid; i < K; i += MlaCfg::NPROD * 32) idx_s[i] = (i <= pos) ? i : -1;
  } else if ((K & 3) == 0 && (reinterpret_cast<uintptr_t>(idx_tok) & 15) == 0) {
    const int4* src = reinterpret_cast<const int4*>(idx_tok);
    int4* dst = reinterpret_cast<int4*>(idx_s);
    for (int i = ptid; i < K / 4; i += MlaCfg::NPROD * 32) dst[i] = __ldg(src + i);
  } else {
    for (int i = ptid; i < K; i += MlaCfg::NPROD * 32) idx_s[i] = __ldg(idx_tok + i);
  }
  mbar_arrive(stage);
  if (!mbar_wait(stage, phase, ab, 27)) return false;
  phase ^= 1u;
  return true;
}

// tmO: out [T, Hq, 512] bf16 as {512, Hq, T}, boxes of 32 values x 32 heads,
// 64-byte swizzled. tmP (split selections only): the partial slots'
// numerators as {512, Hq, slots} f32 with a slot stride of kMlaPartFloats,
// boxes of 16 values x 32 heads, 64-byte swizzled.
template <bool kPaged>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(MlaCfg::NTHREADS, 1)
    sparse_mla_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                      const __grid_constant__ CUtensorMap tmP, const MlaParams p) {
  using C = MlaCfg;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  int* abort_s = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);
  int* rescale_s = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);
  int32_t* idx_s = reinterpret_cast<int32_t*>(smem + C::OFF_IDX);
  uint32_t* vmask_s = reinterpret_cast<uint32_t*>(smem + C::OFF_VMASK);
  const AbortFlag ab{abort_s};
  const uint32_t rank = cluster_ctarank();
  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int cluster_id = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;
  const int nchunk = (p.K + C::NK - 1) / C::NK;
  const MlaSegIter segs0(p, cluster_id, nclusters, nchunk);  // every role walks its own copy
  const int total_msgs = segs0.messages();                    // messages this cluster sends

  if (threadIdx.x == 0) {
    *abort_s = 0;
    rescale_s[0] = 0;
    rescale_s[1] = 0;
    for (int i = 0; i < C::NRING; ++i) {
      mbar_init(bars + C::B_RING_FULL + i, C::NPROD * 32);
      mbar_init(bars + C::B_RING_EMPTY + i, 1);
    }
    for (int i = 0; i < C::NSB; ++i) {
      mbar_init(bars + C::B_S_FULL + i, 1);
      mbar_init(bars + C::B_S_EMPTY + i, 4);
    }
    mbar_init(bars + C::B_Q_READY, 4);
    mbar_init(bars + C::B_Q_FREE, 1);
    for (int i = 0; i < C::NPB; ++i) {
      mbar_init(bars + C::B_P_FREE + i, 1);
      mbar_init(bars + C::B_P_FULL + i, 1);
      mbar_init(bars + C::B_O_READY + i, 4);
    }
    mbar_init(bars + C::B_PV_DONE, 1);
    mbar_init(bars + C::B_STAGE, 4);
    mbar_init(bars + C::B_QUIESCE, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bars + C::B_MASK_FULL + i, C::NPROD);
      mbar_init(bars + C::B_MASK_FREE + i, 4);
    }
    mbar_init(bars + C::B_PSTAGE, C::NPROD * 32);
    fence_mbar_init();
  }
  if (warp == C::W_MMA) tmem_alloc(tmem_base_s, 512);
  __syncthreads();
  griddep_launch_dependents();  // a combine step may be scheduled now; it waits for this grid
  // Value CTA: arm the first use of each P receive buffer before the peer can send.
  if (rank == 1 && threadIdx.x == 0) {
    for (int i = 0; i < C::NPB && i < total_msgs; ++i) {
      const bool last = segs0.last_of_piece(i);
      mbar_arrive_expect_tx(bars + C::B_P_FULL + i, last ? C::MSG_BYTES_LAST : C::MSG_BYTES_MID);
    }
  }
  cluster_sync_all();
  // Launched as a programmatic dependent, the kernel got here (barriers,
  // TMEM, cluster) while the previous kernel was finishing; nothing of
  // global memory is touched before this wait.
  griddep_wait();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_s;
  const uint32_t ring = smem_u32(smem + C::OFF_RING);
  const uint32_t msg = smem_u32(smem + C::OFF_MSG);

  if (rank == 0) {
    // =========================== score CTA ===========================
    if (warp < C::NPROD) {
      const int ptid = threadIdx.x;
      int slot = 0;
      uint32_t ph = 1;
      int n = 0;  // tokens done by this cluster
      uint32_t stage_ph = 0;  // phase of the producers' staging barrier
      // thread 0: where the last token's Q tiles start in the ring and how
      // many it loaded, so that an abort can still wait for its copies in flight
      int q_slot0 = 0;
      uint32_t q_ph0 = 1;
      int q_issued = 0;
      MlaSegIter segs = segs0;
      MlaSeg sg;
      for (; segs.next(sg); ++n) {
        const int tk = sg.tk;
        const __nv_bfloat16* kv_tok;
        int trows;
        token_cache(p, tk, kv_tok, trows);
        bool ok = true;
        // Q[tk] first, before the index row (it does not depend on it): nine
        // 16 KB tiles (128 heads x 64 values, 128-byte swizzled, heads >= Hq
        // zero) through the ring by TMA; the MMA warp copies them into TMEM.
        // Thread 0 arms the slot with the bytes, the other producer threads
        // arrive, as for a gathered tile.
        q_slot0 = slot;
        q_ph0 = ph;
        q_issued = 0;
        for (int i = 0; i < C::NSLAB_QK; ++i) {
          if (!mbar_wait(bars + C::B_RING_EMPTY + slot, ph, ab, 29)) { ok = false; break; }
          if (ptid == 0) {
            mbar_arrive_expect_tx(bars + C::B_RING_FULL + slot, C::SLAB_TILE);
            tma_load_3d(smem + C::OFF_RING + slot * C::SLAB_TILE, &tmQ, bars + C::B_RING_FULL + slot, i * 64, 0, tk);
            q_issued = i + 1;
          } else {
            mbar_arrive(bars + C::B_RING_FULL + slot);
          }
          if (++slot == C::NSST) { slot = 0; ph ^= 1; }
        }
        // the softmax warps are done with this mask buffer (two pieces back)
        const int mb = n & 1;
        if (!ok || !mbar_wait(bars + C::B_MASK_FREE + mb, ((n >> 1) & 1) ^ 1, ab, 30)) break;
        if (!stage_index_row(idx_s, p.idx ? p.idx + static_cast<size_t>(tk) * p.K : nullptr, p.K, ptid,
                             p.causal_q0 + tk, bars + C::B_PSTAGE, stage_ph, ab))
          break;
        // validity bits of every selection entry, 32 per word (entry e -> word e/32)
        for (int wd = static_cast<int>(warp); wd < nchunk * (C::NK / 32); wd += C::NPROD) {
          const int e = wd * 32 + static_cast<int>(lane);
          const int row = (e < p.K) ? idx_s[e] : -1;
          bool present = row >= 0 && row < trows;
          if (kPaged && present) {  // paged: the page must lie inside the pool
            const int page = p.block_table[static_cast<long long>(tk) * p.bt_stride + (row >> p.page_shift)];
            present = page >= 0 && (static_cast<long long>(page) << p.page_shift) +
                                           (row & ((1 << p.page_shift) - 1)) < p.pool_rows;
          }
          const uint32_t m = __ballot_sync(0xffffffffu, present);
          if (lane == 0) vmask_s[mb * (C::KMAX / 32) + wd] = m;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + C::B_MASK_FULL + mb);
        for (int j = sg.c0; j < sg.c1 && ok; ++j) {
          const ChunkRows cr = chunk_rows<kPaged>(p, kv_tok, tk, idx_s, j, p.K, trows, ptid);
          for (int i = 0; i < C::NSLAB_QK; ++i) {
            if (!mbar_wait(bars + C::B_RING_EMPTY + slot, ph, ab, 31)) { ok = false; break; }
            gather_slab_tile(ring + slot * C::SLAB_TILE, cr, i, ptid);
            cp_async_mbar_arrive(bars + C::B_RING_FULL + slot);
            if (++slot == C::NSST) { slot = 0; ph ^= 1; }
          }
        }
        if (!ok) break;
      }
      asm volatile("cp.async.wait_all;" ::: "memory");
      if (ptid == 0 && ab.raised()) {
        // aborted: the token's Q tiles may still be landing in the ring; wait
        // for them (bounded, whatever the abort flag says) before leaving
        int never = 0;
        const AbortFlag no_abort{&never};
        // only the latest use of each slot can still be in flight (a tile that
        // reused a slot was issued after the earlier one had been consumed)
        for (int i = (q_issued > C::NSST ? q_issued - C::NSST : 0); i < q_issued; ++i) {
          const int pos = q_slot0 + i;  // ring position of Q tile i; the parity flips at each wrap
          const uint32_t full_par = (q_ph0 ^ static_cast<uint32_t>((pos / C::NSST) & 1)) ^ 1u;
          mbar_wait(bars + C::B_RING_FULL + pos % C::NSST, full_par, no_abort, 28);
        }
      }
    } else if (warp == C::W_MMA) {
      // The whole warp runs the loop and waits converged; one elected lane
      // issues each slab's MMAs together with every commit that covers them.
      int slot = 0;
      uint32_t ph = 0;
      uint32_t sph = 1;
      uint32_t qfree_ph = 1;
      bool ok = true;
      MlaSegIter segs = segs0;
      MlaSeg sg;
      while (ok && segs.next(sg)) {
        // Q[tk] into TMEM once the previous piece's QK^T has read the old Q
        if (!mbar_wait_warp(bars + C::B_Q_FREE, qfree_ph, ab, 32)) break;
        qfree_ph ^= 1;
        tc_fence_after();
        for (int i = 0; i < C::NSLAB_QK; ++i) {
          if (!mbar_wait_warp(bars + C::B_RING_FULL + slot, ph, ab, 37)) { ok = false; break; }
          tc_fence_after();
          if (elect_one()) {
            const uint32_t tile = ring + slot * C::SLAB_TILE;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc_cp_128x256b(tmem + C::Q_COL + (4 * i + kk) * 8, smem_desc(tile + kk * 32, 16, 1024, kSw128));
            tc_commit(bars + C::B_RING_EMPTY + slot);
          }
          __syncwarp();
          if (++slot == C::NSST) { slot = 0; ph ^= 1; }
        }
        if (!ok) break;
        for (int j = sg.c0; j < sg.c1 && ok; ++j) {
          if (!mbar_wait_warp(bars + C::B_S_EMPTY, sph, ab, 34)) { ok = false; break; }
          sph ^= 1;
          tc_fence_after();
          const uint32_t d = tmem + C::S_COL;
          for (int i = 0; i < C::NSLAB_QK; ++i) {
            if (!mbar_wait_warp(bars + C::B_RING_FULL + slot, ph, ab, 33)) { ok = false; break; }
            tc_fence_after();
            if (elect_one()) {
              const uint32_t tile = ring + slot * C::SLAB_TILE;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t bd = smem_desc(tile + kk * 32, 16, 1024, kSw128);
                mma_bf16_ts(d, tmem + C::Q_COL + (4 * i + kk) * 8, bd, C::IDESC_QK, (i > 0 || kk > 0) ? 1u : 0u);
              }
              tc_commit(bars + C::B_RING_EMPTY + slot);
              if (i == C::NSLAB_QK - 1) {
                tc_commit(bars + C::B_S_FULL);
                if (j == sg.c1 - 1) tc_commit(bars + C::B_Q_FREE);
              }
            }
            __syncwarp();
            if (++slot == C::NSST) { slot = 0; ph ^= 1; }
          }
          if (!ok) break;
        }
      }
    } else {
      // softmax warps: thread = head row (TMEM lane)
      const int quarter = static_cast<int>(warp & 3);
      const int h = quarter * 32 + static_cast<int>(lane);
      const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
      const uint32_t peer_msg = map_to_peer(msg, 1);
      const uint32_t peer_pfull = map_to_peer(smem_u32(bars + C::B_P_FULL), 1);
      uint32_t sph = 0;
      int pb = 0;
      uint32_t pfree_ph = 1;
      uint32_t stage_ph = 0;
      bool ok = true;
      int n = 0;  // pieces done by this cluster
      MlaSegIter segs = segs0;
      MlaSeg sg;
      for (; ok && segs.next(sg); ++n) {
        // Q[tk] reaches TMEM through the ring (TMA + tcgen05.cp by the MMA warp)
        const int ntk = segs.next_token();
        if (h == 0 && ntk >= 0 && ntk != sg.tk) {
          // warm L2 with the next piece's queries
          const char* nq = reinterpret_cast<const char*>(p.q + static_cast<size_t>(ntk) * p.Hq * C::D);
          const uint32_t qbytes = static_cast<uint32_t>(p.Hq) * C::D * 2;
          asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(nq), "r"(qbytes) : "memory");
        }
        float m_ref = -INFINITY;
        float l_sum = 0.f;
        // validity bits of this token's selection, staged by the producer warps
        const int mb = n & 1;
        if (!mbar_wait(bars + C::B_MASK_FULL + mb, (n >> 1) & 1, ab, 39)) break;
        const uint4* vm_tok = reinterpret_cast<const uint4*>(vmask_s + mb * (C::KMAX / 32));
        for (int j = sg.c0; j < sg.c1; ++j) {
          // validity of the chunk's 128 entries (the same for every head)
          const uint4 vm4 = vm_tok[j];
          const uint32_t vmask[4] = {vm4.x, vm4.y, vm4.z, vm4.w};
          if (!mbar_wait(bars + C::B_S_FULL, sph, ab, 36)) { ok = false; break; }
          sph ^= 1;
          tc_fence_after();
          // this head's 128 scores of the chunk into registers; the S buffer
          // goes back to the tensor core at once, so the next chunk's QK^T
          // overlaps this chunk's softmax with a single S buffer in TMEM
          const uint32_t s_addr = tmem + lane_addr + C::S_COL;
          uint32_t sr[4][32];
#pragma unroll
          for (int g = 0; g < 4; ++g) tmem_ld32_nowait(s_addr + g * 32, sr[g]);
#pragma unroll
          for (int g = 0; g < 4; ++g) tmem_ld_wait_fence(sr[g]);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bars + C::B_S_EMPTY);
          // pass 1: the chunk's max. Invalid entries (absent rows, gathered
          // as zeros) are masked to -inf; a chunk without any is the common
          // case and skips the masking.
          const bool all_valid = (vmask[0] & vmask[1] & vmask[2] & vmask[3]) == 0xffffffffu;
          float mc = -INFINITY;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            if (all_valid) {
#pragma unroll
              for (int c = 0; c < 32; ++c) mc = fmaxf(mc, __uint_as_float(sr[g][c]));
            } else {
#pragma unroll
              for (int c = 0; c < 32; ++c)
                if ((vmask[g] >> c) & 1u) mc = fmaxf(mc, __uint_as_float(sr[g][c]));
            }
          }
          mc = (mc == -INFINITY) ? -INFINITY : mc * p.scale_log2;
          float alpha = 1.f;
          if (mc > -INFINITY && (m_ref == -INFINITY || mc > m_ref + 8.f)) {
            alpha = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - mc);
            m_ref = mc;
            l_sum *= alpha;
          }
          const bool last = (j == sg.c1 - 1);
          // staging buffer pb is free once the value CTA's MMA consumed its previous message
          if (!mbar_wait(bars + C::B_P_FREE + pb, pfree_ph, ab, 37)) { ok = false; break; }
          uint8_t* st = smem + C::OFF_MSG + pb * C::MSG_STRIDE;
          // pass 2: p = 2^(s*scale*log2e - m_ref), packed to bf16 into the
          // swizzled P rows; eight independent partial row sums
          const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
          float part[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const uint32_t vm = all_valid ? 0xffffffffu : vmask[g];
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {  // 4 chunks of 8 keys = 16 bytes of the P row
              uint32_t pk[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int c = c4 * 8 + 2 * i;
                float p0 = fast_exp2(__fmaf_rn(__uint_as_float(sr[g][c]), p.scale_log2, neg_m));
                float p1 = fast_exp2(__fmaf_rn(__uint_as_float(sr[g][c + 1]), p.scale_log2, neg_m));
                p0 = ((vm >> c) & 1u) ? p0 : 0.f;
                p1 = ((vm >> (c + 1)) & 1u) ? p1 : 0.f;
                pk[i] = pack_bf16x2(p0, p1);
                part[2 * i] += p0;
                part[2 * i + 1] += p1;
              }
              const int c8 = g * 4 + c4;  // 16-byte chunk index within the 256-byte row
              const int kslab = c8 >> 3, cc = c8 & 7;
              *reinterpret_cast<uint4*>(st + kslab * 16384 + h * 128 + ((cc ^ (h & 7)) << 4)) =
                  make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
          }
          l_sum += ((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7]));
          reinterpret_cast<float*>(st + C::MSG_ALPHA)[h] = alpha;
          const uint32_t any_rs = __ballot_sync(0xffffffffu, alpha != 1.f);
          if (lane == 0 && any_rs) atomicOr(rescale_s + (pb & 1), 1);
          if (last) {
            reinterpret_cast<float*>(st + C::MSG_L)[h] = l_sum;
            reinterpret_cast<float*>(st + C::MSG_M)[h] = m_ref;
          }
          fence_async_shared();
          __syncwarp();
          if (lane == 0) mbar_arrive(bars + C::B_STAGE);
          if (warp == C::W_SM0 && lane == 0) {
            // all four softmax warps have written the staging buffer
            if (!mbar_wait(bars + C::B_STAGE, stage_ph, ab, 38)) { ok = false; }
            if (ok) {
              uint32_t* ctrl = reinterpret_cast<uint32_t*>(st + C::MSG_CTRL);
              ctrl[0] = static_cast<uint32_t>(rescale_s[pb & 1]);
              rescale_s[pb & 1] = 0;
              fence_async_shared();
              const uint32_t bytes = last ? C::MSG_BYTES_LAST : C::MSG_BYTES_MID;
              bulk_copy_to_peer(peer_msg + pb * C::MSG_STRIDE, smem_u32(st), bytes, peer_pfull + pb * 8);
            }
          }
          stage_ph ^= 1;
          if (++pb == C::NPB) { pb = 0; pfree_ph ^= 1; }
          if (!ok) break;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + C::B_MASK_FREE + mb);
      }
    }
  } else {
    // =========================== value CTA ===========================
    if (warp < C::NPROD) {
      const int ptid = threadIdx.x;
      int slot = 0;
      uint32_t ph = 1;
      uint32_t stage_ph = 0;  // phase of the producers' staging barrier
      MlaSegIter segs = segs0;
      MlaSeg sg;
      while (segs.next(sg)) {
        const int tk = sg.tk;
        const __nv_bfloat16* kv_tok;
        int trows;
        token_cache(p, tk, kv_tok, trows);
        if (!stage_index_row(idx_s, p.idx ? p.idx + static_cast<size_t>(tk) * p.K : nullptr, p.K, ptid,
                             p.causal_q0 + tk, bars + C::B_PSTAGE, stage_ph, ab))
          break;
        bool ok = true;
        for (int j = sg.c0; j < sg.c1 && ok; ++j) {
          for (int u = 0; u < C::NK / C::VROWS; ++u) {
            if (!mbar_wait(bars + C::B_RING_EMPTY + slot, ph, ab, 41)) { ok = false; break; }
            gather_value_tile<kPaged>(ring + slot * C::V_TILE, p, kv_tok, tk, idx_s, j, u, p.K, trows, ptid);
            cp_async_mbar_arrive(bars + C::B_RING_FULL + slot);
            if (++slot == C::NVST) { slot = 0; ph ^= 1; }
          }
        }
        if (!ok) break;
      }
      asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp == C::W_MMA) {
      // whole warp waits converged; one elected lane issues and commits
      int slot = 0;
      uint32_t ph = 0;
      int pb = 0;
      uint32_t pph = 0;
      int use = 0;  // messages consumed, to arm the receive barriers ahead
      bool ok = true;
      MlaSegIter segs = segs0;
      MlaSeg sg;
      while (ok && segs.next(sg)) {
        for (int j = sg.c0; j < sg.c1 && ok; ++j) {
          if (!mbar_wait_warp(bars + C::B_P_FULL + pb, pph, ab, 43)) { ok = false; break; }
          const uint32_t any_rs =
              reinterpret_cast<const volatile uint32_t*>(smem + C::OFF_MSG + pb * C::MSG_STRIDE + C::MSG_CTRL)[0];
          // A rescale needs O quiescent: commit everything issued so far to
          // QUIESCE; the correction warps wait on it, rescale, then signal O_READY.
          if (any_rs && j > sg.c0) {
            if (elect_one()) tc_commit(bars + C::B_QUIESCE);
            __syncwarp();
          }
          if (!mbar_wait_warp(bars + C::B_O_READY + pb, pph, ab, 44)) { ok = false; break; }
          tc_fence_after();
          const uint32_t pbase = msg + pb * C::MSG_STRIDE;
          for (int u = 0; u < C::NK / C::VROWS; ++u) {
            if (!mbar_wait_warp(bars + C::B_RING_FULL + slot, ph, ab, 42)) { ok = false; break; }
            tc_fence_after();
            if (elect_one()) {
              const uint32_t vbase = ring + slot * C::V_TILE;
#pragma unroll
              for (int kk = 0; kk < C::VROWS / 16; ++kk) {
                const int ko = u * C::VROWS + kk * 16;  // first key of this k-step within the chunk
                const uint64_t ad = smem_desc(pbase + (ko >> 6) * 16384 + ((ko & 63) >> 4) * 32, 16, 1024, kSw128);
#pragma unroll
                for (int nh = 0; nh < 2; ++nh) {
                  const uint64_t bd = smem_desc(vbase + nh * 4 * C::VSLAB + kk * 2048, C::VSLAB, 1024, kSw128);
                  mma_bf16_ss(tmem + nh * 256, ad, bd, C::IDESC_PV, (j > sg.c0 || u > 0 || kk > 0) ? 1u : 0u);
                }
              }
              tc_commit(bars + C::B_RING_EMPTY + slot);
              if (u == C::NK / C::VROWS - 1) {
                tc_commit_mc(bars + C::B_P_FREE + pb, 0x1);  // the score CTA's buffer pb is free
                if (j == sg.c1 - 1) tc_commit(bars + C::B_PV_DONE);
                // re-arm this receive buffer for message use + NPB
                const int nxt = use + C::NPB;
                if (nxt < total_msgs) {
                  const bool lastm = segs0.last_of_piece(nxt);
                  mbar_arrive_expect_tx(bars + C::B_P_FULL + pb, lastm ? C::MSG_BYTES_LAST : C::MSG_BYTES_MID);
                }
              }
            }
            __syncwarp();
            if (++slot == C::NVST) { slot = 0; ph ^= 1; }
          }
          if (!ok) break;
          ++use;
          if (++pb == C::NPB) { pb = 0; pph ^= 1; }
        }
      }
    } else {
      // correction + epilogue warps: thread = head row
      const int quarter = static_cast<int>(warp & 3);
      const int h = quarter * 32 + static_cast<int>(lane);
      const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
      int pb = 0;
      uint32_t pph = 0;
      uint32_t pv_ph = 0;
      uint32_t qz_ph = 0;
      uint32_t epi_n = 0;  // staging tiles used by this warp (tile epi_n & 1 is next)
      bool ok = true;
      MlaSegIter segs = segs0;
      MlaSeg sg;
      while (ok && segs.next(sg)) {
        const int tk = sg.tk;
        float l_fin = 0.f, m_fin = -INFINITY;
        for (int j = sg.c0; j < sg.c1; ++j) {
          if (!mbar_wait(bars + C::B_P_FULL + pb, pph, ab, 45)) { ok = false; break; }
          const uint8_t* mb = smem + C::OFF_MSG + pb * C::MSG_STRIDE;
          const uint32_t any_rs = reinterpret_cast<const volatile uint32_t*>(mb + C::MSG_CTRL)[0];
          if (j == sg.c1 - 1) {
            l_fin = reinterpret_cast<const float*>(mb + C::MSG_L)[h];
            m_fin = reinterpret_cast<const float*>(mb + C::MSG_M)[h];
          }
          if (any_rs && j > sg.c0) {
            const float alpha = reinterpret_cast<const float*>(mb + C::MSG_ALPHA)[h];
            if (!mbar_wait(bars + C::B_QUIESCE, qz_ph, ab, 46)) { ok = false; break; }
            qz_ph ^= 1;
            tc_fence_after();
#pragma unroll 1
            for (int cb = 0; cb < C::DV / 32; ++cb) {
              uint32_t r[32];
              tmem_ld32(tmem + lane_addr + cb * 32, r);
#pragma unroll
              for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * alpha);
              tmem_st32(tmem + lane_addr + cb * 32, r);
            }
            tmem_st_wait();
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bars + C::B_O_READY + pb);
          if (++pb == C::NPB) { pb = 0; pph ^= 1; }
        }
        if (!ok) break;
        // the token's last PV has landed in TMEM
        if (!mbar_wait(bars + C::B_PV_DONE, pv_ph, ab, 47)) break;
        pv_ph ^= 1;
        tc_fence_after();
        // The output leaves by bulk tensor stores: a warp writes 64-byte row
        // segments of its 32 rows (heads) into one of its two staging tiles
        // (64-byte swizzle: 16-byte chunk c of row r at c ^ ((r >> 1) & 3)),
        // and one lane stores the tile, so the global writes take no
        // load/store-unit issue and each staging tile is reused once its
        // store has read it. A whole token gets u = O / l in bf16 (32 values
        // per tile); part of a token (a split selection) gets its
        // unnormalised fp32 numerators (16 values per tile) in the piece's
        // partial slot and its statistics, for the combine step.
        const bool partial = sg.slot >= 0;
        const bool empty = !(l_fin > 0.f);
        const float inv = partial ? 1.f : (empty ? 0.f : 1.f / l_fin);
        uint8_t* stage = smem + C::OFF_EPI + quarter * 2 * C::EPI_TILE;
        const uint32_t swz = (lane >> 1) & 3u;
        auto emit = [&](const uint32_t (&w4)[4][4], int x) {  // 64 bytes of this lane's row, at value x
          uint8_t* buf = stage + (epi_n & 1) * C::EPI_TILE;
          if (lane == 0) bulk_wait_read_1();  // the store issued from this tile two tiles ago has read it
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(buf + lane * 64 + ((c ^ swz) << 4)) =
                make_uint4(w4[c][0], w4[c][1], w4[c][2], w4[c][3]);
          fence_async_shared();
          __syncwarp();
          if (lane == 0) {
            if (quarter * 32 < p.Hq) {  // a box wholly past the last head has nothing to write
              if (partial) tma_store_3d(&tmP, buf, x, quarter * 32, sg.slot);
              else tma_store_3d(&tmO, buf, x, quarter * 32, tk);
            }
            bulk_commit();
          }
          ++epi_n;
        };
        auto store_block = [&](int cb, const uint32_t (&r)[32]) {
          uint32_t w4[4][4];
          if (partial) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
              for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int e = 0; e < 4; ++e) w4[c][e] = r[16 * hf + 4 * c + e];
              emit(w4, cb * 32 + 16 * hf);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
              for (int e = 0; e < 4; ++e)
                w4[c][e] = pack_bf16x2(__uint_as_float(r[8 * c + 2 * e]) * inv, __uint_as_float(r[8 * c + 2 * e + 1]) * inv);
            emit(w4, cb * 32);
          }
        };
        // the next block's TMEM load is in flight while a block is stored
        uint32_t ra[32], rb[32];
        tmem_ld32_nowait(tmem + lane_addr, ra);
        tmem_ld_wait_fence(ra);
#pragma unroll 1
        for (int cb = 0; cb < C::DV / 32; cb += 2) {
          tmem_ld32_nowait(tmem + lane_addr + (cb + 1) * 32, rb);
          store_block(cb, ra);
          tmem_ld_wait_fence(rb);
          if (cb + 2 < C::DV / 32) tmem_ld32_nowait(tmem + lane_addr + (cb + 2) * 32, ra);
          store_block(cb + 1, rb);
          if (cb + 2 < C::DV / 32) tmem_ld_wait_fence(ra);
        }
        float* part = partial ? p.part + static_cast<size_t>(sg.slot) * kMlaPartFloats : nullptr;
        if (h < p.Hq) {
          if (partial) {
            part[128 * C::DV + h] = m_fin;
            part[128 * C::DV + 128 + h] = l_fin;
          } else if (p.lse) {
            p.lse[static_cast<size_t>(tk) * p.Hq + h] =
                empty ? -INFINITY : (m_fin + log2f(l_fin)) * 0.69314718055994531f;
          }
        }
        tc_fence_before();
      }
    }
  }

  // the value CTA's output stores have completed before the CTA leaves
  if (rank == 1 && warp >= C::W_SM0 && lane == 0) bulk_wait_all();
  __syncthreads();
  cluster_sync_all();
  if (warp == C::W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Tokens whose chunks were spread over several clusters: exactly those that
// hold a cluster boundary start(g), 0 < g < G, strictly inside them. Returns
// how many there are and, for want >= 0, the want-th of them in *tk.
__host__ __device__ __forceinline__ int mla_split_tokens(int T, int nchunk, int G, int want, int* tk) {
  const long long U = static_cast<long long>(T) * nchunk;
  int n = 0, last = -1;
  for (int g = 1; g < G; ++g) {
    const long long u = mla_unit_start(g, U, G);
    if (u % nchunk == 0) continue;  // a boundary between tokens splits nothing
    const int t = static_cast<int>(u / nchunk);
    if (t == last) continue;        // several boundaries inside one token
    last = t;
    if (n == want) *tk = t;
    ++n;
  }
  return n;
}

// Combine step of the split selections: block (j, y) merges the j-th split
// token (mla_split_tokens) for heads 2y, 2y + 1. Each part i holds numerators
// O_i = sum 2^(z - m_i) v, sums l_i = sum 2^(z - m_i) and its reference
// maximum m_i (z = score * scale * log2 e); with M = max_i m_i,
//     u = sum_i 2^(m_i - M) O_i / sum_i 2^(m_i - M) l_i,
//     lse = (M + log2 sum_i 2^(m_i - M) l_i) * ln 2,
// the softmax over the union of the parts' rows. A token whose parts hold no
// valid row gets u = 0 and lse = -inf, as in the unsplit kernel.
constexpr int kMlaMaxParts = MlaCfg::KMAX / MlaCfg::NK;  // a part holds at least one chunk
constexpr int kCombineHeads = 2;                          // heads per block (128 threads each)
__global__ void __launch_bounds__(256)
    mla_combine_kernel(const float* __restrict__ part, int T, int nchunk, int G, int Hq,
                       __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  __shared__ float wgt[kCombineHeads][kMlaMaxParts];
  __shared__ int slot_s[kMlaMaxParts];
  __shared__ int tk_s, np_s;
  griddep_wait();  // launched as a programmatic dependent of the attention kernel
  const long long U = static_cast<long long>(T) * nchunk;
  if (threadIdx.x < 32) {
    // warp 0 finds the blockIdx.x-th split token: boundary g counts when it
    // lies strictly inside a token that no earlier boundary lies in
    const int lane = static_cast<int>(threadIdx.x);
    int found = -1, seen = 0;
    for (int g0 = 1; g0 < G && found < 0; g0 += 32) {
      const int g = g0 + lane;
      bool first = false;
      int t = 0;
      if (g < G) {
        const long long u = mla_unit_start(g, U, G), up = mla_unit_start(g - 1, U, G);
        t = static_cast<int>(u / nchunk);
        first = (u % nchunk != 0) && (g == 1 || up / nchunk != t || up % nchunk == 0);
      }
      const uint32_t m = __ballot_sync(0xffffffffu, first);
      const int want = static_cast<int>(blockIdx.x) - seen;
      if (want < __popc(m)) {
        // the want-th set bit of m
        uint32_t mm = m;
        for (int k = 0; k < want; ++k) mm &= mm - 1;
        found = __shfl_sync(0xffffffffu, t, __ffs(mm) - 1);
      }
      seen += __popc(m);
    }
    int np = 0;
    if (found >= 0) {
      const long long a = static_cast<long long>(found) * nchunk;  // the token's units [a, a + nchunk)
      const int g_lo = mla_unit_owner(a, U, G), g_hi = mla_unit_owner(a + nchunk - 1, U, G);
      np = g_hi - g_lo + 1;
      if (np > kMlaMaxParts) np = 0;  // cannot happen: every cluster holds at least one unit
      if (lane < np) {
        const int gi = g_lo + lane;
        // the token is the first piece of a cluster that starts inside it,
        // else the last piece of the cluster that started before it
        slot_s[lane] = (mla_unit_start(gi, U, G) >= a) ? 2 * gi : 2 * gi + 1;
      }
    }
    if (lane == 0) {
      tk_s = found;
      np_s = np;
    }
  }
  __syncthreads();
  const int tk = tk_s, np = np_s;
  if (tk < 0 || np < 2) return;  // (cannot happen: the host launches one block per split token)
  const int hl = static_cast<int>(threadIdx.x) >> 7;  // head of this thread within the block
  const int h = blockIdx.y * kCombineHeads + hl;
  const bool active = h < Hq;  // an odd Hq leaves the last block's second head empty
  const int t = static_cast<int>(threadIdx.x) & 127;
  if (active && t < 32) {
    // the head's weights: lane i takes part i
    const float* pi = part + static_cast<size_t>(slot_s[min(t, np - 1)]) * kMlaPartFloats + 128 * 512;
    const float mi = (t < np) ? pi[h] : -INFINITY;
    const float li = (t < np) ? pi[128 + h] : 0.f;
    float M = mi;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float e = (mi == -INFINITY) ? 0.f : exp2f(mi - M);
    float Lsum = e * li;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, off);
    const bool empty = !(Lsum > 0.f);
    if (t < np) wgt[hl][t] = empty ? 0.f : e / Lsum;
    if (t == 0 && lse)
      lse[static_cast<size_t>(tk) * Hq + h] = empty ? -INFINITY : (M + log2f(Lsum)) * 0.69314718055994531f;
  }
  __syncthreads();
  if (!active) return;
  // four values per thread (coalesced reads and writes); every part's load
  // is issued before the sums (NP >= np loads, the ones past np re-read the
  // last part with weight 0)
  const int d = 4 * t;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  auto merge = [&](auto np_c) {
    constexpr int NP = decltype(np_c)::value;
    float4 o[NP];
    // issued back to back (ordered asm), so all NP loads are in flight together
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      const float* src = part + static_cast<size_t>(slot_s[min(i, np - 1)]) * kMlaPartFloats +
                         static_cast<size_t>(h) * 512 + d;
      asm volatile("ld.global.v4.f32 {%0, %1, %2, %3}, [%4];"
                   : "=f"(o[i].x), "=f"(o[i].y), "=f"(o[i].z), "=f"(o[i].w)
                   : "l"(src));
    }
    // no use of a loaded value before the last load is issued
#pragma unroll
    for (int i = 0; i < NP; ++i) asm volatile("" : "+f"(o[i].x), "+f"(o[i].y), "+f"(o[i].z), "+f"(o[i].w));
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      const float wv = (i < np) ? wgt[hl][i] : 0.f;
      acc.x = __fmaf_rn(wv, o[i].x, acc.x);
      acc.y = __fmaf_rn(wv, o[i].y, acc.y);
      acc.z = __fmaf_rn(wv, o[i].z, acc.z);
      acc.w = __fmaf_rn(wv, o[i].w, acc.w);
    }
  };
  if (np <= 2) merge(std::integral_constant<int, 2>{});
  else if (np <= 4) merge(std::integral_constant<int, 4>{});
  else if (np <= 8) merge(std::integral_constant<int, 8>{});
  else merge(std::integral_constant<int, kMlaMaxParts>{});
  __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(out + (static_cast<size_t>(tk) * Hq + h) * 512 + d);
  dst[0] = __floats2bfloat162_rn(acc.x, acc.y);
  dst[1] = __floats2bfloat162_rn(acc.z, acc.w);
}

}  // namespace dsa
