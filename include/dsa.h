/*
 * dsa.h — C ABI of the B200 (sm_100a) DeepSeek Sparse Attention hot path.
 *
 * The method (DeepSeek-V3.2-Exp): a lightning indexer scores every causal
 * (query t, key s) pair with a few FP8 heads, a fine-grained selection keeps
 * the top-k keys per query, and multi-query attention runs over only those
 * entries of the MLA latent cache ("DeepSeek-V3.2-Exp解析", dtcms.com, section
 * 一.1, the three-stage workflow; "Lightning Indexer 的计算过程", adg.csdn.net/
 * 695234..., steps 1-4).
 *
 * Conventions for every call:
 *  - All array arguments are DEVICE pointers (CUDA global memory of the
 *    current device), row-major, owned by the caller. The library never
 *    allocates, frees or keeps them. Arrays must be 16-byte aligned.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream). Calls only
 *    enqueue work; they return before it runs.
 *  - The return value reports argument validation and launch errors; nothing
 *    is enqueued unless it is DSA_OK. A kernel that gives up on an internal
 *    wait (bounded, about a second) records a code that dsa_get_device_error()
 *    reads. Indices outside [0, rows) given to the attention calls are
 *    skipped and reported the same way.
 *  - e4m3 = OCP FP8 E4M3 ("fn": no infinities), one byte per value.
 *    bf16 = bfloat16 bits, two bytes per value.
 *  - Supported shapes: H_I in {8, 64} and d_I in {64, 128} for prefill,
 *    H_I = 64 and d_I in {64, 128} for decode; 1 <= topk <= 2048;
 *    Hq in [1, 128]; the latent row is 576 values (512 + 64 RoPE) and the
 *    value is its first 512. Other shapes return DSA_ERR_UNSUPPORTED.
 */
#ifndef DSA_B200_H
#define DSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = -1, /* null pointer, negative size, misaligned array */
  DSA_ERR_UNSUPPORTED = -2, /* shape outside the supported set */
  DSA_ERR_CUDA = -3,        /* a CUDA call or launch failed (see dsa_last_error) */
  DSA_ERR_TIMEOUT = -4,     /* reported by dsa_get_device_error: a kernel gave up on a wait */
  DSA_ERR_WORKSPACE = -5,   /* workspace null or smaller than the *_workspace_size() result */
  DSA_ERR_BAD_INDEX = -6    /* reported by dsa_get_device_error: an index or page entry outside its cache */
} dsa_status;

/* Latent row geometry of the MLA cache (576 = 512 latent + 64 RoPE values). */
#define DSA_D_QK 576
#define DSA_D_V 512
#define DSA_MAX_TOPK 2048

/* ------------------------------------------------------------------------
 * Prefill indexer + top-k.
 *
 * For one causal sequence of L tokens ("Lightning Indexer 的计算过程" steps 3-4;
 * deepseek.csdn.net section 2.2 细粒度词元选择):
 *   I[t,s] = q_scale[t] * k_scale[s] * sum_j w[t,j] * ReLU(e4m3(q_I[t,j,:]) . e4m3(k_cache[s,:]))
 * for s <= t, and idx[t, 0..topk) = the min(topk, t+1) keys s <= t with the
 * largest I[t,s], ordered by (I descending, s ascending), then -1.
 *
 *   q_I      [L, H_I, d_I] e4m3     indexer queries (post-RoPE, quantised per token)
 *   q_scale  [L] f32 (> 0)          per-token query scale
 *   w        [L, H_I] f32           per-head weights (any sign)
 *   k_cache  [L, d_I] e4m3          indexer keys (one key shared by all heads)
 *   k_scale  [L] f32 (> 0)          per-token key scale
 *   idx      [L, topk] int32        output
 *   workspace, ws_bytes             device scratch of at least
 *                                   dsa_index_topk_workspace_size(L, H_I, d_I, topk)
 *                                   bytes; its contents are not kept between calls.
 * The L x L score matrix is never formed: scores are streamed into per-row
 * candidate lists bounded by the workspace size. Long rows first score a
 * stratified sample of 8 key tiles and start their threshold at a sampled
 * score expected to admit ~2.5 * topk keys; a row that ends with fewer than
 * topk admitted keys is recomputed without the sample within the same call,
 * so the result never depends on the sample.
 * ------------------------------------------------------------------------ */
size_t dsa_index_topk_workspace_size(int L, int H_I, int d_I, int topk);

dsa_status dsa_index_topk(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_cache,
                          const float* k_scale, int L, int H_I, int d_I, int topk, int32_t* idx, void* workspace,
                          size_t ws_bytes, void* stream);

/* Chunked prefill: the same selection for a chunk of Tq new query tokens at
 * positions q0 .. q0+Tq-1 against a key cache of L >= q0 + Tq tokens (the
 * cache already holds the chunk's own keys; query r sees keys s <= q0 + r).
 * Row r of the result equals row q0 + r of dsa_index_topk over the first
 * q0 + Tq tokens.
 *
 *   q_I      [Tq, H_I, d_I] e4m3      q_scale [Tq]   w [Tq, H_I]
 *   k_cache  [L, d_I] e4m3            k_scale [L]
 *   idx      [Tq, topk] int32         output (key positions, -1 padded)
 *   workspace, ws_bytes               at least dsa_index_topk_workspace_size(Tq, H_I, d_I, topk)
 * Errors: DSA_ERR_INVALID_ARG unless q0 >= 0, Tq >= 1 and q0 + Tq <= L;
 * otherwise as dsa_index_topk. A serving step of the method (the pages'
 * prefill and decoding cost figure covers the two extremes, Tq = L and
 * Tq = 1); the selection rule is unchanged. */
dsa_status dsa_index_topk_chunk(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_cache,
                                const float* k_scale, int q0, int Tq, int L, int H_I, int d_I, int topk, int32_t* idx,
                                void* workspace, size_t ws_bytes, void* stream);

/* Chunked prefill over a paged FP8 key cache (one sequence): k_pool
 * [pool_rows, d_I] e4m3 and k_scale_pool [pool_rows] f32 hold pages of
 * page_size rows (a power of two, 16..4096; pool_rows a multiple of it); key
 * s is pool row block_table[s / page_size] * page_size + s % page_size
 * (block_table [max_blocks] int32, device, max_blocks * page_size >= L).
 * Same result as dsa_index_topk_chunk over the gathered contiguous cache, bit
 * for bit; same workspace. A page entry outside [0, pool_rows / page_size)
 * for a key below L gives that page's keys zero codes and zero scale and is
 * reported as DSA_ERR_BAD_INDEX by dsa_get_device_error. H_I = 64 only.
 * Serving layout, no counterpart step in the pages. */
dsa_status dsa_index_topk_chunk_paged(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_pool,
                                      const float* k_scale_pool, const int32_t* block_table, int max_blocks,
                                      int page_size, int pool_rows, int q0, int Tq, int L, int H_I, int d_I, int topk,
                                      int32_t* idx, void* workspace, size_t ws_bytes, void* stream);

/* Packed batch of sequences (cu_seqlens form): sequence b owns query rows
 * [cu_q[b], cu_q[b+1]) of q_I / q_scale / w and keys [cu_k[b], cu_k[b+1]) of
 * k_cache / k_scale; its queries sit at positions q_pos0[b] .. q_pos0[b] +
 * (cu_q[b+1] - cu_q[b]) - 1 of its own cache (q_pos0 NULL: the queries are the
 * last tokens of each cache). Row i of idx [cu_q[nseq], topk] is the selection
 * of query row i, as key positions local to its sequence (0 = the sequence's
 * first key), -1 padded. Each sequence's rows equal what dsa_index_topk_chunk
 * gives for that sequence alone. cu_q, cu_k, q_pos0 are HOST arrays (the
 * call builds a longest-first row-block table from them and copies it into
 * the workspace); everything else is device memory.
 * Errors: DSA_ERR_INVALID_ARG unless cu_q[0] = cu_k[0] = 0, the offsets do
 * not decrease, and every sequence has q_pos0 >= 0 and q_pos0 + queries <=
 * keys; otherwise as dsa_index_topk. Serving layout of the same selection
 * rule; no counterpart step in the pages. */
size_t dsa_index_topk_varlen_workspace_size(int total_q, int nseq, int H_I, int d_I, int topk);
dsa_status dsa_index_topk_varlen(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_cache,
                                 const float* k_scale, const int32_t* cu_q, const int32_t* cu_k,
                                 const int32_t* q_pos0, int nseq, int H_I, int d_I, int topk, int32_t* idx,
                                 void* workspace, size_t ws_bytes, void* stream);

/* Test hook: after dsa_index_topk returned with this workspace (and the same
 * L, H_I, d_I, topk), the number of row blocks of 8 tokens whose sampled
 * starting threshold proved too high and that were therefore recomputed with
 * plain streaming (the result is the same either way). Synchronises `stream`
 * and copies one int to *count. No counterpart in the pages: it only exposes
 * how often this implementation's shortcut had to be undone. */
dsa_status dsa_index_topk_rerun_count(const void* workspace, int L, int H_I, int d_I, int topk, int* count,
                                      void* stream);

/* Test hook: the same kernel's fp32 scores for query rows [row0, row0+nrows),
 * written to scores[nrows, L] (row r is query t = row0 + r; entries s > t are
 * -INFINITY). Bit-identical to the values the selection of dsa_index_topk
 * ranks. Needs no workspace. */
dsa_status dsa_index_scores(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_cache,
                            const float* k_scale, int L, int H_I, int d_I, int row0, int nrows, float* scores,
                            void* stream);

/* ------------------------------------------------------------------------
 * Sparse MQA attention over the MLA latent cache (prefill).
 *
 * For every query token t and head h (deepseek.csdn.net section 2.2; the
 * 576-value latent row of yudonglee.me "DeepSeek-V3.2 explained" section 2.4):
 *   z_s = scale * q[t,h,:] . kv[s,:]          for s in idx[t,:], s >= 0
 *   out[t,h,:] = sum_s softmax(z)_s * kv[s, 0:512]   (bf16 out, fp32 math)
 *   lse[t,h] = log(sum_s exp(z_s))            (natural log; -inf if no entry)
 * All heads share each selected row. Entries < 0 are skipped; an entry >= L
 * is skipped too and reported as DSA_ERR_BAD_INDEX by dsa_get_device_error.
 * T = 0 is a no-op that launches nothing (q, idx, out may then be NULL).
 *
 *   q        [T, Hq, 576] bf16
 *   kv       [L, 576] bf16         latent cache rows
 *   idx      [T, topk] int32       rows of kv (-1 = none)
 *   out      [T, Hq, 512] bf16     output
 *   lse      [T, Hq] f32 or NULL
 *   scale    softmax scale, finite and > 0 (1/sqrt(576) for the latent row)
 * No workspace.
 * ------------------------------------------------------------------------ */
dsa_status dsa_sparse_mla_attn(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int T, int L, int Hq,
                               int topk, float scale, uint16_t* out, float* lse, void* stream);

/* Sparse MQA attention over a packed batch of sequences (cu_seqlens form),
 * the attention that follows dsa_index_topk_varlen: sequence b owns query
 * tokens cu_q[b] .. cu_q[b+1]-1 of q / idx / out / lse and latent rows
 * cu_k[b] .. cu_k[b+1]-1 of kv [total_k, 576]; idx holds row numbers local to
 * the token's sequence (as dsa_index_topk_varlen returns them). cu_q and cu_k
 * [nseq+1] int32 are DEVICE arrays (the indexer's varlen call takes host
 * arrays), non-decreasing, cu_q[0] = cu_k[0] = 0, cu_q[nseq] = T, cu_k[nseq]
 * <= total_k; each token finds its sequence on the device. A local index at
 * or past its sequence's row count is skipped and reported as
 * DSA_ERR_BAD_INDEX; offsets outside [0, total_k] are clamped into it, so no
 * read leaves kv. Per token the result equals dsa_sparse_mla_attn over that
 * sequence's rows. Serving layout (continuous batching), no counterpart step
 * in the pages. */
dsa_status dsa_sparse_mla_attn_varlen(const uint16_t* q, const uint16_t* kv, const int32_t* idx, const int32_t* cu_q,
                                      const int32_t* cu_k, int nseq, int T, int total_k, int Hq, int topk, float scale,
                                      uint16_t* out, float* lse, void* stream);

/* Sparse MQA attention over a paged latent cache: kv_pool [pool_rows, 576]
 * holds pages of page_size rows (a power of two, 16..4096); logical row r of
 * token t is physical row block_table[t * bt_stride + r / page_size] *
 * page_size + r % page_size (bt_stride 0: every token uses the first table
 * row, as the tokens of one prefill do; bt_stride = max_blocks: one table row
 * per token, as in decode). idx [T, topk] holds logical rows < rows, with
 * rows <= max_blocks * page_size. Same results as dsa_sparse_mla_attn over
 * the contiguous cache; a page entry outside the pool skips its rows and is
 * reported as DSA_ERR_BAD_INDEX by dsa_get_device_error. workspace /
 * ws_bytes as for dsa_sparse_mla_attn_decode (NULL: whole tokens per
 * cluster, the better choice for long prefills). Serving layout, no
 * counterpart step in the pages. */
dsa_status dsa_sparse_mla_attn_paged(const uint16_t* q, const uint16_t* kv_pool, const int32_t* block_table,
                                     const int32_t* idx, int T, int rows, int pool_rows, int bt_stride,
                                     int max_blocks, int page_size, int Hq, int topk, float scale, uint16_t* out,
                                     float* lse, void* workspace, size_t ws_bytes, void* stream);

/* FP8 quantiser for newly appended tokens (indexer keys or queries): for each
 * of n rows of d fp32 values, scale[r] = absmax/448 (1 for an all-zero row)
 * and codes[r, i] = E4M3(x[r, i] / scale[r]), nearest with ties to even,
 * saturating to +-448 ("Lightning Indexer 的计算过程", step 2 <2>, FP8 量化).
 * Bit-identical to that definition evaluated in fp32. x [n, d] f32, codes
 * [n, d] e4m3 bytes, scale [n] f32, all device memory; codes and scale must
 * not overlap x (DSA_ERR_INVALID_ARG). n = 0 is a no-op. */
dsa_status dsa_quantize_e4m3_rows(const float* x, int n, int d, uint8_t* codes, float* scale, void* stream);

/* RoPE + FP8 quantiser for newly appended indexer queries or keys
 * ("Lightning Indexer 的计算过程", step 2 <1> then <2>). Row r of x [n, heads,
 * d] f32 (device) has the first rope_dim dimensions of every head rotated by
 * position pos[r] (pos [n] int32, device): pair i < rope_dim/2 turns by
 * pos[r] * base^(-2i / rope_dim) radians, (a, b) -> (a cos - b sin, a sin +
 * b cos), the pairs being dimensions (2i, 2i+1) when interleaved != 0, else
 * (i, i + rope_dim/2); the other dimensions pass through. The rotation is
 * evaluated in float64 and rounded once to fp32; the fp32 row is then
 * quantised exactly as by dsa_quantize_e4m3_rows with one scale over its
 * heads * d values. codes [n, heads * d] e4m3, scale [n] f32, rotated
 * [n, heads * d] f32 or NULL (receives the fp32 rotated rows). rope_dim even,
 * 2 <= rope_dim <= min(d, 128); base finite and > 0. Each row is read twice
 * and a thread reads values other threads rotate, so rotated, codes and
 * scale must not overlap x: an in-place call returns DSA_ERR_INVALID_ARG.
 * n = 0 is a no-op. */
dsa_status dsa_rope_quantize_e4m3_rows(const float* x, const int32_t* pos, int n, int heads, int d, int rope_dim,
                                       double base, int interleaved, uint8_t* codes, float* scale, float* rotated,
                                       void* stream);

/* Short-sequence dense fallback: when a sequence has at most DSA_MAX_TOPK
 * tokens every causal key is selected anyway, so the indexer can be skipped
 * and token t (position q0 + t) attends to kv rows 0..q0+t directly, with the
 * same arithmetic as dsa_sparse_mla_attn over the selection {0..q0+t}
 * (causal MQA over the latent rows: the short-input mode of
 * "DeepSeek-V3.2-Exp解析" section 一.1, where the selection covers
 * everything). q [T, Hq, 576], kv [L, 576] (L <= DSA_MAX_TOPK, q0 + T <= L),
 * out [T, Hq, 512], lse [T, Hq] or NULL. Errors: DSA_ERR_UNSUPPORTED for
 * L > DSA_MAX_TOPK, otherwise as dsa_sparse_mla_attn. */
dsa_status dsa_dense_mla_attn_causal(const uint16_t* q, const uint16_t* kv, int T, int L, int q0, int Hq, float scale,
                                     uint16_t* out, float* lse, void* stream);

/* ------------------------------------------------------------------------
 * Decode: B sequences, one new query each, at position t = lens[b]-1 of its
 * own cache (the new token's key and latent row are already cached). Caches
 * are strided by L_max tokens per sequence. Same definitions as prefill with
 * t = lens[b]-1 (the decode curve of adg.csdn.net/695234..., figure (b)).
 *
 *   q_I      [B, H_I, d_I] e4m3     q_scale [B] f32     w [B, H_I] f32
 *   k_cache  [B, L_max, d_I] e4m3   k_scale [B, L_max] f32
 *   lens     [B] int32 (device), 1 <= lens[b] <= L_max
 *   idx      [B, topk] int32 out    (rows of sequence b's own cache)
 *   workspace                       >= dsa_index_topk_decode_workspace_size(B, L_max, topk)
 *                                   bytes: the per-key scores and the selection.
 * ------------------------------------------------------------------------ */
size_t dsa_index_topk_decode_workspace_size(int B, int L_max, int topk);

dsa_status dsa_index_topk_decode(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_cache,
                                 const float* k_scale, const int32_t* lens, int B, int L_max, int H_I, int d_I,
                                 int topk, int32_t* idx, void* workspace, size_t ws_bytes, void* stream);

/* Decode indexer + top-k over a paged FP8 key cache. k_pool [pool_rows, d_I]
 * e4m3 and k_scale_pool [pool_rows] f32 hold pages of page_size rows (a power
 * of two, 16..4096; pool_rows a multiple of it); key s of sequence b is pool
 * row block_table[b * max_blocks + s / page_size] * page_size + s % page_size
 * (block_table [B, max_blocks] int32, device). Entries for pages at or past
 * lens[b] are never read. Equivalent to dsa_index_topk_decode with L_max =
 * max_blocks * page_size over the gathered contiguous cache: same scores bit
 * for bit, same idx. Workspace: dsa_index_topk_decode_workspace_size(B,
 * max_blocks * page_size, topk). A page entry outside [0, pool_rows /
 * page_size) for a key below lens[b] gives that page's keys zero codes and
 * zero scale (score 0) and is reported as DSA_ERR_BAD_INDEX by
 * dsa_get_device_error. Serving layout, no counterpart step in the pages. */
dsa_status dsa_index_topk_decode_paged(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_pool,
                                       const float* k_scale_pool, const int32_t* block_table, const int32_t* lens,
                                       int B, int max_blocks, int page_size, int pool_rows, int H_I, int d_I, int topk,
                                       int32_t* idx, void* workspace, size_t ws_bytes, void* stream);

/* Test hook: decode scores[B, L_max] f32 (entries s >= lens[b] untouched). */
dsa_status dsa_index_scores_decode(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_cache,
                                   const float* k_scale, const int32_t* lens, int B, int L_max, int H_I, int d_I,
                                   float* scores, void* stream);

/*   q [B, Hq, 576] bf16, kv [B, L_max, 576] bf16, idx [B, topk] int32 (rows of
 *   sequence b's cache, -1 = none), out [B, Hq, 512] bf16, lse [B, Hq] f32 or NULL.
 *
 * Split selections (flash-decoding): with a workspace of at least
 * dsa_sparse_mla_attn_split_workspace_size(B, topk) bytes (device, 16-byte
 * aligned), a batch small enough to leave at least half of the GPU's 2-SM
 * clusters idle (2 * B <= clusters; 74 clusters on a 148-SM B200) has its
 * B x ceil(topk/128) (sequence, 128-entry chunk) units cut into one
 * contiguous range per cluster, so it still uses every SM; a sequence whose
 * chunks fall to several clusters gets, from each, its unnormalised output
 * and softmax statistics in the workspace, and a combine step merges them
 * (the softmax over the union of the rows). The result equals the unsplit
 * one up to fp32 rounding order. Larger batches, and workspace NULL, run one
 * cluster per sequence with no combine step. A workspace given but too small
 * returns DSA_ERR_WORKSPACE. No counterpart step in the pages (the decode
 * regime of the cost figure (b) is what it serves). */
size_t dsa_sparse_mla_attn_split_workspace_size(int T, int topk);

dsa_status dsa_sparse_mla_attn_decode(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int B, int L_max,
                                      int Hq, int topk, float scale, uint16_t* out, float* lse, void* workspace,
                                      size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Decode indexer + top-k with no caller workspace and no allocation.
 *
 * The pages describe nothing like this call; it exists for callers that
 * cannot allocate device memory: plugins inside a host framework that owns
 * every device allocation and gives its extensions no allocator, and
 * latency-bound serving loops where a cudaMalloc (which may synchronise the
 * whole device) is not acceptable. It computes exactly what
 * dsa_index_topk_decode computes (same kernels, same results), but its
 * scratch (the per-key scores and the selected keys) is a fixed array inside
 * this library, in the device memory of every GPU that loads the library,
 * held until the process exits.
 *
 * Limits: B * L_max <= DSA_NOALLOC_MAX_SCORES and B * topk <=
 * DSA_NOALLOC_MAX_KEYS; larger calls return DSA_ERR_UNSUPPORTED (nothing is
 * enqueued) with the limit in dsa_last_error().
 * The first call on each device looks up the array's device address (a
 * runtime query, no allocation); make that first call before any stream
 * capture. The address is kept for the life of the process, so after a
 * cudaDeviceReset (or anything else that re-creates a device's primary
 * context) this entry point must not be called on that device again. Every
 * call shares the one array: calls whose work overlaps on the
 * GPU (different streams, or several host threads) race and must be ordered
 * by the caller. Nothing in the array needs to start at zero: each call
 * writes every element it later reads. No cudaMalloc, cudaFree or
 * allocating library routine is called.
 * Arguments as for dsa_index_topk_decode, without workspace / ws_bytes.
 * ------------------------------------------------------------------------ */
#define DSA_NOALLOC_MAX_SCORES (1u << 20) /* 4 MiB of fp32 scores */
#define DSA_NOALLOC_MAX_KEYS (1u << 16)   /* 512 KiB of selected keys */

dsa_status dsa_index_topk_decode_noalloc(const uint8_t* q_I, const float* q_scale, const float* w,
                                         const uint8_t* k_cache, const float* k_scale, const int32_t* lens, int B,
                                         int L_max, int H_I, int d_I, int topk, int32_t* idx, void* stream);

/* ------------------------------------------------------------------------
 * Errors.
 * ------------------------------------------------------------------------ */
/* Failure-path self-test: enqueues on `stream` one small kernel that waits,
 * with the same bounded wait every kernel here uses, on a barrier nothing
 * completes. After wait_cycles SM cycles (0: the library's own bound of 2^31
 * cycles, about a second; at most 2^31) the wait gives up, records
 * DSA_ERR_TIMEOUT with site 99 and the kernel exits; the next
 * dsa_get_device_error reports it and the context stays usable. Returns the
 * launch status, or DSA_ERR_INVALID_ARG for wait_cycles outside [0, 2^31].
 * No counterpart in the pages. */
dsa_status dsa_selftest_wait_timeout(long long wait_cycles, void* stream);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device: DSA_OK, DSA_ERR_TIMEOUT or DSA_ERR_BAD_INDEX (*detail gets
 * the raw word, may be NULL); DSA_ERR_CUDA if the synchronisation fails. */
dsa_status dsa_get_device_error(void* stream, unsigned int* detail);

/* Static, NUL-terminated name of a status code ("unknown status" for any
 * other value); never NULL, never to be freed. */
const char* dsa_status_string(dsa_status s);
/* Message of the last failing call on this host thread ("" if none); the
 * buffer belongs to the library and is overwritten by the thread's next
 * failing call. */
const char* dsa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_B200_H */
