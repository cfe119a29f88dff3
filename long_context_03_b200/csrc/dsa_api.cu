// C ABI of the DSA hot path (see include/dsa.h): argument checks, workspace
// carving, TMA descriptors and kernel launches. One translation unit holds
// every kernel so the device error word is a single symbol.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <algorithm>
#include <atomic>
#include <vector>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/dsa.h"
#include "dsa_common.cuh"
#include "indexer_decode.cuh"
#include "indexer_prefill.cuh"
#include "sparse_mla.cuh"
#include "quantize.cuh"
#include "topk_select.cuh"

using namespace dsa;

namespace {

thread_local char g_last_error[512] = "";

dsa_status fail(dsa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

dsa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(DSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Whether the byte ranges [a, a + na) and [b, b + nb) share a byte.
bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

int num_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  int n = 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 1;
}

// ---- TMA descriptor encoding through the driver entry point ----
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D byte tensor [outer, inner] (row-major, rows of `inner` bytes), box
// [box_outer, box_inner], swizzled to match the tensor-core layouts.
dsa_status make_map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                       uint32_t box_outer) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = (inner == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return DSA_OK;
}

// Queries [T, Hq, 576] bf16 as a 3-D map {576, Hq, T}; boxes of 64 values x
// 128 heads x 1 token, 128-byte swizzled (heads >= Hq lie outside the map and
// load as zeros).
dsa_status make_map_q_bf16(CUtensorMap* m, const void* base, int T, int Hq) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[3] = {576, static_cast<cuuint64_t>(Hq), static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[2] = {576 * 2, static_cast<cuuint64_t>(Hq) * 576 * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled(q) failed (%d)", static_cast<int>(r));
  return DSA_OK;
}

// Output [T, Hq, 512] bf16 as a 3-D map {512, Hq, T} for bulk tensor
// stores: boxes of 32 values x 32 heads x 1 token, 64-byte swizzled (heads
// >= Hq lie outside the map and are not written).
dsa_status make_map_out_bf16(CUtensorMap* m, const void* base, int T, int Hq) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[3] = {512, static_cast<cuuint64_t>(Hq), static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[2] = {512 * 2, static_cast<cuuint64_t>(Hq) * 512 * 2};
  const cuuint32_t box[3] = {32, 32, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled(out) failed (%d)", static_cast<int>(r));
  return DSA_OK;
}

// The partial slots' numerators [slots][Hq rows of 512] f32 (slot stride
// kMlaPartFloats) as a 3-D map {512, Hq, slots}: boxes of 16 values x 32
// heads x 1 slot, 64-byte swizzled.
dsa_status make_map_part_f32(CUtensorMap* m, const float* base, int slots, int Hq) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[3] = {512, static_cast<cuuint64_t>(Hq), static_cast<cuuint64_t>(slots)};
  const cuuint64_t strides[2] = {512 * 4, static_cast<cuuint64_t>(kMlaPartFloats) * 4};
  const cuuint32_t box[3] = {16, 32, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled(part) failed (%d)", static_cast<int>(r));
  return DSA_OK;
}

template <typename K>
dsa_status set_smem(K kernel, int bytes) {
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  return DSA_OK;
}

dsa_status check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  return DSA_OK;
}

// Launch as a programmatic dependent of the previous kernel in the stream
// (programmatic stream serialization): the kernel may be scheduled while
// that kernel finishes and waits for it (griddep_wait) before touching
// global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ---- prefill indexer ----
constexpr int kNetPrefill = 16 * 32;  // epilogue threads of the prefill indexer

// keys per thread per quarter sub-list in a list cut; list capacity = 4 * MQ * 256
int select_mq(int topk) { return (topk <= 128) ? 1 : 4; }
int select_cap(int topk) { return 4 * select_mq(topk) * kNetPrefill; }

int rows_per_block(int H_I) { return 2 * (256 / H_I); }

bool prefill_shape_ok(int H_I, int d_I) { return (H_I == 8 || H_I == 64) && (d_I == 64 || d_I == 128); }

// Workspace of the prefill selection: the persistent CTAs' candidate lists,
// then the re-run list.
struct WsPrefill {
  uint64_t* cand;
  int* redo;  // [0]: count, [4 ..]: row blocks to re-run
  size_t bytes;
};

WsPrefill prefill_ws_layout(void* base, int L, int H_I, int topk, int grid) {
  WsPrefill w;
  const int nrb = (L + rows_per_block(H_I) - 1) / rows_per_block(H_I);
  const size_t cand_bytes = static_cast<size_t>(grid) * rows_per_block(H_I) * select_cap(topk) * 8;
  const size_t redo_bytes = (static_cast<size_t>(nrb) + 4) * 4;
  w.cand = reinterpret_cast<uint64_t*>(base);
  w.redo = reinterpret_cast<int*>(reinterpret_cast<char*>(base) + cand_bytes);
  w.bytes = cand_bytes + redo_bytes;
  return w;
}

// Rows at least this long start from a sampled threshold (twice the list
// capacity: shorter rows rarely cut their lists anyway).
int spec_min_row(int topk) { return 2 * select_cap(topk) > 4096 ? 2 * select_cap(topk) : 4096; }

template <int HI, int DI, bool kSelect, int MQ, bool kPaged = false>
dsa_status launch_prefill(const uint8_t* q_I, const uint8_t* k_cache, const IdxPrefillParams& p, int grid,
                          cudaStream_t st) {
  using C = IdxPrefillCfg<HI, DI>;
  CUtensorMap tmQ, tmK;
  dsa_status s = make_map_u8(&tmQ, q_I, DI, static_cast<uint64_t>(p.Tq) * HI, DI, C::QBOX);
  if (s != DSA_OK) return s;
  if (kPaged) {
    // the pool's rows, one page (at most one key tile) per box
    const int page = 1 << p.page_shift;
    s = make_map_u8(&tmK, k_cache, DI, static_cast<uint64_t>(p.pool_pages) * page, DI,
                    static_cast<uint32_t>(page < C::BM ? page : C::BM));
  } else {
    s = make_map_u8(&tmK, k_cache, DI, static_cast<uint64_t>(p.L), DI, C::BM);
  }
  if (s != DSA_OK) return s;
  auto kern = indexer_prefill_kernel<HI, DI, kSelect, MQ, kPaged>;
  s = set_smem(kern, C::SMEM_BYTES);
  if (s != DSA_OK) return s;
  kern<<<grid, C::NTHREADS, C::SMEM_BYTES, st>>>(tmQ, tmK, p);
  return check_launch("indexer_prefill_kernel");
}

template <bool kSelect, int MQ>
dsa_status dispatch_prefill(int H_I, int d_I, const uint8_t* q_I, const uint8_t* k_cache, const IdxPrefillParams& p,
                            int grid, cudaStream_t st) {
  if constexpr (kSelect) {
    if (p.block_table) {  // paged key cache: the H_I = 64 shapes
      if (H_I == 64 && d_I == 128) return launch_prefill<64, 128, true, MQ, true>(q_I, k_cache, p, grid, st);
      if (H_I == 64 && d_I == 64) return launch_prefill<64, 64, true, MQ, true>(q_I, k_cache, p, grid, st);
      return fail(DSA_ERR_UNSUPPORTED, "paged keys: H_I=%d d_I=%d not supported", H_I, d_I);
    }
  }
  if (H_I == 64 && d_I == 128) return launch_prefill<64, 128, kSelect, MQ>(q_I, k_cache, p, grid, st);
  if (H_I == 64 && d_I == 64) return launch_prefill<64, 64, kSelect, MQ>(q_I, k_cache, p, grid, st);
  if (H_I == 8 && d_I == 128) return launch_prefill<8, 128, kSelect, MQ>(q_I, k_cache, p, grid, st);
  if (H_I == 8 && d_I == 64) return launch_prefill<8, 64, kSelect, MQ>(q_I, k_cache, p, grid, st);
  return fail(DSA_ERR_UNSUPPORTED, "H_I=%d d_I=%d not supported", H_I, d_I);
}

__global__ void fill_f32_kernel(float* p, size_t n, float v) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    p[i] = v;
}

// ---- failure-path self-test ----
// One CTA waits, with the library's bounded wait, on an mbarrier that no
// thread arrives on: the wait gives up after `bound` cycles, records a timeout
// with site kSelftestSite in the device error word and the kernel returns,
// leaving the context usable.
constexpr unsigned int kSelftestSite = 99;
__global__ void selftest_wait_timeout_kernel(long long bound) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const AbortFlag ab{&abort_flag};
  if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, ab, kSelftestSite, bound);
  __syncthreads();
}

// ---- decode ----

template <int HI, int DI>
dsa_status launch_decode_scores(const uint8_t* q_I, const uint8_t* k_cache, int B, const IdxDecodeParams& p,
                                cudaStream_t st) {
  using C = IdxDecodeCfg<HI, DI>;
  const bool paged = p.block_table != nullptr;
  CUtensorMap tmQ, tmK;
  dsa_status s = make_map_u8(&tmQ, q_I, DI, static_cast<uint64_t>(B) * HI, DI, HI);
  if (s != DSA_OK) return s;
  if (paged) {
    // the pool's rows, loaded one page (at most one tile) per box
    const int page = 1 << p.page_shift;
    s = make_map_u8(&tmK, k_cache, DI, static_cast<uint64_t>(p.pool_pages) * page, DI,
                    static_cast<uint32_t>(page < C::BM ? page : C::BM));
  } else {
    s = make_map_u8(&tmK, k_cache, DI, static_cast<uint64_t>(B) * p.L_max, DI, C::BM);
  }
  if (s != DSA_OK) return s;
  auto kern = paged ? indexer_decode_kernel<HI, DI, true> : indexer_decode_kernel<HI, DI, false>;
  s = set_smem(kern, C::SMEM_BYTES);
  if (s != DSA_OK) return s;
  const int items = ((p.L_max + C::CHUNK - 1) / C::CHUNK) * B;
  const int slots = 2 * num_sms();  // two persistent CTAs per SM (shared memory)
  kern<<<items < slots ? items : slots, C::NTHREADS, C::SMEM_BYTES, st>>>(tmQ, tmK, p);
  return check_launch("indexer_decode_kernel");
}

struct KeyPaging {
  const int32_t* block_table = nullptr;
  int bt_stride = 0, page_shift = 0, pool_pages = 0;
};

dsa_status decode_scores(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_cache,
                         const float* k_scale, const int32_t* lens, int B, int L_max, int H_I, int d_I, float* scores,
                         uint32_t* hist, cudaStream_t st, KeyPaging pg = KeyPaging()) {
  IdxDecodeParams p;
  p.block_table = pg.block_table;
  p.bt_stride = pg.bt_stride;
  p.page_shift = pg.page_shift;
  p.pool_pages = pg.pool_pages;
  p.hist = hist;
  p.q_scale = q_scale;
  p.w = w;
  p.k_scale = k_scale;
  p.lens = lens;
  p.L_max = L_max;
  p.B = B;
  p.scores = scores;
  if (H_I == 64 && d_I == 128) return launch_decode_scores<64, 128>(q_I, k_cache, B, p, st);
  if (H_I == 64 && d_I == 64) return launch_decode_scores<64, 64>(q_I, k_cache, B, p, st);
  return fail(DSA_ERR_UNSUPPORTED, "decode: H_I=%d d_I=%d not supported", H_I, d_I);
}

// Selection and ranking of every sequence's top-k: one CTA per sequence
// selects, then sorts its keys in shared memory and writes idx.
dsa_status launch_decode_select(const float* scores, const int32_t* lens, int L_max, int topk, const uint32_t* hist,
                                uint64_t* sel, int32_t* idx, int B, cudaStream_t st) {
  const int smem = kDecodeSelBinCap * 8 + (2048 + select_scratch_ints(kDecodeSelThreads)) * 4;
  dsa_status s = set_smem(decode_select_kernel, smem);
  if (s != DSA_OK) return s;
  if (hist) {
    // two CTAs per sequence (a cluster) split the pass over the scores
    s = set_smem(decode_select_pair_kernel, smem);
    if (s != DSA_OK) return s;
    const cudaError_t e = launch_dependent(decode_select_pair_kernel, dim3(2 * B), dim3(kDecodeSelThreads), smem, st,
                                           scores, lens, L_max, topk, hist, sel, idx);
    if (e != cudaSuccess) return cuda_fail(e, "decode_select_pair_kernel launch");
    return check_launch("decode_select_pair_kernel");
  }
  const cudaError_t e = launch_dependent(decode_select_kernel, dim3(B), dim3(kDecodeSelThreads), smem, st, scores,
                                         lens, L_max, topk, hist, sel, idx);
  if (e != cudaSuccess) return cuda_fail(e, "decode_select_kernel launch");
  return check_launch("decode_select_kernel");
}

dsa_status check_decode_args(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_cache,
                             const float* k_scale, const int32_t* lens, int B, int L_max, int H_I, int d_I) {
  if (!q_I || !q_scale || !w || !k_cache || !k_scale || !lens) return fail(DSA_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || L_max <= 0) return fail(DSA_ERR_INVALID_ARG, "B=%d L_max=%d", B, L_max);
  if (!aligned16(q_I) || !aligned16(k_cache)) return fail(DSA_ERR_INVALID_ARG, "q_I / k_cache not 16-byte aligned");
  if (!(H_I == 64 && (d_I == 64 || d_I == 128)))
    return fail(DSA_ERR_UNSUPPORTED, "decode: H_I=%d d_I=%d not supported", H_I, d_I);
  if (static_cast<long long>(B) * L_max >= (1ll << 31)) return fail(DSA_ERR_UNSUPPORTED, "B*L_max too large");
  return DSA_OK;
}

// ---- attention ----
struct MlaPaging {
  const int32_t* block_table = nullptr;
  int bt_stride = 0, page_shift = 0, pool_rows = 0;
};
struct MlaPacked {  // packed batch: device cu_seqlens of the queries and of the cache rows
  const int32_t* cu_q = nullptr;
  const int32_t* cu_k = nullptr;
  int nseq = 0;
};
// Co-resident 2-CTA clusters of the attention kernel, looked up once (the
// same for both instances: same resources); concurrent first calls compute
// the same value.
int mla_max_clusters() {
  static std::atomic<int> cache{0};
  int n = cache.load(std::memory_order_relaxed);
  if (n == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 512, 1, 1);
    cfg.blockDim = dim3(MlaCfg::NTHREADS, 1, 1);
    cfg.dynamicSmemBytes = MlaCfg::SMEM_BYTES;
    if (set_smem(sparse_mla_kernel<false>, MlaCfg::SMEM_BYTES) != DSA_OK ||
        cudaOccupancyMaxActiveClusters(&n, sparse_mla_kernel<false>, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = num_sms() / 2;
    }
    if (n > num_sms() / 2) n = num_sms() / 2;
    if (n < 1) n = 1;
    cache.store(n, std::memory_order_relaxed);
  }
  return n;
}

// Partial slots of a split attention call over T tokens: two per cluster.
size_t mla_split_bytes(int T, int topk) {
  const long long units = static_cast<long long>(T) * ((topk + MlaCfg::NK - 1) / MlaCfg::NK);
  const long long gmax = num_sms() / 2 > 1 ? num_sms() / 2 : 1;
  const long long g = units < gmax ? units : gmax;
  return static_cast<size_t>(2 * g) * kMlaPartFloats * 4;
}

// part != null: split the selections over all clusters (flash-decoding) with
// partial slots in `part` (mla_split_bytes), then the combine step.
dsa_status launch_mla(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int T, int rows, long long kv_stride,
                      int Hq, int topk, float scale, uint16_t* out, float* lse, cudaStream_t st, int causal_q0 = 0,
                      MlaPaging pg = MlaPaging(), MlaPacked pk = MlaPacked(), float* part = nullptr) {
  MlaParams p = {};
  p.q = reinterpret_cast<const __nv_bfloat16*>(q);
  p.kv = reinterpret_cast<const __nv_bfloat16*>(kv);
  p.idx = idx;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.kv_token_stride = kv_stride;
  p.rows = rows;
  p.T = T;
  p.Hq = Hq;
  p.K = topk;
  p.causal_q0 = causal_q0;
  p.block_table = pg.block_table;
  p.bt_stride = pg.bt_stride;
  p.page_shift = pg.page_shift;
  p.pool_rows = pg.pool_rows;
  p.seq_cu_q = pk.cu_q;
  p.seq_cu_k = pk.cu_k;
  p.nseq = pk.nseq;
  p.scale_log2 = scale * 1.4426950408889634f;
  CUtensorMap tmQ, tmO, tmP;
  dsa_status s = make_map_q_bf16(&tmQ, q, T, Hq);
  if (s != DSA_OK) return s;
  s = make_map_out_bf16(&tmO, out, T, Hq);
  if (s != DSA_OK) return s;
  std::memset(&tmP, 0, sizeof(tmP));  // used only by split calls
  auto kern = pg.block_table ? sparse_mla_kernel<true> : sparse_mla_kernel<false>;
  s = set_smem(kern, MlaCfg::SMEM_BYTES);
  if (s != DSA_OK) return s;
  const int max_clusters = mla_max_clusters();
  const int nchunk = (topk + MlaCfg::NK - 1) / MlaCfg::NK;
  const long long units = static_cast<long long>(T) * nchunk;
  // Split only batches that leave at least half of the clusters idle: with
  // more tokens the whole-token schedule already fills the GPU and a split
  // would only add partial writes and the combine step.
  if (2 * T > max_clusters) part = nullptr;
  p.part = part;
  const int nclusters = part ? static_cast<int>(units < max_clusters ? units : max_clusters)
                             : (T < max_clusters ? T : max_clusters);
  if (part) {
    s = make_map_part_f32(&tmP, part, 2 * nclusters, Hq);
    if (s != DSA_OK) return s;
  }
  const cudaError_t e = launch_dependent(kern, dim3(2 * nclusters), dim3(MlaCfg::NTHREADS), MlaCfg::SMEM_BYTES, st,
                                         tmQ, tmO, tmP, p);
  if (e != cudaSuccess) return cuda_fail(e, "sparse_mla_kernel launch");
  s = check_launch("sparse_mla_kernel");
  if (s != DSA_OK || !part) return s;
  const int nsplit = mla_split_tokens(T, nchunk, nclusters, -1, nullptr);
  if (nsplit == 0) return DSA_OK;  // every token was held whole by one cluster
  const dim3 cgrid(nsplit, (Hq + kCombineHeads - 1) / kCombineHeads);
  const cudaError_t e2 = launch_dependent(mla_combine_kernel, cgrid, dim3(256), 0, st, part, T, nchunk, nclusters,
                                          Hq, p.out, lse);
  if (e2 != cudaSuccess) return cuda_fail(e2, "mla_combine_kernel launch");
  return check_launch("mla_combine_kernel");
}

// Optional workspace of a split attention call: NULL (unsplit) or at least
// mla_split_bytes(T, topk) bytes, 16-byte aligned.
dsa_status check_split_workspace(void* workspace, size_t ws_bytes, int T, int topk, float** part) {
  *part = nullptr;
  if (!workspace) return DSA_OK;
  if (static_cast<long long>(T) * ((topk + MlaCfg::NK - 1) / MlaCfg::NK) >= (1ll << 31))
    return fail(DSA_ERR_UNSUPPORTED, "T=%d too large for a split call", T);
  const size_t need = mla_split_bytes(T, topk);
  if (ws_bytes < need) return fail(DSA_ERR_WORKSPACE, "workspace %zu bytes, need %zu", ws_bytes, need);
  if (!aligned16(workspace)) return fail(DSA_ERR_INVALID_ARG, "workspace not 16-byte aligned");
  *part = static_cast<float*>(workspace);
  return DSA_OK;
}

dsa_status check_mla_args(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int T, int L, int Hq, int topk,
                          float scale, const uint16_t* out) {
  if (T < 0 || L <= 0) return fail(DSA_ERR_INVALID_ARG, "T=%d L=%d", T, L);
  if (!kv || (T > 0 && (!q || !idx || !out))) return fail(DSA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(kv) || !aligned16(out) || !aligned16(idx))
    return fail(DSA_ERR_INVALID_ARG, "q / kv / idx / out not 16-byte aligned");
  if (Hq < 1 || Hq > 128) return fail(DSA_ERR_UNSUPPORTED, "Hq=%d not in [1, 128]", Hq);
  if (topk < 1 || topk > DSA_MAX_TOPK) return fail(DSA_ERR_UNSUPPORTED, "topk=%d not in [1, %d]", topk, DSA_MAX_TOPK);
  if (!std::isfinite(scale) || !(scale > 0.f)) return fail(DSA_ERR_INVALID_ARG, "scale must be finite and > 0");
  return DSA_OK;
}

}  // namespace

extern "C" {

size_t dsa_index_topk_workspace_size(int L, int H_I, int d_I, int topk) {
  if (L <= 0 || topk <= 0 || !prefill_shape_ok(H_I, d_I)) return 0;
  const int nrb = (L + rows_per_block(H_I) - 1) / rows_per_block(H_I);
  const int grid = nrb < num_sms() ? nrb : num_sms();
  return prefill_ws_layout(nullptr, L, H_I, topk, grid).bytes;
}

// Queries r = 0..Tq-1 at positions q0 + r against keys 0..L-1 (q0 + Tq <= L).
struct PrefillKeyPaging {
  const int32_t* block_table = nullptr;
  int page_shift = 0, pool_pages = 0;
};

static dsa_status index_topk_impl(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_cache,
                           const float* k_scale, int q0, int Tq, int L, int H_I, int d_I, int topk, int32_t* idx,
                           void* workspace, size_t ws_bytes, cudaStream_t st,
                           PrefillKeyPaging pg = PrefillKeyPaging()) {
  if (!q_I || !q_scale || !w || !k_cache || !k_scale || !idx) return fail(DSA_ERR_INVALID_ARG, "null pointer");
  if (L <= 0 || Tq <= 0 || q0 < 0 || static_cast<long long>(q0) + Tq > L)
    return fail(DSA_ERR_INVALID_ARG, "q0=%d Tq=%d L=%d (need q0 >= 0, Tq >= 1, q0 + Tq <= L)", q0, Tq, L);
  if (!prefill_shape_ok(H_I, d_I)) return fail(DSA_ERR_UNSUPPORTED, "H_I=%d d_I=%d not supported", H_I, d_I);
  if (topk < 1 || topk > DSA_MAX_TOPK) return fail(DSA_ERR_UNSUPPORTED, "topk=%d not in [1, %d]", topk, DSA_MAX_TOPK);
  if (static_cast<long long>(Tq) * H_I >= (1ll << 31)) return fail(DSA_ERR_UNSUPPORTED, "Tq*H_I too large");
  if (!aligned16(q_I) || !aligned16(k_cache)) return fail(DSA_ERR_INVALID_ARG, "q_I / k_cache not 16-byte aligned");
  const int rb = rows_per_block(H_I);
  const int nrb = (Tq + rb - 1) / rb;
  const int grid = nrb < num_sms() ? nrb : num_sms();
  const WsPrefill ws = prefill_ws_layout(workspace, Tq, H_I, topk, grid);
  if (!workspace || ws_bytes < ws.bytes)
    return fail(DSA_ERR_WORKSPACE, "workspace %zu bytes, need %zu", ws_bytes, ws.bytes);
  if (!aligned16(workspace)) return fail(DSA_ERR_INVALID_ARG, "workspace not 16-byte aligned");
  IdxPrefillParams p = {};
  p.q_scale = q_scale;
  p.w = w;
  p.k_scale = k_scale;
  p.L = L;
  p.q0 = q0;
  p.Tq = Tq;
  p.topk = topk;
  p.rb_begin = 0;
  p.rb_end = nrb;
  p.cand = ws.cand;
  p.cap = select_cap(topk);
  p.idx = idx;
  p.spec_min_t = spec_min_row(topk);
  p.redo_count = ws.redo;
  p.redo_list = ws.redo + 4;
  p.block_table = pg.block_table;
  p.page_shift = pg.page_shift;
  p.pool_pages = pg.pool_pages;
  const cudaError_t me = cudaMemsetAsync(ws.redo, 0, sizeof(int), st);
  if (me != cudaSuccess) return cuda_fail(me, "cudaMemsetAsync");
  dsa_status s = (select_mq(topk) == 1) ? dispatch_prefill<true, 1>(H_I, d_I, q_I, k_cache, p, grid, st)
                                        : dispatch_prefill<true, 4>(H_I, d_I, q_I, k_cache, p, grid, st);
  if (s != DSA_OK) return s;
  // Row blocks whose sampled start proved too high run again with plain
  // streaming; the count is read on the device, so an empty list costs one
  // short launch and no host synchronisation.
  IdxPrefillParams r = p;
  r.spec_min_t = 0;
  r.rb_list = ws.redo + 4;
  r.list_count = ws.redo;
  r.redo_count = nullptr;
  r.redo_list = nullptr;
  return (select_mq(topk) == 1) ? dispatch_prefill<true, 1>(H_I, d_I, q_I, k_cache, r, grid, st)
                                : dispatch_prefill<true, 4>(H_I, d_I, q_I, k_cache, r, grid, st);
}

dsa_status dsa_index_topk(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_cache,
                          const float* k_scale, int L, int H_I, int d_I, int topk, int32_t* idx, void* workspace,
                          size_t ws_bytes, void* stream) {
  return index_topk_impl(q_I, q_scale, w, k_cache, k_scale, 0, L, L, H_I, d_I, topk, idx, workspace, ws_bytes,
                         static_cast<cudaStream_t>(stream));
}

dsa_status dsa_index_topk_chunk(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_cache,
                                const float* k_scale, int q0, int Tq, int L, int H_I, int d_I, int topk, int32_t* idx,
                                void* workspace, size_t ws_bytes, void* stream) {
  return index_topk_impl(q_I, q_scale, w, k_cache, k_scale, q0, Tq, L, H_I, d_I, topk, idx, workspace, ws_bytes,
                         static_cast<cudaStream_t>(stream));
}

dsa_status dsa_index_topk_chunk_paged(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_pool,
                                      const float* k_scale_pool, const int32_t* block_table, int max_blocks,
                                      int page_size, int pool_rows, int q0, int Tq, int L, int H_I, int d_I, int topk,
                                      int32_t* idx, void* workspace, size_t ws_bytes, void* stream) {
  if (!block_table) return fail(DSA_ERR_INVALID_ARG, "null pointer");
  if (page_size < 16 || page_size > 4096 || (page_size & (page_size - 1)))
    return fail(DSA_ERR_INVALID_ARG, "page_size=%d must be a power of two in [16, 4096]", page_size);
  if (pool_rows <= 0 || pool_rows % page_size)
    return fail(DSA_ERR_INVALID_ARG, "pool_rows=%d (a positive multiple of page_size)", pool_rows);
  if (max_blocks <= 0 || static_cast<long long>(max_blocks) * page_size < L)
    return fail(DSA_ERR_INVALID_ARG, "max_blocks=%d pages of %d rows do not cover L=%d", max_blocks, page_size, L);
  if (H_I != 64) return fail(DSA_ERR_UNSUPPORTED, "paged keys: H_I=%d not supported", H_I);
  PrefillKeyPaging pg;
  pg.block_table = block_table;
  pg.page_shift = __builtin_ctz(static_cast<unsigned>(page_size));
  pg.pool_pages = pool_rows / page_size;
  return index_topk_impl(q_I, q_scale, w, k_pool, k_scale_pool, q0, Tq, L, H_I, d_I, topk, idx, workspace, ws_bytes,
                         static_cast<cudaStream_t>(stream), pg);
}

// ---- packed batch of sequences (cu_seqlens) ----
// Workspace: candidate lists as for one sequence, then the re-run list and
// the row-block table (upper bound on the block count).
struct WsVarlen {
  uint64_t* cand;
  int* redo;
  int* table;  // blk_seq[nb_max], blk_lrb[nb_max], cuq[nseq+1], cuk[nseq+1], q0[nseq]
  size_t bytes;
};
static int varlen_max_blocks(int total_q, int nseq, int H_I) { return total_q / rows_per_block(H_I) + nseq + 1; }
static WsVarlen varlen_ws_layout(void* base, int total_q, int nseq, int H_I, int topk, int grid) {
  WsVarlen w;
  const size_t cand_bytes = static_cast<size_t>(grid) * rows_per_block(H_I) * select_cap(topk) * 8;
  const int nbm = varlen_max_blocks(total_q, nseq, H_I);
  const size_t redo_bytes = (static_cast<size_t>(nbm) + 4) * 4;
  const size_t table_bytes = (2 * static_cast<size_t>(nbm) + 3 * static_cast<size_t>(nseq) + 2) * 4;
  char* c = reinterpret_cast<char*>(base);
  w.cand = reinterpret_cast<uint64_t*>(c);
  w.redo = reinterpret_cast<int*>(c + cand_bytes);
  w.table = reinterpret_cast<int*>(c + cand_bytes + redo_bytes);
  w.bytes = cand_bytes + redo_bytes + table_bytes;
  return w;
}

size_t dsa_index_topk_varlen_workspace_size(int total_q, int nseq, int H_I, int d_I, int topk) {
  if (total_q <= 0 || nseq <= 0 || topk <= 0 || !prefill_shape_ok(H_I, d_I)) return 0;
  const int nbm = varlen_max_blocks(total_q, nseq, H_I);
  const int grid = nbm < num_sms() ? nbm : num_sms();
  return varlen_ws_layout(nullptr, total_q, nseq, H_I, topk, grid).bytes;
}

dsa_status dsa_index_topk_varlen(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_cache,
                                 const float* k_scale, const int32_t* cu_q, const int32_t* cu_k,
                                 const int32_t* q_pos0, int nseq, int H_I, int d_I, int topk, int32_t* idx,
                                 void* workspace, size_t ws_bytes, void* stream) {
  if (!q_I || !q_scale || !w || !k_cache || !k_scale || !idx || !cu_q || !cu_k)
    return fail(DSA_ERR_INVALID_ARG, "null pointer");
  if (nseq <= 0) return fail(DSA_ERR_INVALID_ARG, "nseq=%d", nseq);
  if (!prefill_shape_ok(H_I, d_I)) return fail(DSA_ERR_UNSUPPORTED, "H_I=%d d_I=%d not supported", H_I, d_I);
  if (topk < 1 || topk > DSA_MAX_TOPK) return fail(DSA_ERR_UNSUPPORTED, "topk=%d not in [1, %d]", topk, DSA_MAX_TOPK);
  if (cu_q[0] != 0 || cu_k[0] != 0) return fail(DSA_ERR_INVALID_ARG, "cu_q[0] and cu_k[0] must be 0");
  const int RB = rows_per_block(H_I);
  std::vector<int> q0(nseq);
  std::vector<long long> order;  // (-(last position) << 32 | block): longest first
  for (int b = 0; b < nseq; ++b) {
    const int tq = cu_q[b + 1] - cu_q[b], lk = cu_k[b + 1] - cu_k[b];
    q0[b] = q_pos0 ? q_pos0[b] : lk - tq;
    if (tq < 0 || lk < 0 || q0[b] < 0 || static_cast<long long>(q0[b]) + tq > lk)
      return fail(DSA_ERR_INVALID_ARG, "sequence %d: %d queries at position %d, %d keys", b, tq, q0[b], lk);
  }
  const int total_q = cu_q[nseq], total_k = cu_k[nseq];
  if (total_q <= 0 || total_k <= 0) return fail(DSA_ERR_INVALID_ARG, "total_q=%d total_k=%d", total_q, total_k);
  if (static_cast<long long>(total_q) * H_I >= (1ll << 31)) return fail(DSA_ERR_UNSUPPORTED, "total_q*H_I too large");
  if (!aligned16(q_I) || !aligned16(k_cache)) return fail(DSA_ERR_INVALID_ARG, "q_I / k_cache not 16-byte aligned");
  std::vector<int> bseq, blrb;
  {
    std::vector<std::pair<long long, int>> keyed;  // (last position, block) to sort longest first
    std::vector<std::pair<int, int>> blocks;
    for (int b = 0; b < nseq; ++b) {
      const int tq = cu_q[b + 1] - cu_q[b];
      for (int l = 0; l * RB < tq; ++l) {
        keyed.push_back({static_cast<long long>(q0[b]) + std::min((l + 1) * RB, tq), static_cast<int>(blocks.size())});
        blocks.push_back({b, l});
      }
    }
    std::stable_sort(keyed.begin(), keyed.end(), [](const auto& a, const auto& c) { return a.first > c.first; });
    for (const auto& k : keyed) {
      bseq.push_back(blocks[k.second].first);
      blrb.push_back(blocks[k.second].second);
    }
  }
  const int nblk = static_cast<int>(bseq.size());
  const int nbm = varlen_max_blocks(total_q, nseq, H_I);
  const int grid = nbm < num_sms() ? nbm : num_sms();
  const WsVarlen ws = varlen_ws_layout(workspace, total_q, nseq, H_I, topk, grid);
  if (!workspace || ws_bytes < ws.bytes)
    return fail(DSA_ERR_WORKSPACE, "workspace %zu bytes, need %zu", ws_bytes, ws.bytes);
  if (!aligned16(workspace)) return fail(DSA_ERR_INVALID_ARG, "workspace not 16-byte aligned");
  // the table to the device (staged from this host buffer before the call returns)
  std::vector<int> host(2 * static_cast<size_t>(nbm) + 3 * static_cast<size_t>(nseq) + 2, 0);
  std::copy(bseq.begin(), bseq.end(), host.begin());
  std::copy(blrb.begin(), blrb.end(), host.begin() + nbm);
  for (int b = 0; b <= nseq; ++b) {
    host[2 * nbm + b] = cu_q[b];
    host[2 * nbm + nseq + 1 + b] = cu_k[b];
  }
  for (int b = 0; b < nseq; ++b) host[2 * nbm + 2 * (nseq + 1) + b] = q0[b];
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(ws.table, host.data(), host.size() * 4, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(row-block table)");
  e = cudaMemsetAsync(ws.redo, 0, sizeof(int), st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  IdxPrefillParams p = {};
  p.q_scale = q_scale;
  p.w = w;
  p.k_scale = k_scale;
  p.L = total_k;
  p.q0 = 0;
  p.Tq = total_q;
  p.topk = topk;
  p.rb_begin = 0;
  p.rb_end = nblk;
  p.cand = ws.cand;
  p.cap = select_cap(topk);
  p.idx = idx;
  p.spec_min_t = spec_min_row(topk);
  p.redo_count = ws.redo;
  p.redo_list = ws.redo + 4;
  p.blk_seq = ws.table;
  p.blk_lrb = ws.table + nbm;
  p.seq_cuq = ws.table + 2 * nbm;
  p.seq_cuk = ws.table + 2 * nbm + nseq + 1;
  p.seq_q0 = ws.table + 2 * nbm + 2 * (nseq + 1);
  const int g = nblk < grid ? nblk : grid;
  dsa_status s = (select_mq(topk) == 1) ? dispatch_prefill<true, 1>(H_I, d_I, q_I, k_cache, p, g, st)
                                        : dispatch_prefill<true, 4>(H_I, d_I, q_I, k_cache, p, g, st);
  if (s != DSA_OK) return s;
  IdxPrefillParams r = p;
  r.spec_min_t = 0;
  r.rb_list = ws.redo + 4;
  r.list_count = ws.redo;
  r.redo_count = nullptr;
  r.redo_list = nullptr;
  return (select_mq(topk) == 1) ? dispatch_prefill<true, 1>(H_I, d_I, q_I, k_cache, r, g, st)
                                : dispatch_prefill<true, 4>(H_I, d_I, q_I, k_cache, r, g, st);
}

dsa_status dsa_index_topk_rerun_count(const void* workspace, int L, int H_I, int d_I, int topk, int* count,
                                     void* stream) {
  if (!workspace || !count) return fail(DSA_ERR_INVALID_ARG, "null pointer");
  if (L <= 0 || !prefill_shape_ok(H_I, d_I)) return fail(DSA_ERR_INVALID_ARG, "L=%d H_I=%d d_I=%d", L, H_I, d_I);
  const int rb = rows_per_block(H_I);
  const int nrb = (L + rb - 1) / rb;
  const int grid = nrb < num_sms() ? nrb : num_sms();
  const WsPrefill ws = prefill_ws_layout(const_cast<void*>(workspace), L, H_I, topk, grid);
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  e = cudaMemcpy(count, ws.redo, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy");
  return DSA_OK;
}

dsa_status dsa_index_scores(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_cache,
                            const float* k_scale, int L, int H_I, int d_I, int row0, int nrows, float* scores,
                            void* stream) {
  if (!q_I || !q_scale || !w || !k_cache || !k_scale || !scores) return fail(DSA_ERR_INVALID_ARG, "null pointer");
  if (L <= 0 || row0 < 0 || nrows < 0 || row0 + nrows > L)
    return fail(DSA_ERR_INVALID_ARG, "L=%d row0=%d nrows=%d", L, row0, nrows);
  if (!prefill_shape_ok(H_I, d_I)) return fail(DSA_ERR_UNSUPPORTED, "H_I=%d d_I=%d not supported", H_I, d_I);
  if (!aligned16(q_I) || !aligned16(k_cache)) return fail(DSA_ERR_INVALID_ARG, "q_I / k_cache not 16-byte aligned");
  if (nrows == 0) return DSA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t n = static_cast<size_t>(nrows) * L;
  fill_f32_kernel<<<1024, 256, 0, st>>>(scores, n, -INFINITY);
  dsa_status s = check_launch("fill_f32_kernel");
  if (s != DSA_OK) return s;
  const int rb = rows_per_block(H_I);
  IdxPrefillParams p = {};
  p.q_scale = q_scale;
  p.w = w;
  p.k_scale = k_scale;
  p.L = L;
  p.q0 = 0;
  p.Tq = L;
  p.topk = 1;
  p.rb_begin = row0 / rb;
  p.rb_end = (row0 + nrows + rb - 1) / rb;
  p.scores = scores;
  p.row0 = row0;
  p.nrows = nrows;
  const int nrb = p.rb_end - p.rb_begin;
  const int grid = nrb < num_sms() ? nrb : num_sms();
  return dispatch_prefill<false, 1>(H_I, d_I, q_I, k_cache, p, grid, st);
}

dsa_status dsa_sparse_mla_attn_paged(const uint16_t* q, const uint16_t* kv_pool, const int32_t* block_table,
                                     const int32_t* idx, int T, int rows, int pool_rows, int bt_stride,
                                     int max_blocks, int page_size, int Hq, int topk, float scale, uint16_t* out,
                                     float* lse, void* workspace, size_t ws_bytes, void* stream) {
  dsa_status s = check_mla_args(q, kv_pool, idx, T, rows, Hq, topk, scale, out);
  if (s != DSA_OK) return s;
  if (!block_table && T > 0) return fail(DSA_ERR_INVALID_ARG, "null pointer");
  if (page_size < 16 || page_size > 4096 || (page_size & (page_size - 1)) != 0)
    return fail(DSA_ERR_UNSUPPORTED, "page_size=%d (a power of two in [16, 4096])", page_size);
  if (pool_rows <= 0 || bt_stride < 0 || max_blocks <= 0 ||
      static_cast<long long>(max_blocks) * page_size < rows)
    return fail(DSA_ERR_INVALID_ARG, "pool_rows=%d bt_stride=%d max_blocks=%d page_size=%d rows=%d", pool_rows,
                bt_stride, max_blocks, page_size, rows);
  if (T == 0) return DSA_OK;
  float* part = nullptr;
  s = check_split_workspace(workspace, ws_bytes, T, topk, &part);
  if (s != DSA_OK) return s;
  MlaPaging pg;
  pg.block_table = block_table;
  pg.bt_stride = bt_stride;
  pg.page_shift = __builtin_ctz(static_cast<unsigned>(page_size));
  pg.pool_rows = pool_rows;
  return launch_mla(q, kv_pool, idx, T, rows, 0, Hq, topk, scale, out, lse, static_cast<cudaStream_t>(stream), 0, pg,
                    MlaPacked(), part);
}

dsa_status dsa_quantize_e4m3_rows(const float* x, int n, int d, uint8_t* codes, float* scale, void* stream) {
  if (n < 0 || d <= 0) return fail(DSA_ERR_INVALID_ARG, "n=%d d=%d", n, d);
  if (n == 0) return DSA_OK;
  if (!x || !codes || !scale) return fail(DSA_ERR_INVALID_ARG, "null pointer");
  const size_t nx = static_cast<size_t>(n) * d;
  if (overlaps(x, nx * 4, codes, nx) || overlaps(x, nx * 4, scale, static_cast<size_t>(n) * 4))
    return fail(DSA_ERR_INVALID_ARG, "codes / scale overlap x");
  const int grid = n < 8 * num_sms() ? n : 8 * num_sms();
  quantize_e4m3_rows_kernel<<<grid, kQuantThreads, 0, static_cast<cudaStream_t>(stream)>>>(x, n, d, codes, scale);
  return check_launch("quantize_e4m3_rows_kernel");
}

dsa_status dsa_rope_quantize_e4m3_rows(const float* x, const int32_t* pos, int n, int heads, int d, int rope_dim,
                                       double base, int interleaved, uint8_t* codes, float* scale, float* rotated,
                                       void* stream) {
  if (n < 0 || heads <= 0 || d <= 0) return fail(DSA_ERR_INVALID_ARG, "n=%d heads=%d d=%d", n, heads, d);
  if (static_cast<long long>(heads) * d >= (1ll << 31)) return fail(DSA_ERR_UNSUPPORTED, "heads*d too large");
  if (rope_dim < 2 || (rope_dim & 1) || rope_dim > d || rope_dim > 2 * kRopeMaxHalf)
    return fail(DSA_ERR_UNSUPPORTED, "rope_dim=%d must be even, in [2, min(d, %d)]", rope_dim, 2 * kRopeMaxHalf);
  if (!std::isfinite(base) || !(base > 0.0)) return fail(DSA_ERR_INVALID_ARG, "base must be finite and > 0");
  if (n == 0) return DSA_OK;
  if (!x || !pos || !codes || !scale) return fail(DSA_ERR_INVALID_ARG, "null pointer");
  const size_t nx = static_cast<size_t>(n) * heads * d;
  if (overlaps(x, nx * 4, rotated, nx * 4) || overlaps(x, nx * 4, codes, nx) ||
      overlaps(x, nx * 4, scale, static_cast<size_t>(n) * 4))
    return fail(DSA_ERR_INVALID_ARG, "rotated / codes / scale overlap x (no in-place rotation)");
  const int grid = n < 8 * num_sms() ? n : 8 * num_sms();
  rope_quantize_e4m3_rows_kernel<<<grid, kQuantThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      x, pos, n, heads, d, rope_dim, base, interleaved, codes, scale, rotated);
  return check_launch("rope_quantize_e4m3_rows_kernel");
}

dsa_status dsa_dense_mla_attn_causal(const uint16_t* q, const uint16_t* kv, int T, int L, int q0, int Hq, float scale,
                                     uint16_t* out, float* lse, void* stream) {
  if (T < 0 || L <= 0 || q0 < 0 || static_cast<long long>(q0) + T > L)
    return fail(DSA_ERR_INVALID_ARG, "T=%d L=%d q0=%d (need q0 + T <= L)", T, L, q0);
  if (L > DSA_MAX_TOPK)
    return fail(DSA_ERR_UNSUPPORTED, "dense causal attention covers L <= %d (longer sequences take the selection)",
                DSA_MAX_TOPK);
  if (!kv || (T > 0 && (!q || !out))) return fail(DSA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(kv) || !aligned16(out)) return fail(DSA_ERR_INVALID_ARG, "q / kv / out not 16-byte aligned");
  if (Hq < 1 || Hq > 128) return fail(DSA_ERR_UNSUPPORTED, "Hq=%d not in [1, 128]", Hq);
  if (!std::isfinite(scale) || !(scale > 0.f)) return fail(DSA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (T == 0) return DSA_OK;
  return launch_mla(q, kv, nullptr, T, L, 0, Hq, L, scale, out, lse, static_cast<cudaStream_t>(stream), q0);
}

dsa_status dsa_sparse_mla_attn_varlen(const uint16_t* q, const uint16_t* kv, const int32_t* idx, const int32_t* cu_q,
                                      const int32_t* cu_k, int nseq, int T, int total_k, int Hq, int topk, float scale,
                                      uint16_t* out, float* lse, void* stream) {
  dsa_status s = check_mla_args(q, kv, idx, T, total_k, Hq, topk, scale, out);
  if (s != DSA_OK) return s;
  if (nseq < 1) return fail(DSA_ERR_INVALID_ARG, "nseq=%d", nseq);
  if (!cu_q || !cu_k) return fail(DSA_ERR_INVALID_ARG, "null pointer");
  if (T == 0) return DSA_OK;
  MlaPacked pk;
  pk.cu_q = cu_q;
  pk.cu_k = cu_k;
  pk.nseq = nseq;
  return launch_mla(q, kv, idx, T, total_k, 0, Hq, topk, scale, out, lse, static_cast<cudaStream_t>(stream), 0,
                    MlaPaging(), pk);
}

dsa_status dsa_sparse_mla_attn(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int T, int L, int Hq,
                               int topk, float scale, uint16_t* out, float* lse, void* stream) {
  dsa_status s = check_mla_args(q, kv, idx, T, L, Hq, topk, scale, out);
  if (s != DSA_OK) return s;
  if (T == 0) return DSA_OK;
  return launch_mla(q, kv, idx, T, L, 0, Hq, topk, scale, out, lse, static_cast<cudaStream_t>(stream));
}

size_t dsa_index_topk_decode_workspace_size(int B, int L_max, int topk) {
  if (B <= 0 || L_max <= 0 || topk <= 0) return 0;
  const size_t scores = (static_cast<size_t>(B) * L_max * 4 + 255) / 256 * 256;
  const size_t keys = (static_cast<size_t>(B) * topk * 8 + 255) / 256 * 256;
  return scores + keys + static_cast<size_t>(B) * 2048 * 4;
}

dsa_status dsa_index_topk_decode(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_cache,
                                 const float* k_scale, const int32_t* lens, int B, int L_max, int H_I, int d_I,
                                 int topk, int32_t* idx, void* workspace, size_t ws_bytes, void* stream) {
  dsa_status s = check_decode_args(q_I, q_scale, w, k_cache, k_scale, lens, B, L_max, H_I, d_I);
  if (s != DSA_OK) return s;
  if (!idx) return fail(DSA_ERR_INVALID_ARG, "null pointer");
  if (topk < 1 || topk > DSA_MAX_TOPK) return fail(DSA_ERR_UNSUPPORTED, "topk=%d not in [1, %d]", topk, DSA_MAX_TOPK);
  const size_t need = dsa_index_topk_decode_workspace_size(B, L_max, topk);
  if (!workspace || ws_bytes < need) return fail(DSA_ERR_WORKSPACE, "workspace %zu bytes, need %zu", ws_bytes, need);
  if (!aligned16(workspace)) return fail(DSA_ERR_INVALID_ARG, "workspace not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* base = reinterpret_cast<char*>(workspace);
  float* scores = reinterpret_cast<float*>(base);
  const size_t off_keys = (static_cast<size_t>(B) * L_max * 4 + 255) / 256 * 256;
  uint64_t* sel = reinterpret_cast<uint64_t*>(base + off_keys);
  uint32_t* hist = reinterpret_cast<uint32_t*>(base + off_keys + (static_cast<size_t>(B) * topk * 8 + 255) / 256 * 256);
  const cudaError_t e = cudaMemsetAsync(hist, 0, static_cast<size_t>(B) * 2048 * 4, st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(histogram)");
  s = decode_scores(q_I, q_scale, w, k_cache, k_scale, lens, B, L_max, H_I, d_I, scores, hist, st);
  if (s != DSA_OK) return s;
  return launch_decode_select(scores, lens, L_max, topk, hist, sel, idx, B, st);
}

dsa_status dsa_index_topk_decode_paged(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_pool,
                                       const float* k_scale_pool, const int32_t* block_table, const int32_t* lens,
                                       int B, int max_blocks, int page_size, int pool_rows, int H_I, int d_I, int topk,
                                       int32_t* idx, void* workspace, size_t ws_bytes, void* stream) {
  if (!block_table) return fail(DSA_ERR_INVALID_ARG, "null pointer");
  if (page_size < 16 || page_size > 4096 || (page_size & (page_size - 1)))
    return fail(DSA_ERR_INVALID_ARG, "page_size=%d must be a power of two in [16, 4096]", page_size);
  if (max_blocks <= 0 || pool_rows <= 0 || pool_rows % page_size)
    return fail(DSA_ERR_INVALID_ARG, "max_blocks=%d pool_rows=%d (a positive multiple of page_size)", max_blocks,
                pool_rows);
  if (static_cast<long long>(max_blocks) * page_size >= (1ll << 31))
    return fail(DSA_ERR_UNSUPPORTED, "max_blocks*page_size too large");
  const int L_max = max_blocks * page_size;
  dsa_status s = check_decode_args(q_I, q_scale, w, k_pool, k_scale_pool, lens, B, L_max, H_I, d_I);
  if (s != DSA_OK) return s;
  if (!idx) return fail(DSA_ERR_INVALID_ARG, "null pointer");
  if (topk < 1 || topk > DSA_MAX_TOPK) return fail(DSA_ERR_UNSUPPORTED, "topk=%d not in [1, %d]", topk, DSA_MAX_TOPK);
  const size_t need = dsa_index_topk_decode_workspace_size(B, L_max, topk);
  if (!workspace || ws_bytes < need) return fail(DSA_ERR_WORKSPACE, "workspace %zu bytes, need %zu", ws_bytes, need);
  if (!aligned16(workspace)) return fail(DSA_ERR_INVALID_ARG, "workspace not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* base = reinterpret_cast<char*>(workspace);
  float* scores = reinterpret_cast<float*>(base);
  const size_t off_keys = (static_cast<size_t>(B) * L_max * 4 + 255) / 256 * 256;
  uint64_t* sel = reinterpret_cast<uint64_t*>(base + off_keys);
  uint32_t* hist = reinterpret_cast<uint32_t*>(base + off_keys + (static_cast<size_t>(B) * topk * 8 + 255) / 256 * 256);
  const cudaError_t e = cudaMemsetAsync(hist, 0, static_cast<size_t>(B) * 2048 * 4, st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(histogram)");
  KeyPaging pg;
  pg.block_table = block_table;
  pg.bt_stride = max_blocks;
  pg.page_shift = __builtin_ctz(static_cast<unsigned>(page_size));
  pg.pool_pages = pool_rows / page_size;
  s = decode_scores(q_I, q_scale, w, k_pool, k_scale_pool, lens, B, L_max, H_I, d_I, scores, hist, st, pg);
  if (s != DSA_OK) return s;
  return launch_decode_select(scores, lens, L_max, topk, hist, sel, idx, B, st);
}

dsa_status dsa_index_scores_decode(const uint8_t* q_I, const float* q_scale, const float* w, const uint8_t* k_cache,
                                   const float* k_scale, const int32_t* lens, int B, int L_max, int H_I, int d_I,
                                   float* scores, void* stream) {
  dsa_status s = check_decode_args(q_I, q_scale, w, k_cache, k_scale, lens, B, L_max, H_I, d_I);
  if (s != DSA_OK) return s;
  if (!scores) return fail(DSA_ERR_INVALID_ARG, "null pointer");
  return decode_scores(q_I, q_scale, w, k_cache, k_scale, lens, B, L_max, H_I, d_I, scores, nullptr,
                       static_cast<cudaStream_t>(stream));
}

size_t dsa_sparse_mla_attn_split_workspace_size(int T, int topk) {
  if (T <= 0 || topk <= 0) return 0;
  return mla_split_bytes(T, topk);
}

dsa_status dsa_sparse_mla_attn_decode(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int B, int L_max,
                                      int Hq, int topk, float scale, uint16_t* out, float* lse, void* workspace,
                                      size_t ws_bytes, void* stream) {
  dsa_status s = check_mla_args(q, kv, idx, B, L_max, Hq, topk, scale, out);
  if (s != DSA_OK) return s;
  if (B == 0) return DSA_OK;
  float* part = nullptr;
  s = check_split_workspace(workspace, ws_bytes, B, topk, &part);
  if (s != DSA_OK) return s;
  return launch_mla(q, kv, idx, B, L_max, static_cast<long long>(L_max) * DSA_D_QK, Hq, topk, scale, out, lse,
                    static_cast<cudaStream_t>(stream), 0, MlaPaging(), MlaPacked(), part);
}

// ---- decode indexer + top-k with library-owned scratch ----
// For callers that cannot allocate device memory (see dsa.h). The scratch
// lives in this fixed device array: per-key fp32 scores first, then the
// selected 64-bit keys. Host code must not pass the symbol itself to a
// kernel (on the host it only names a stand-in); the device address comes
// from cudaGetSymbolAddress, looked up once per device.
constexpr size_t kNoAllocScoreBytes = static_cast<size_t>(DSA_NOALLOC_MAX_SCORES) * 4;
constexpr size_t kNoAllocKeyBytes = static_cast<size_t>(DSA_NOALLOC_MAX_KEYS) * 8;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScoreBytes + kNoAllocKeyBytes];

namespace {
std::mutex g_noalloc_mu;
constexpr int kNoAllocMaxDevices = 64;
void* g_noalloc_addr[kNoAllocMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (set up on the
// first call per device, with that device current).
dsa_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(DSA_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) return cuda_fail(e, "cudaGetSymbolAddress(g_noalloc_scratch)");
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return DSA_OK;
}
}  // namespace

dsa_status dsa_index_topk_decode_noalloc(const uint8_t* q_I, const float* q_scale, const float* w,
                                         const uint8_t* k_cache, const float* k_scale, const int32_t* lens, int B,
                                         int L_max, int H_I, int d_I, int topk, int32_t* idx, void* stream) {
  dsa_status s = check_decode_args(q_I, q_scale, w, k_cache, k_scale, lens, B, L_max, H_I, d_I);
  if (s != DSA_OK) return s;
  if (!idx) return fail(DSA_ERR_INVALID_ARG, "null pointer");
  if (topk < 1 || topk > DSA_MAX_TOPK) return fail(DSA_ERR_UNSUPPORTED, "topk=%d not in [1, %d]", topk, DSA_MAX_TOPK);
  if (static_cast<unsigned long long>(B) * L_max > DSA_NOALLOC_MAX_SCORES)
    return fail(DSA_ERR_UNSUPPORTED, "B*L_max=%lld exceeds the fixed scratch limit of %u scores",
                static_cast<long long>(B) * L_max, DSA_NOALLOC_MAX_SCORES);
  if (static_cast<unsigned long long>(B) * topk > DSA_NOALLOC_MAX_KEYS)
    return fail(DSA_ERR_UNSUPPORTED, "B*topk=%lld exceeds the fixed scratch limit of %u keys",
                static_cast<long long>(B) * topk, DSA_NOALLOC_MAX_KEYS);
  void* base = nullptr;
  s = noalloc_scratch(&base);
  if (s != DSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* scores = reinterpret_cast<float*>(base);
  uint64_t* sel = reinterpret_cast<uint64_t*>(reinterpret_cast<char*>(base) + kNoAllocScoreBytes);
  s = decode_scores(q_I, q_scale, w, k_cache, k_scale, lens, B, L_max, H_I, d_I, scores, nullptr, st);
  if (s != DSA_OK) return s;
  return launch_decode_select(scores, lens, L_max, topk, nullptr, sel, idx, B, st);
}

dsa_status dsa_get_device_error(void* stream, unsigned int* detail) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int h = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&h, g_device_error, sizeof(h), 0, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "dsa_get_device_error");
  if (detail) *detail = h;
  if (h == 0) return DSA_OK;
  const unsigned int zero = 0;
  e = cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "dsa_get_device_error (clear)");
  const unsigned int code = h & 0xFFu;
  if (code == kErrTimeout) return fail(DSA_ERR_TIMEOUT, "a kernel gave up waiting (site %u)", h >> 8);
  return fail(DSA_ERR_BAD_INDEX, "an index or page-table entry was outside its cache (site %u)", h >> 8);
}

dsa_status dsa_selftest_wait_timeout(long long wait_cycles, void* stream) {
  if (wait_cycles < 0 || wait_cycles > kWaitBoundCycles)
    return fail(DSA_ERR_INVALID_ARG, "wait_cycles=%lld not in [0, %lld]", wait_cycles, kWaitBoundCycles);
  selftest_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(wait_cycles ? wait_cycles
                                                                                         : kWaitBoundCycles);
  return check_launch("selftest_wait_timeout_kernel");
}

const char* dsa_status_string(dsa_status s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_TIMEOUT: return "device wait timed out";
    case DSA_ERR_WORKSPACE: return "workspace too small";
    case DSA_ERR_BAD_INDEX: return "index outside the cache";
  }
  return "unknown status";
}

const char* dsa_last_error(void) { return g_last_error; }

}  // extern "C"
