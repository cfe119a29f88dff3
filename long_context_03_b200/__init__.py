"""B200 (sm_100a) DeepSeek Sparse Attention hot path: thin Python binding.

Every call here marshals torch CUDA tensors into the C ABI of
libdsa_b200.so (declared in include/dsa.h) and nothing else: the indexer, the
selection and the attention all run in the library's CUDA kernels. PyTorch
only provides device memory and the current stream. There is no CPU fallback:
if the library is missing or fails to load, every call raises.

Build the library first with `python -m long_context_03_b200.build` (or
`__graft_entry__.build()`).
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa_b200.so")

D_QK = 576
D_V = 512
MAX_TOPK = 2048

STATUS = {0: "ok", -1: "invalid argument", -2: "unsupported shape", -3: "CUDA error",
          -4: "device wait timed out", -5: "workspace too small", -6: "index outside the cache"}

_lock = threading.Lock()
_lib = None


class DSAError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded CUDA library (raises if it was not built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m long_context_03_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            P, I, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
            L.dsa_index_topk_workspace_size.argtypes = [I, I, I, I]
            L.dsa_index_topk_workspace_size.restype = SZ
            L.dsa_index_topk.argtypes = [P, P, P, P, P, I, I, I, I, P, P, SZ, P]
            L.dsa_index_scores.argtypes = [P, P, P, P, P, I, I, I, I, I, P, P]
            L.dsa_index_topk_rerun_count.argtypes = [P, I, I, I, I, ctypes.POINTER(I), P]
            L.dsa_index_topk_chunk.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, P, SZ, P]
            L.dsa_index_topk_chunk_paged.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, P, P, SZ, P]
            L.dsa_index_topk_varlen_workspace_size.argtypes = [I, I, I, I, I]
            L.dsa_index_topk_varlen_workspace_size.restype = SZ
            L.dsa_index_topk_varlen.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, P, P, SZ, P]
            L.dsa_sparse_mla_attn.argtypes = [P, P, P, I, I, I, I, F, P, P, P]
            L.dsa_dense_mla_attn_causal.argtypes = [P, P, I, I, I, I, F, P, P, P]
            L.dsa_quantize_e4m3_rows.argtypes = [P, I, I, P, P, P]
            L.dsa_rope_quantize_e4m3_rows.argtypes = [P, P, I, I, I, I, ctypes.c_double, I, P, P, P, P]
            L.dsa_sparse_mla_attn_paged.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, F, P, P, P, SZ, P]
            L.dsa_sparse_mla_attn_varlen.argtypes = [P, P, P, P, P, I, I, I, I, I, F, P, P, P]
            L.dsa_index_topk_decode_workspace_size.argtypes = [I, I, I]
            L.dsa_index_topk_decode_workspace_size.restype = SZ
            L.dsa_index_topk_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, P, P, SZ, P]
            L.dsa_index_topk_decode_paged.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, SZ, P]
            L.dsa_index_scores_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, P, P]
            L.dsa_sparse_mla_attn_split_workspace_size.argtypes = [I, I]
            L.dsa_sparse_mla_attn_split_workspace_size.restype = SZ
            L.dsa_sparse_mla_attn_decode.argtypes = [P, P, P, I, I, I, I, F, P, P, P, SZ, P]
            L.dsa_index_topk_decode_noalloc.argtypes = [P, P, P, P, P, P, I, I, I, I, I, P, P]
            L.dsa_get_device_error.argtypes = [P, ctypes.POINTER(ctypes.c_uint)]
            L.dsa_selftest_wait_timeout.argtypes = [ctypes.c_longlong, P]
            L.dsa_status_string.argtypes = [I]
            L.dsa_status_string.restype = ctypes.c_char_p
            L.dsa_last_error.argtypes = []
            L.dsa_last_error.restype = ctypes.c_char_p
            for name in ("dsa_index_topk", "dsa_index_topk_rerun_count", "dsa_index_topk_chunk",
                         "dsa_index_topk_chunk_paged",
                         "dsa_index_topk_varlen", "dsa_dense_mla_attn_causal", "dsa_quantize_e4m3_rows",
                         "dsa_rope_quantize_e4m3_rows",
                         "dsa_sparse_mla_attn_paged", "dsa_sparse_mla_attn_varlen",
                         "dsa_index_scores", "dsa_sparse_mla_attn", "dsa_index_topk_decode",
                         "dsa_index_scores_decode", "dsa_sparse_mla_attn_decode", "dsa_get_device_error",
                         "dsa_index_topk_decode_noalloc", "dsa_index_topk_decode_paged",
                         "dsa_selftest_wait_timeout"):
                getattr(L, name).restype = I
            _lib = L
    return _lib


def _check(status: int):
    if status != 0:
        raise DSAError(status, lib().dsa_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _req(t: torch.Tensor, name: str, dtype, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _ws(workspace, need: int, device) -> torch.Tensor:
    """The caller's workspace (a contiguous CUDA tensor on the inputs' device; the
    library checks its size and alignment) or a new one of `need` bytes."""
    if workspace is None:
        return torch.empty(max(need, 16), dtype=torch.uint8, device=device)
    if not isinstance(workspace, torch.Tensor) or not workspace.is_cuda or workspace.device != device:
        raise ValueError(f"workspace must be a CUDA tensor on {device}")
    if not workspace.is_contiguous():
        raise ValueError("workspace must be contiguous")
    return workspace


def _u8(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.uint8) if t.dtype == torch.float8_e4m3fn else t


# ----------------------------------------------------------------- prefill

def index_topk_workspace_size(L: int, H_I: int, d_I: int, topk: int) -> int:
    return int(lib().dsa_index_topk_workspace_size(L, H_I, d_I, topk))


def index_topk(q_I, q_scale, w, k_cache, k_scale, topk: int, *, idx=None, workspace=None) -> torch.Tensor:
    """Prefill indexer + top-k: idx [L, topk] int32 (ranked, -1 padded)."""
    q_I, k_cache = _u8(q_I), _u8(k_cache)
    L, H_I, d_I = q_I.shape
    _req(q_I, "q_I", torch.uint8)
    _req(q_scale, "q_scale", torch.float32, (L,))
    _req(w, "w", torch.float32, (L, H_I))
    _req(k_cache, "k_cache", torch.uint8, (L, d_I))
    _req(k_scale, "k_scale", torch.float32, (L,))
    if idx is None:
        idx = torch.empty((L, topk), dtype=torch.int32, device=q_I.device)
    _req(idx, "idx", torch.int32, (L, topk))
    need = index_topk_workspace_size(L, H_I, d_I, topk)
    workspace = _ws(workspace, need, q_I.device)
    _check(lib().dsa_index_topk(_ptr(q_I), _ptr(q_scale), _ptr(w), _ptr(k_cache), _ptr(k_scale), L, H_I, d_I,
                                topk, _ptr(idx), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream(q_I.device)))
    return idx


def index_topk_chunk(q_I, q_scale, w, k_cache, k_scale, q0: int, topk: int, *, idx=None, workspace=None):
    """Chunked prefill: queries q_I [Tq, H_I, d_I] at positions q0..q0+Tq-1 against
    k_cache [L, d_I] (L >= q0 + Tq); idx [Tq, topk] int32 (ranked key positions, -1 padded)."""
    q_I, k_cache = _u8(q_I), _u8(k_cache)
    Tq, H_I, d_I = q_I.shape
    L = k_cache.shape[0]
    _req(q_I, "q_I", torch.uint8)
    _req(q_scale, "q_scale", torch.float32, (Tq,))
    _req(w, "w", torch.float32, (Tq, H_I))
    _req(k_cache, "k_cache", torch.uint8, (L, d_I))
    _req(k_scale, "k_scale", torch.float32, (L,))
    if idx is None:
        idx = torch.empty((Tq, topk), dtype=torch.int32, device=q_I.device)
    _req(idx, "idx", torch.int32, (Tq, topk))
    need = index_topk_workspace_size(Tq, H_I, d_I, topk)
    workspace = _ws(workspace, need, q_I.device)
    _check(lib().dsa_index_topk_chunk(_ptr(q_I), _ptr(q_scale), _ptr(w), _ptr(k_cache), _ptr(k_scale), q0, Tq, L,
                                      H_I, d_I, topk, _ptr(idx), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(q_I.device)))
    return idx


def index_topk_chunk_paged(q_I, q_scale, w, k_pool, k_scale_pool, block_table, q0: int, L: int, topk: int, *,
                          page_size: int = 64, idx=None, workspace=None):
    """Chunked prefill over a paged key cache: k_pool [pool_rows, d_I] e4m3 and k_scale_pool
    [pool_rows] f32 in pages of page_size rows; key s is in page block_table[s // page_size]
    (block_table [max_blocks] int32). Same idx as index_topk_chunk over the gathered cache."""
    q_I, k_pool = _u8(q_I), _u8(k_pool)
    Tq, H_I, d_I = q_I.shape
    pool_rows = k_pool.shape[0]
    bt = block_table.reshape(-1)
    _req(q_I, "q_I", torch.uint8)
    _req(q_scale, "q_scale", torch.float32, (Tq,))
    _req(w, "w", torch.float32, (Tq, H_I))
    _req(k_pool, "k_pool", torch.uint8, (pool_rows, d_I))
    _req(k_scale_pool, "k_scale_pool", torch.float32, (pool_rows,))
    _req(bt, "block_table", torch.int32, (bt.numel(),))
    if idx is None:
        idx = torch.empty((Tq, topk), dtype=torch.int32, device=q_I.device)
    _req(idx, "idx", torch.int32, (Tq, topk))
    need = index_topk_workspace_size(Tq, H_I, d_I, topk)
    workspace = _ws(workspace, need, q_I.device)
    _check(lib().dsa_index_topk_chunk_paged(_ptr(q_I), _ptr(q_scale), _ptr(w), _ptr(k_pool), _ptr(k_scale_pool),
                                            _ptr(bt), bt.numel(), page_size, pool_rows, q0, Tq, L, H_I, d_I, topk,
                                            _ptr(idx), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                            _stream(q_I.device)))
    return idx


def index_topk_varlen(q_I, q_scale, w, k_cache, k_scale, cu_q, cu_k, topk: int, *, q_pos0=None, idx=None,
                      workspace=None):
    """Packed batch: sequence b owns query rows cu_q[b]:cu_q[b+1] and keys cu_k[b]:cu_k[b+1]
    (host integer sequences); its queries sit at positions q_pos0[b].. of its cache (default: the
    last tokens). idx [total_q, topk] int32 of key positions local to each sequence."""
    q_I, k_cache = _u8(q_I), _u8(k_cache)
    total_q, H_I, d_I = q_I.shape
    total_k = k_cache.shape[0]
    cu_q = [int(x) for x in cu_q]
    cu_k = [int(x) for x in cu_k]
    nseq = len(cu_q) - 1
    if len(cu_k) != nseq + 1 or cu_q[-1] != total_q or cu_k[-1] != total_k:
        raise ValueError("cu_q / cu_k do not match the packed tensors")
    _req(q_I, "q_I", torch.uint8)
    _req(q_scale, "q_scale", torch.float32, (total_q,))
    _req(w, "w", torch.float32, (total_q, H_I))
    _req(k_cache, "k_cache", torch.uint8, (total_k, d_I))
    _req(k_scale, "k_scale", torch.float32, (total_k,))
    if idx is None:
        idx = torch.empty((total_q, topk), dtype=torch.int32, device=q_I.device)
    _req(idx, "idx", torch.int32, (total_q, topk))
    need = int(lib().dsa_index_topk_varlen_workspace_size(total_q, nseq, H_I, d_I, topk))
    workspace = _ws(workspace, need, q_I.device)
    IA = ctypes.c_int32 * (nseq + 1)
    cq, ck = IA(*cu_q), IA(*cu_k)
    qp = None if q_pos0 is None else (ctypes.c_int32 * nseq)(*[int(x) for x in q_pos0])
    _check(lib().dsa_index_topk_varlen(_ptr(q_I), _ptr(q_scale), _ptr(w), _ptr(k_cache), _ptr(k_scale),
                                       ctypes.cast(cq, ctypes.c_void_p), ctypes.cast(ck, ctypes.c_void_p),
                                       None if qp is None else ctypes.cast(qp, ctypes.c_void_p), nseq, H_I, d_I,
                                       topk, _ptr(idx), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(q_I.device)))
    return idx


def index_topk_rerun_count(workspace, L: int, H_I: int, d_I: int, topk: int) -> int:
    """Test hook: row blocks the last index_topk call with this workspace recomputed
    because their sampled starting threshold was too high (synchronises)."""
    n = ctypes.c_int(0)
    if not isinstance(workspace, torch.Tensor) or not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA tensor")
    _check(lib().dsa_index_topk_rerun_count(_ptr(workspace), L, H_I, d_I, topk, ctypes.byref(n),
                                            _stream(workspace.device)))
    return int(n.value)


def index_scores(q_I, q_scale, w, k_cache, k_scale, row0: int = 0, nrows: Optional[int] = None,
                 *, scores=None) -> torch.Tensor:
    """Test hook: the GPU's own fp32 scores [nrows, L] for rows row0.. (-inf for s > t)."""
    q_I, k_cache = _u8(q_I), _u8(k_cache)
    L, H_I, d_I = q_I.shape
    if nrows is None:
        nrows = L - row0
    _req(q_I, "q_I", torch.uint8)
    _req(q_scale, "q_scale", torch.float32, (L,))
    _req(w, "w", torch.float32, (L, H_I))
    _req(k_cache, "k_cache", torch.uint8, (L, d_I))
    _req(k_scale, "k_scale", torch.float32, (L,))
    if scores is None:
        scores = torch.empty((nrows, L), dtype=torch.float32, device=q_I.device)
    _req(scores, "scores", torch.float32, (nrows, L))
    _check(lib().dsa_index_scores(_ptr(q_I), _ptr(q_scale), _ptr(w), _ptr(k_cache), _ptr(k_scale), L, H_I, d_I,
                                  row0, nrows, _ptr(scores), _stream(q_I.device)))
    return scores


def sparse_mla_attn(q, kv, idx, scale: float, *, out=None, lse=None, want_lse: bool = False
                    ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Sparse MQA over the latent cache: out [T, Hq, 512] bf16 (and lse [T, Hq] f32)."""
    T, Hq, D = q.shape
    L = kv.shape[0]
    topk = idx.shape[1]
    _req(q, "q", torch.bfloat16, (T, Hq, D_QK))
    _req(kv, "kv", torch.bfloat16, (L, D_QK))
    _req(idx, "idx", torch.int32, (T, topk))
    if out is None:
        out = torch.empty((T, Hq, D_V), dtype=torch.bfloat16, device=q.device)
    _req(out, "out", torch.bfloat16, (T, Hq, D_V))
    if lse is None and want_lse:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _req(lse, "lse", torch.float32, (T, Hq))
    _check(lib().dsa_sparse_mla_attn(_ptr(q), _ptr(kv), _ptr(idx), T, L, Hq, topk, float(scale), _ptr(out),
                                     _ptr(lse), _stream(q.device)))
    return out, lse


def split_workspace_size(T: int, topk: int) -> int:
    """Bytes of the workspace that lets an attention call split the selections over every SM."""
    return int(lib().dsa_sparse_mla_attn_split_workspace_size(T, topk))


def _split_ws(split: bool, workspace, T: int, topk: int, device):
    if not split or T == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(split_workspace_size(T, topk), dtype=torch.uint8, device=device)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous device tensor")
    return workspace, workspace.numel() * workspace.element_size()


def sparse_mla_attn_paged(q, kv_pool, block_table, idx, rows: int, scale: float, *, page_size: int = 64,
                          out=None, lse=None, want_lse: bool = False, split: bool = False, workspace=None):
    """Attention over a paged latent cache. block_table [T, max_blocks] (one table row per token)
    or [1, max_blocks] (shared by all tokens); idx holds logical rows < rows. split: spread the
    selections over every SM with a combine step (decode batches; see sparse_mla_attn_decode)."""
    T, Hq, D = q.shape
    pool_rows = kv_pool.shape[0]
    topk = idx.shape[1]
    nbt, max_blocks = block_table.shape
    _req(q, "q", torch.bfloat16, (T, Hq, D_QK))
    _req(kv_pool, "kv_pool", torch.bfloat16, (pool_rows, D_QK))
    _req(block_table, "block_table", torch.int32, (nbt, max_blocks))
    _req(idx, "idx", torch.int32, (T, topk))
    if nbt not in (1, T):
        raise ValueError("block_table needs one row per token or a single shared row")
    bt_stride = 0 if nbt == 1 else max_blocks
    if out is None:
        out = torch.empty((T, Hq, D_V), dtype=torch.bfloat16, device=q.device)
    _req(out, "out", torch.bfloat16, (T, Hq, D_V))
    if lse is None and want_lse:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _req(lse, "lse", torch.float32, (T, Hq))
    ws, ws_bytes = _split_ws(split, workspace, T, topk, q.device)
    _check(lib().dsa_sparse_mla_attn_paged(_ptr(q), _ptr(kv_pool), _ptr(block_table), _ptr(idx), T, rows, pool_rows,
                                           bt_stride, max_blocks, page_size, Hq, topk, float(scale), _ptr(out),
                                           _ptr(lse), _ptr(ws), ws_bytes, _stream(q.device)))
    return out, lse


def sparse_mla_attn_varlen(q, kv, idx, cu_q, cu_k, scale: float, *, out=None, lse=None, want_lse: bool = False):
    """Attention over a packed batch: sequence b owns query tokens cu_q[b]:cu_q[b+1] and latent rows
    cu_k[b]:cu_k[b+1] of kv; idx holds sequence-local rows (as index_topk_varlen returns them).
    cu_q / cu_k: int32 [nseq+1] on the device (lists are copied there)."""
    T, Hq, D = q.shape
    total_k = kv.shape[0]
    topk = idx.shape[1]
    cu_q = torch.as_tensor(cu_q, dtype=torch.int32, device=q.device).contiguous()
    cu_k = torch.as_tensor(cu_k, dtype=torch.int32, device=q.device).contiguous()
    nseq = cu_q.numel() - 1
    _req(q, "q", torch.bfloat16, (T, Hq, D_QK))
    _req(kv, "kv", torch.bfloat16, (total_k, D_QK))
    _req(idx, "idx", torch.int32, (T, topk))
    _req(cu_q, "cu_q", torch.int32, (nseq + 1,))
    _req(cu_k, "cu_k", torch.int32, (nseq + 1,))
    if out is None:
        out = torch.empty((T, Hq, D_V), dtype=torch.bfloat16, device=q.device)
    _req(out, "out", torch.bfloat16, (T, Hq, D_V))
    if lse is None and want_lse:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _req(lse, "lse", torch.float32, (T, Hq))
    _check(lib().dsa_sparse_mla_attn_varlen(_ptr(q), _ptr(kv), _ptr(idx), _ptr(cu_q), _ptr(cu_k), nseq, T, total_k,
                                            Hq, topk, float(scale), _ptr(out), _ptr(lse), _stream(q.device)))
    return out, lse


def quantize_e4m3_rows(x, *, codes=None, scale=None):
    """x [n, d] f32 (device) -> (codes uint8 [n, d], scale f32 [n]): per-row absmax/448 scale, E4M3 RNE codes."""
    n, d = x.shape
    _req(x, "x", torch.float32, (n, d))
    if codes is None:
        codes = torch.empty((n, d), dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty((n,), dtype=torch.float32, device=x.device)
    _req(codes, "codes", torch.uint8, (n, d))
    _req(scale, "scale", torch.float32, (n,))
    _check(lib().dsa_quantize_e4m3_rows(_ptr(x), n, d, _ptr(codes), _ptr(scale), _stream(x.device)))
    return codes, scale


def rope_quantize_e4m3_rows(x, pos, *, rope_dim: int = 64, base: float = 10000.0, interleaved: bool = True,
                            codes=None, scale=None, want_rotated: bool = False):
    """RoPE on the first rope_dim dims of each head, then the per-row E4M3 quantiser.

    x [n, heads, d] (or [n, d]) f32, pos [n] int32 positions (device) -> (codes uint8 of x's shape,
    scale f32 [n], rotated f32 of x's shape or None)."""
    squeeze = x.dim() == 2
    n = x.shape[0]
    heads, d = (1, x.shape[1]) if squeeze else (x.shape[1], x.shape[2])
    _req(x, "x", torch.float32, tuple(x.shape))
    _req(pos, "pos", torch.int32, (n,))
    if codes is None:
        codes = torch.empty(tuple(x.shape), dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty((n,), dtype=torch.float32, device=x.device)
    _req(codes, "codes", torch.uint8, tuple(x.shape))
    _req(scale, "scale", torch.float32, (n,))
    rotated = torch.empty(tuple(x.shape), dtype=torch.float32, device=x.device) if want_rotated else None
    _check(lib().dsa_rope_quantize_e4m3_rows(_ptr(x), _ptr(pos), n, heads, d, rope_dim, float(base),
                                             1 if interleaved else 0, _ptr(codes), _ptr(scale),
                                             _ptr(rotated) if rotated is not None else None, _stream(x.device)))
    return codes, scale, rotated


def dense_mla_attn_causal(q, kv, scale: float, *, q0: int = 0, out=None, lse=None, want_lse: bool = False):
    """Short sequences (L <= 2048): token t at position q0 + t attends to kv rows 0..q0+t, no indexer.
    q [T, Hq, 576], kv [L, 576] -> out [T, Hq, 512] bf16 (and lse [T, Hq] f32)."""
    T, Hq, D = q.shape
    L = kv.shape[0]
    _req(q, "q", torch.bfloat16, (T, Hq, D_QK))
    _req(kv, "kv", torch.bfloat16, (L, D_QK))
    if out is None:
        out = torch.empty((T, Hq, D_V), dtype=torch.bfloat16, device=q.device)
    _req(out, "out", torch.bfloat16, (T, Hq, D_V))
    if lse is None and want_lse:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _req(lse, "lse", torch.float32, (T, Hq))
    _check(lib().dsa_dense_mla_attn_causal(_ptr(q), _ptr(kv), T, L, q0, Hq, float(scale), _ptr(out), _ptr(lse),
                                           _stream(q.device)))
    return out, lse


# ------------------------------------------------------------------ decode

def index_topk_decode_workspace_size(B: int, L_max: int, topk: int) -> int:
    return int(lib().dsa_index_topk_decode_workspace_size(B, L_max, topk))


def _req_decode(q_I, q_scale, w, k_cache, k_scale, lens):
    B, H_I, d_I = q_I.shape
    L_max = k_cache.shape[1]
    _req(q_I, "q_I", torch.uint8)
    _req(q_scale, "q_scale", torch.float32, (B,))
    _req(w, "w", torch.float32, (B, H_I))
    _req(k_cache, "k_cache", torch.uint8, (B, L_max, d_I))
    _req(k_scale, "k_scale", torch.float32, (B, L_max))
    _req(lens, "lens", torch.int32, (B,))
    return B, H_I, d_I, L_max


def index_topk_decode(q_I, q_scale, w, k_cache, k_scale, lens, topk: int, *, idx=None, workspace=None):
    """Decode indexer + top-k: idx [B, topk] int32 (rows of each sequence's cache)."""
    q_I, k_cache = _u8(q_I), _u8(k_cache)
    B, H_I, d_I, L_max = _req_decode(q_I, q_scale, w, k_cache, k_scale, lens)
    if idx is None:
        idx = torch.empty((B, topk), dtype=torch.int32, device=q_I.device)
    _req(idx, "idx", torch.int32, (B, topk))
    need = index_topk_decode_workspace_size(B, L_max, topk)
    workspace = _ws(workspace, need, q_I.device)
    _check(lib().dsa_index_topk_decode(_ptr(q_I), _ptr(q_scale), _ptr(w), _ptr(k_cache), _ptr(k_scale),
                                       _ptr(lens), B, L_max, H_I, d_I, topk, _ptr(idx), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(q_I.device)))
    return idx


def index_topk_decode_paged(q_I, q_scale, w, k_pool, k_scale_pool, block_table, lens, topk: int, *,
                            page_size: int = 64, idx=None, workspace=None):
    """Decode indexer + top-k over a paged FP8 key cache: k_pool [pool_rows, d_I] e4m3 and
    k_scale_pool [pool_rows] f32 in pages of page_size rows, block_table [B, max_blocks] int32
    (page of key s of sequence b: block_table[b, s // page_size]). Same idx as index_topk_decode
    over the gathered contiguous cache with L_max = max_blocks * page_size."""
    q_I, k_pool = _u8(q_I), _u8(k_pool)
    B, H_I, d_I = q_I.shape
    pool_rows = k_pool.shape[0]
    max_blocks = block_table.shape[1]
    _req(q_I, "q_I", torch.uint8)
    _req(q_scale, "q_scale", torch.float32, (B,))
    _req(w, "w", torch.float32, (B, H_I))
    _req(k_pool, "k_pool", torch.uint8, (pool_rows, d_I))
    _req(k_scale_pool, "k_scale_pool", torch.float32, (pool_rows,))
    _req(block_table, "block_table", torch.int32, (B, max_blocks))
    _req(lens, "lens", torch.int32, (B,))
    if idx is None:
        idx = torch.empty((B, topk), dtype=torch.int32, device=q_I.device)
    _req(idx, "idx", torch.int32, (B, topk))
    need = index_topk_decode_workspace_size(B, max_blocks * page_size, topk)
    workspace = _ws(workspace, need, q_I.device)
    _check(lib().dsa_index_topk_decode_paged(_ptr(q_I), _ptr(q_scale), _ptr(w), _ptr(k_pool), _ptr(k_scale_pool),
                                             _ptr(block_table), _ptr(lens), B, max_blocks, page_size, pool_rows,
                                             H_I, d_I, topk, _ptr(idx), _ptr(workspace),
                                             workspace.numel() * workspace.element_size(), _stream(q_I.device)))
    return idx


def index_topk_decode_noalloc(q_I, q_scale, w, k_cache, k_scale, lens, topk: int, *, idx=None):
    """Decode indexer + top-k whose scratch is a fixed array inside the library
    (for callers that cannot allocate device memory; limits in include/dsa.h).
    Same result as index_topk_decode. Calls overlapping on the GPU race on the
    shared scratch."""
    q_I, k_cache = _u8(q_I), _u8(k_cache)
    B, H_I, d_I, L_max = _req_decode(q_I, q_scale, w, k_cache, k_scale, lens)
    if idx is None:
        idx = torch.empty((B, topk), dtype=torch.int32, device=q_I.device)
    _req(idx, "idx", torch.int32, (B, topk))
    _check(lib().dsa_index_topk_decode_noalloc(_ptr(q_I), _ptr(q_scale), _ptr(w), _ptr(k_cache), _ptr(k_scale),
                                               _ptr(lens), B, L_max, H_I, d_I, topk, _ptr(idx),
                                               _stream(q_I.device)))
    return idx


def index_scores_decode(q_I, q_scale, w, k_cache, k_scale, lens, *, scores=None) -> torch.Tensor:
    """Test hook: decode fp32 scores [B, L_max] (entries s >= lens[b] are left as allocated)."""
    q_I, k_cache = _u8(q_I), _u8(k_cache)
    B, H_I, d_I, L_max = _req_decode(q_I, q_scale, w, k_cache, k_scale, lens)
    if scores is None:
        scores = torch.full((B, L_max), float("-inf"), dtype=torch.float32, device=q_I.device)
    _req(scores, "scores", torch.float32, (B, L_max))
    _check(lib().dsa_index_scores_decode(_ptr(q_I), _ptr(q_scale), _ptr(w), _ptr(k_cache), _ptr(k_scale),
                                         _ptr(lens), B, L_max, H_I, d_I, _ptr(scores), _stream(q_I.device)))
    return scores


def sparse_mla_attn_decode(q, kv, idx, scale: float, *, out=None, lse=None, want_lse: bool = False,
                           split: bool = True, workspace=None):
    """Decode sparse MQA: q [B, Hq, 576], kv [B, L_max, 576] -> out [B, Hq, 512] bf16 (and lse).
    split (default): the (sequence, chunk) work is spread over every SM and a combine step merges
    the parts; workspace (optional, split_workspace_size(B, topk) bytes) avoids an allocation."""
    B, Hq, D = q.shape
    L_max = kv.shape[1]
    topk = idx.shape[1]
    _req(q, "q", torch.bfloat16, (B, Hq, D_QK))
    _req(kv, "kv", torch.bfloat16, (B, L_max, D_QK))
    _req(idx, "idx", torch.int32, (B, topk))
    if out is None:
        out = torch.empty((B, Hq, D_V), dtype=torch.bfloat16, device=q.device)
    _req(out, "out", torch.bfloat16, (B, Hq, D_V))
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _req(lse, "lse", torch.float32, (B, Hq))
    ws, ws_bytes = _split_ws(split, workspace, B, topk, q.device)
    _check(lib().dsa_sparse_mla_attn_decode(_ptr(q), _ptr(kv), _ptr(idx), B, L_max, Hq, topk, float(scale),
                                            _ptr(out), _ptr(lse), _ptr(ws), ws_bytes, _stream(q.device)))
    return out, lse


def device_error(device=None) -> Tuple[int, int]:
    """Synchronise the current stream and read/clear the device error word: (status, raw word)."""
    detail = ctypes.c_uint(0)
    st = lib().dsa_get_device_error(_stream(device), ctypes.byref(detail))
    return int(st), int(detail.value)


def selftest_wait_timeout(wait_cycles: int = 0, device=None):
    """Enqueue the failure-path self-test: a kernel whose bounded wait runs out
    after wait_cycles SM cycles (0: the library's ~1 s bound) and records
    DSA_ERR_TIMEOUT; read it with device_error()."""
    _check(lib().dsa_selftest_wait_timeout(int(wait_cycles), _stream(device)))


def check_device_error(device=None):
    st, raw = device_error(device)
    if st != 0:
        raise DSAError(st, f"{lib().dsa_last_error().decode()} (raw {raw:#x})")
