"""Float64 CPU oracle for the DSA hot path (ctypes binding of dsa_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg use it to check and time the CUDA library. The CUDA library
never imports it, and it imports nothing from the CUDA library.

Functions take host arrays (numpy, or CPU torch tensors) and return numpy
float64 / int32 arrays. The C sources say which passage each step follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB = os.path.join(_HERE, "libdsa_oracle.so")
_lock = threading.Lock()
_lib = None

D_QK = 576
D_V = 512


def build(force: bool = False) -> str:
    """Compile dsa_oracle.c with gcc (-O2, OpenMP) into libdsa_oracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            i64, i32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double
            lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_to_double.restype = f64
            lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_bf16_to_double.restype = f64
            lib.oracle_index_scores.argtypes = [P, P, P, P, P, i64, i32, i32, P, i64, P]
            lib.oracle_index_scores.restype = None
            lib.oracle_topk.argtypes = [P, i64, P, i64, i32, P]
            lib.oracle_topk.restype = None
            lib.oracle_sparse_mla.argtypes = [P, P, P, i32, i64, i32, i32, i32, f64, P, P]
            lib.oracle_sparse_mla.restype = None
            lib.oracle_double_to_e4m3.argtypes = [f64]
            lib.oracle_double_to_e4m3.restype = ctypes.c_uint8
            lib.oracle_quantize_e4m3.argtypes = [P, i64, i64, P, P]
            lib.oracle_quantize_e4m3.restype = None
            lib.oracle_num_threads.argtypes = []
            lib.oracle_num_threads.restype = i32
            _lib = lib
    return _lib


def _np(x, dtype=None):
    """Host numpy view of x (torch CPU tensors via their raw bytes)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                x = x.view(torch.int16).numpy().view(np.uint16)
            elif x.dtype == torch.float8_e4m3fn:
                x = x.view(torch.uint8).numpy()
            else:
                x = x.numpy()
    except ImportError:
        pass
    x = np.ascontiguousarray(x)
    if dtype is not None and x.dtype != dtype:
        x = x.astype(dtype)
    return x


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def e4m3_to_f64(codes) -> np.ndarray:
    """Decode e4m3 bytes with the oracle's own decoder."""
    lib = _load()
    lut = np.array([lib.oracle_e4m3_to_double(c) for c in range(256)], dtype=np.float64)
    return lut[_np(codes, np.uint8)]


def bf16_to_f64(bits) -> np.ndarray:
    lib = _load()
    b = _np(bits)
    if b.dtype != np.uint16:
        b = b.view(np.uint16)
    lut = np.array([lib.oracle_bf16_to_double(c) for c in range(65536)], dtype=np.float64)
    return lut[b]


def double_to_e4m3(x: float) -> int:
    """E4M3 code of x: nearest representable value, ties to even, saturating to +-448."""
    return int(_load().oracle_double_to_e4m3(float(x)))


def quantize_e4m3(x) -> tuple:
    """Per-row quantiser: x [n, d] fp32 -> (codes uint8 [n, d], scale fp32 [n]), scale = absmax/448."""
    xf = np.ascontiguousarray(_np(x, np.float32))
    n, d = xf.shape
    codes = np.empty((n, d), dtype=np.uint8)
    scale = np.empty(n, dtype=np.float32)
    _load().oracle_quantize_e4m3(_ptr(xf), n, d, _ptr(codes), _ptr(scale))
    return codes, scale


def index_scores(q_I, q_scale, w, k_cache, k_scale, rows, *, query_rows=None) -> np.ndarray:
    """I[t, s] in float64 for t in rows, all s < S (-inf where s > t).

    q_I [T, H, D] e4m3 bytes, q_scale [T], w [T, H], k_cache [S, D], k_scale [S].
    Query r is q_I[query_rows[r]] (default: rows[r]) at causal position rows[r].
    """
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    qr = rows if query_rows is None else np.asarray(query_rows, dtype=np.int64)
    q8 = np.ascontiguousarray(_np(q_I, np.uint8)[qr])
    n, H, D = q8.shape
    qs = np.ascontiguousarray(_np(q_scale, np.float32)[qr])
    ww = np.ascontiguousarray(_np(w, np.float32)[qr])
    k8 = _np(k_cache, np.uint8)
    S = k8.shape[0]
    assert k8.shape[1] == D
    ks = _np(k_scale, np.float32)
    assert rows.size == 0 or (rows.min() >= 0 and rows.max() < S)
    out = np.empty((rows.size, S), dtype=np.float64)
    _load().oracle_index_scores(_ptr(q8), _ptr(qs), _ptr(ww), _ptr(k8), _ptr(ks), S, H, D,
                                _ptr(rows), rows.size, _ptr(out))
    return out


def topk(scores, rows, k: int) -> np.ndarray:
    """Ranked top-k of each row's s <= t entries: (score desc, s asc), -1 padded."""
    sc = _np(scores, np.float64)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    assert sc.shape[0] == rows.size
    assert rows.size == 0 or rows.max() < sc.shape[1]
    idx = np.empty((rows.size, k), dtype=np.int32)
    _load().oracle_topk(_ptr(sc), sc.shape[1], _ptr(rows), rows.size, int(k), _ptr(idx))
    return idx


def _bf16_bits(x) -> np.ndarray:
    b = _np(x)
    return b.view(np.uint16) if b.dtype != np.uint16 else b


def sparse_mla(q_rows, kv, idx, scale: float, Dv: int = D_V):
    """u[r, h, :Dv] and lse[r, h] in float64 over the kv rows idx[r] (entries < 0 skipped).

    q_rows [n, Hq, Dqk] bf16 (one entry per query), kv [S, Dqk] bf16, idx [n, k] int32.
    """
    qb = np.ascontiguousarray(_bf16_bits(q_rows))
    kb = _bf16_bits(kv)
    n, Hq, Dqk = qb.shape
    ix = _np(idx, np.int32)
    assert ix.shape[0] == n
    if ix.size:
        assert ix.max() < kb.shape[0]
    k = ix.shape[1]
    out = np.empty((n, Hq, Dv), dtype=np.float64)
    lse = np.empty((n, Hq), dtype=np.float64)
    _load().oracle_sparse_mla(_ptr(qb), _ptr(kb), _ptr(ix), k, n, Hq, Dqk, Dv,
                              float(scale), _ptr(out), _ptr(lse))
    return out, lse


def prefill_rows(inp, rows):
    """All three steps for the given query rows of a PrefillInputs.

    Returns (scores [n, L] f64, idx [n, topk] i32, out [n, Hq, 512] f64, lse [n, Hq] f64).
    """
    rows = np.asarray(rows, dtype=np.int64)
    sc = index_scores(inp.q_I, inp.q_scale, inp.w, inp.k_cache, inp.k_scale, rows)
    ix = topk(sc, rows, inp.topk)
    qb = _bf16_bits(inp.q)[rows]
    out, lse = sparse_mla(qb, inp.kv, ix, inp.scale)
    return sc, ix, out, lse


def decode_seqs(inp, seqs):
    """All three steps for sequences `seqs` of a DecodeInputs (query at t = lens[b]-1).

    Returns a list of (scores [lens[b]] f64, idx [topk] i32, out [Hq, 512] f64, lse [Hq] f64).
    """
    res = []
    lens = _np(inp.lens, np.int32)
    for b in seqs:
        n = int(lens[b])
        t = n - 1
        sc = index_scores(inp.q_I[b:b + 1], inp.q_scale[b:b + 1], inp.w[b:b + 1],
                          inp.k_cache[b, :n], inp.k_scale[b, :n], [t], query_rows=[0])[0]
        ix = topk(sc[None], [t], inp.topk)[0]
        out, lse = sparse_mla(_bf16_bits(inp.q[b:b + 1]), inp.kv[b, :n], ix[None], inp.scale)
        res.append((sc, ix, out[0], lse[0]))
    return res


# ---------------------------------------------------------------------------
# Rotary position encoding of newly appended indexer queries / keys, before
# their FP8 quantisation ("Lightning Indexer 的计算过程", step 2 <1>: the first
# rope_head_dim = 64 dimensions of each query head and of the key are split
# off, rotated by the token's position and joined back to the rest; step 2
# <2>: the result is quantised to FP8 with a scale). The pages do not spell
# the rotation out; this is the rotary encoding as its authors define it
# (RoFormer): dimension pairs are rotated by pos * theta_i with
# theta_i = base^(-2i / rope_dim), i < rope_dim / 2. Which dimensions form a
# pair is a convention the pages leave open: consecutive dimensions
# (2i, 2i+1) when `interleaved`, else (i, i + rope_dim/2).
# ---------------------------------------------------------------------------

def rope(x, pos, *, rope_dim: int = 64, base: float = 10000.0, interleaved: bool = True) -> np.ndarray:
    """Rotate the first rope_dim dimensions of every head of x by its row's position.

    x [n, H, d] or [n, d] (one head), pos [n] integer positions; returns float64
    of x's shape. Dimensions >= rope_dim are returned unchanged.
    """
    xv = np.asarray(_np(x), dtype=np.float64)
    squeeze = xv.ndim == 2
    if squeeze:
        xv = xv[:, None, :]
    n, H, d = xv.shape
    if rope_dim % 2 or rope_dim > d:
        raise ValueError(f"rope_dim={rope_dim} must be even and <= d={d}")
    p = np.asarray(_np(pos), dtype=np.int64).reshape(n)
    half = rope_dim // 2
    out = xv.copy()
    for i in range(half):
        theta = base ** (-2.0 * i / rope_dim)
        ang = p.astype(np.float64) * theta  # exact product of an integer and a double, rounded once
        c, s = np.cos(ang)[:, None], np.sin(ang)[:, None]
        a_dim, b_dim = (2 * i, 2 * i + 1) if interleaved else (i, i + half)
        a, b = xv[:, :, a_dim], xv[:, :, b_dim]
        out[:, :, a_dim] = a * c - b * s
        out[:, :, b_dim] = a * s + b * c
    return out[:, 0, :] if squeeze else out


def rope_quantize_e4m3(x, pos, *, rope_dim: int = 64, base: float = 10000.0, interleaved: bool = True) -> tuple:
    """RoPE, then the per-row FP8 quantiser: x [n, H, d] or [n, d] fp32 ->
    (codes uint8 of x's shape, scale fp32 [n]). The rotated row is rounded to
    fp32 (the quantiser's input precision) and quantised with one scale over
    all of the row's H * d values."""
    r = rope(x, pos, rope_dim=rope_dim, base=base, interleaved=interleaved)
    shape = r.shape
    codes, scale = quantize_e4m3(r.reshape(shape[0], -1).astype(np.float32))
    return codes.reshape(shape), scale
