"""The C ABI library: builds, loads, exports every declared symbol, and
rejects bad arguments before touching the GPU (runs without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from long_context_03_b200 import build
    build.build()
    import long_context_03_b200 as m
    return m.lib()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "dsa_index_topk" in names and "dsa_sparse_mla_attn" in names
    for n in names:
        assert hasattr(lib, n), n


def test_null_pointers_are_rejected(lib):
    st = lib.dsa_index_topk(None, None, None, None, None, 16, 64, 128, 8, None, None, 0, None)
    assert st == -1
    assert b"null" in lib.dsa_last_error()
    st = lib.dsa_sparse_mla_attn(None, None, None, 1, 1, 1, 1, ctypes.c_float(1.0), None, None, None)
    assert st == -1


def test_unsupported_shapes_are_rejected(lib):
    p = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    assert lib.dsa_index_topk(p, p, p, p, p, 16, 32, 128, 8, p, p, 1 << 30, None) == -2
    assert lib.dsa_index_topk(p, p, p, p, p, 16, 64, 128, 4096, p, p, 1 << 30, None) == -2
    assert lib.dsa_sparse_mla_attn(p, p, p, 1, 1, 129, 8, ctypes.c_float(1.0), p, None, None) == -2
    assert lib.dsa_index_topk_decode(p, p, p, p, p, p, 1, 16, 8, 128, 8, p, p, 1 << 30, None) == -2


def test_misaligned_arrays_are_rejected(lib):
    p, bad = ctypes.c_void_p(256), ctypes.c_void_p(257)
    assert lib.dsa_sparse_mla_attn(bad, p, p, 1, 1, 16, 8, ctypes.c_float(1.0), p, None, None) == -1


def test_status_strings(lib):
    assert lib.dsa_status_string(0) == b"ok"
    assert lib.dsa_status_string(-5) == b"workspace too small"


def test_empty_attention_batch_needs_no_pointers(lib):
    # T = 0 returns before any CUDA call, so this runs without a GPU
    kv = ctypes.c_void_p(256)
    assert lib.dsa_sparse_mla_attn(None, kv, None, 0, 4, 16, 8, ctypes.c_float(0.1), None, None, None) == 0
    assert lib.dsa_sparse_mla_attn(None, None, None, 0, 4, 16, 8, ctypes.c_float(0.1), None, None, None) == -1


def test_chunk_entry_rejects_bad_offsets(lib):
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    # q0 + Tq > L
    assert lib.dsa_index_topk_chunk(p, p, p, p, p, 100, 50, 120, 64, 128, 8, p, p, 1 << 30, None) == -1
    # Tq = 0, negative q0
    assert lib.dsa_index_topk_chunk(p, p, p, p, p, 0, 0, 120, 64, 128, 8, p, p, 1 << 30, None) == -1
    assert lib.dsa_index_topk_chunk(p, p, p, p, p, -1, 8, 120, 64, 128, 8, p, p, 1 << 30, None) == -1


def test_varlen_entry_validates_offsets_on_the_host(lib):
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    IA = ctypes.c_int32 * 3
    bad_first = IA(1, 5, 9)
    ok_q, ok_k = IA(0, 4, 8), IA(0, 10, 20)
    too_many_q = IA(0, 12, 16)  # 12 queries against 10 keys
    call = lambda cq, ck: lib.dsa_index_topk_varlen(p, p, p, p, p, ctypes.cast(cq, ctypes.c_void_p),
                                                    ctypes.cast(ck, ctypes.c_void_p), None, 2, 64, 128, 8, p, p,
                                                    1 << 40, None)
    assert call(bad_first, ok_k) == -1
    assert call(too_many_q, ok_k) == -1
    assert lib.dsa_index_topk_varlen_workspace_size(8, 2, 64, 128, 8) > 0


def test_dense_fallback_limits(lib):
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    f = ctypes.c_float(0.1)
    assert lib.dsa_dense_mla_attn_causal(p, p, 4, 4096, 0, 16, f, p, None, None) == -2  # L > 2048
    assert lib.dsa_dense_mla_attn_causal(p, p, 10, 100, 95, 16, f, p, None, None) == -1  # q0 + T > L
    assert lib.dsa_dense_mla_attn_causal(None, p, 0, 100, 0, 16, f, None, None, None) == 0  # empty batch


def test_quantiser_argument_checks(lib):
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    assert lib.dsa_quantize_e4m3_rows(None, 0, 128, None, None, None) == 0  # nothing to do
    assert lib.dsa_quantize_e4m3_rows(p, 4, 0, p, p, None) == -1
    assert lib.dsa_quantize_e4m3_rows(None, 4, 128, p, p, None) == -1


def test_paged_attention_argument_checks(lib):
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    f = ctypes.c_float(0.1)
    # page size not a power of two; table too small for the rows
    assert lib.dsa_sparse_mla_attn_paged(p, p, p, p, 2, 1000, 4096, 16, 16, 48, 16, 8, f, p, None, None, 0,
                                         None) == -2
    assert lib.dsa_sparse_mla_attn_paged(p, p, p, p, 2, 1000, 4096, 15, 15, 64, 16, 8, f, p, None, None, 0,
                                         None) == -1
    # a split workspace that is too small
    assert lib.dsa_sparse_mla_attn_paged(p, p, p, p, 2, 1000, 4096, 16, 16, 64, 16, 8, f, p, None, p, 16,
                                         None) == -5


def test_split_attention_workspace(lib):
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    f = ctypes.c_float(0.1)
    one_slot = (128 * 512 + 256) * 4
    assert lib.dsa_sparse_mla_attn_split_workspace_size(0, 2048) == 0
    # at least two partial slots, and never more than two per possible cluster
    n = lib.dsa_sparse_mla_attn_split_workspace_size(64, 2048)
    assert n >= 2 * one_slot and n % one_slot == 0
    assert lib.dsa_sparse_mla_attn_split_workspace_size(1, 64) == 2 * one_slot  # one chunk: one cluster
    # (q, kv, idx, B, L_max, Hq, topk, scale, out, lse, workspace, ws_bytes, stream)
    assert lib.dsa_sparse_mla_attn_decode(p, p, p, 4, 1000, 16, 256, f, p, None, p, 1024, None) == -5
    assert lib.dsa_sparse_mla_attn_decode(p, p, p, 0, 1000, 16, 256, f, p, None, p, 1024, None) == 0  # nothing to do


def test_paged_decode_indexer_argument_checks(lib):
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    # (q_I, q_scale, w, k_pool, k_scale_pool, table, lens, B, max_blocks, page, pool_rows, H_I, d_I, topk,
    #  idx, workspace, ws_bytes, stream)
    assert lib.dsa_index_topk_decode_paged(p, p, p, p, p, None, p, 2, 8, 64, 1024, 64, 128, 16, p, p, 1 << 30,
                                           None) == -1  # no table
    assert lib.dsa_index_topk_decode_paged(p, p, p, p, p, p, p, 2, 8, 48, 1024, 64, 128, 16, p, p, 1 << 30,
                                           None) == -1  # page not a power of two
    assert lib.dsa_index_topk_decode_paged(p, p, p, p, p, p, p, 2, 8, 64, 1000, 64, 128, 16, p, p, 1 << 30,
                                           None) == -1  # pool not whole pages
    assert lib.dsa_index_topk_decode_paged(p, p, p, p, p, p, p, 2, 8, 64, 1024, 64, 128, 16, p, None, 0,
                                           None) == -5  # no workspace
    assert lib.dsa_index_topk_decode_paged(p, p, p, p, p, p, p, 2, 8, 64, 1024, 32, 128, 16, p, p, 1 << 30,
                                           None) == -2  # H_I outside the supported set


def test_rope_quantiser_argument_checks(lib):
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    b = ctypes.c_double(10000.0)
    # (x, pos, n, heads, d, rope_dim, base, interleaved, codes, scale, rotated, stream)
    assert lib.dsa_rope_quantize_e4m3_rows(p, p, 4, 64, 128, 63, b, 1, p, p, None, None) == -2  # odd
    assert lib.dsa_rope_quantize_e4m3_rows(p, p, 4, 64, 128, 256, b, 1, p, p, None, None) == -2  # > d
    assert lib.dsa_rope_quantize_e4m3_rows(p, p, 4, 64, 128, 64, ctypes.c_double(-1.0), 1, p, p, None,
                                           None) == -1  # base
    assert lib.dsa_rope_quantize_e4m3_rows(None, p, 4, 64, 128, 64, b, 1, p, p, None, None) == -1  # null x
    assert lib.dsa_rope_quantize_e4m3_rows(None, None, 0, 64, 128, 64, b, 1, None, None, None, None) == 0  # empty


def test_quantisers_refuse_outputs_that_overlap_the_input(lib):
    # pointers are only compared, never dereferenced: the overlap check fails first
    x = 1 << 20
    n, heads, d = 4, 64, 128
    row_bytes = heads * d * 4
    other = ctypes.c_void_p(x + 64 * n * row_bytes)
    b = ctypes.c_double(10000.0)
    X = ctypes.c_void_p(x)
    inside = ctypes.c_void_p(x + row_bytes)  # the second row of x
    # (x, pos, n, heads, d, rope_dim, base, interleaved, codes, scale, rotated, stream)
    assert lib.dsa_rope_quantize_e4m3_rows(X, other, n, heads, d, 64, b, 1, other, other, X, None) == -1  # in place
    assert lib.dsa_rope_quantize_e4m3_rows(X, other, n, heads, d, 64, b, 1, other, other, inside, None) == -1
    assert lib.dsa_rope_quantize_e4m3_rows(X, other, n, heads, d, 64, b, 1, inside, other, None, None) == -1
    assert lib.dsa_rope_quantize_e4m3_rows(X, other, n, heads, d, 64, b, 1, other, inside, None, None) == -1
    assert b"overlap" in lib.dsa_last_error()
    # (x, n, d, codes, scale, stream)
    assert lib.dsa_quantize_e4m3_rows(X, n, heads * d, inside, other, None) == -1
    assert lib.dsa_quantize_e4m3_rows(X, n, heads * d, other, X, None) == -1


def test_paged_prefill_chunk_argument_checks(lib):
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    # (q_I, q_scale, w, k_pool, k_scale_pool, table, max_blocks, page, pool_rows, q0, Tq, L, H_I, d_I, topk,
    #  idx, workspace, ws_bytes, stream)
    args = [p, p, p, p, p, p, 16, 64, 1024, 0, 1000, 1000, 64, 128, 64, p, p, 1 << 30, None]
    bad_table = list(args); bad_table[5] = None
    assert lib.dsa_index_topk_chunk_paged(*bad_table) == -1
    bad_page = list(args); bad_page[7] = 100
    assert lib.dsa_index_topk_chunk_paged(*bad_page) == -1
    short_table = list(args); short_table[6] = 15  # 15 pages of 64 rows < L = 1000
    assert lib.dsa_index_topk_chunk_paged(*short_table) == -1
    heads8 = list(args); heads8[12] = 8
    assert lib.dsa_index_topk_chunk_paged(*heads8) == -2


def test_error_strings_cover_every_status(lib):
    for st in (0, -1, -2, -3, -4, -5, -6):
        assert lib.dsa_status_string(st) not in (None, b"unknown status")


def _declared_arity():
    """Number of parameters of every function declared in include/dsa.h."""
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for name, args in re.findall(r"\b(dsa_[a-z_0-9]+)\s*\(([^)]*)\)\s*;", src):
        args = args.strip()
        out[name] = 0 if args in ("", "void") else args.count(",") + 1
    return out


def test_binding_declares_every_entry_with_its_arity(lib):
    # the ctypes binding sets argtypes for each ABI call, with as many arguments as the header
    import long_context_03_b200 as m
    L = m.lib()
    arity = _declared_arity()
    assert len(arity) >= 20
    for name, n in arity.items():
        fn = getattr(L, name)
        assert fn.argtypes is not None, name
        assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)
