"""The allocation-free decode indexer entry point.

dsa_index_topk_decode_noalloc serves callers that cannot allocate device
memory (plugins inside a host framework that owns every device allocation,
serving loops that cannot afford a device-synchronising cudaMalloc). Its
scratch is a fixed array inside the library, so these tests check, through
the C ABI, that it returns exactly what the workspace entry point returns,
on two calls in a row (the array keeps the previous call's contents), and
that it refuses sizes beyond its fixed limit.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import long_context_03_b200 as m
    m.lib()
    return m


def _call_noalloc(dsa, d, topk, idx):
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    B, H_I, d_I = d.q_I.shape
    L_max = d.k_cache.shape[1]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return dsa.lib().dsa_index_topk_decode_noalloc(p(d.q_I), p(d.q_scale), p(d.w), p(d.k_cache), p(d.k_scale),
                                                   p(d.lens), B, L_max, H_I, d_I, topk, p(idx), stream)


def test_noalloc_matches_workspace_entry_point_twice_in_a_row(dsa):
    B, L, k = 8, 65536, 2048          # B*L = 2^19 scores, B*k = 2^14 keys: inside the fixed limit
    lens = [65536, 65535, 1, 2048, 2049, 40000, 12345, 65536]
    d = workloads.make_decode(B, L, 64, 128, 16, k, seed=41, lens=lens, device="cuda")
    ref = dsa.index_topk_decode(d.q_I, d.q_scale, d.w, d.k_cache, d.k_scale, d.lens, k)
    torch.cuda.synchronize()
    for _ in range(2):
        idx = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
        assert _call_noalloc(dsa, d, k, idx) == 0, dsa.lib().dsa_last_error()
        torch.cuda.synchronize()
        dsa.check_device_error()
        assert torch.equal(idx, ref)
    # a different problem right after: the leftover scratch contents must not leak in
    d2 = workloads.make_decode(3, 9000, 64, 64, 16, 512, seed=42, lens=[9000, 100, 4500], device="cuda")
    ref2 = dsa.index_topk_decode(d2.q_I, d2.q_scale, d2.w, d2.k_cache, d2.k_scale, d2.lens, 512)
    idx2 = torch.full((3, 512), -7, dtype=torch.int32, device="cuda")
    assert _call_noalloc(dsa, d2, 512, idx2) == 0, dsa.lib().dsa_last_error()
    torch.cuda.synchronize()
    dsa.check_device_error()
    assert torch.equal(idx2, ref2)


def test_noalloc_refuses_sizes_beyond_its_limit(dsa):
    d = workloads.make_decode(2, 256, 64, 128, 16, 64, seed=43, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    idx = torch.empty((64, 64), dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # B * L_max = 64 * 65536 > 2^20: refused before anything is enqueued
    st = dsa.lib().dsa_index_topk_decode_noalloc(p(d.q_I), p(d.q_scale), p(d.w), p(d.k_cache), p(d.k_scale),
                                                 p(d.lens), 64, 65536, 64, 128, 64, p(idx), stream)
    assert st == -2
    assert b"limit" in dsa.lib().dsa_last_error()
