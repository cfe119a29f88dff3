"""Prefill indexer + top-k on the GPU against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_helpers import cpu_topk_of, overlap_excluding_ties, score_tolerance_ok

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import long_context_03_b200 as m
    m.lib()
    return m


CASES = [
    # (L, H_I, d_I, topk, extra)
    (512, 8, 64, 64, {}),                     # the tiny workload's shapes
    (1000, 64, 128, 64, {}),                  # ragged tail, many list cuts (cap 512)
    (777, 64, 64, 100, {}),
    (300, 8, 128, 64, {}),
    (1000, 64, 128, 128, {"signed_w": True}),  # signed head weights
]


@pytest.mark.parametrize("L,H,D,k,extra", CASES)
def test_scores_match_oracle(dsa, L, H, D, k, extra):
    inp = workloads.make_prefill(L, H, D, 16, k, seed=11, **extra)
    d = inp.to("cuda")
    sc = dsa.index_scores(d.q_I, d.q_scale, d.w, d.k_cache, d.k_scale).cpu().numpy()
    dsa.check_device_error()
    rows = np.arange(L)
    ref = oracle.index_scores(inp.q_I, inp.q_scale, inp.w, inp.k_cache, inp.k_scale, rows)
    ok, worst = score_tolerance_ok(sc, ref, rows)
    assert ok, f"worst error / allowance = {worst}"
    assert np.all(np.isneginf(sc[np.triu_indices(L, 1)]))


@pytest.mark.parametrize("L,H,D,k,extra", CASES)
def test_topk_bit_exact_on_own_scores_and_overlaps_oracle(dsa, L, H, D, k, extra):
    inp = workloads.make_prefill(L, H, D, 16, k, seed=12, **extra)
    d = inp.to("cuda")
    idx = dsa.index_topk(d.q_I, d.q_scale, d.w, d.k_cache, d.k_scale, k).cpu().numpy()
    sc = dsa.index_scores(d.q_I, d.q_scale, d.w, d.k_cache, d.k_scale).cpu().numpy()
    dsa.check_device_error()
    rows = np.arange(L)
    assert np.array_equal(idx, cpu_topk_of(sc, rows, k))
    ref_sc = oracle.index_scores(inp.q_I, inp.q_scale, inp.w, inp.k_cache, inp.k_scale, rows)
    ref_idx = oracle.topk(ref_sc, rows, k)
    assert overlap_excluding_ties(idx, ref_idx, ref_sc, rows, k) >= 0.999
    for t in range(L):  # causality and padding
        n = min(k, t + 1)
        assert np.all((idx[t, :n] >= 0) & (idx[t, :n] <= t))
        assert np.all(idx[t, n:] == -1)


def test_topk_2048_streaming_cuts(dsa):
    # L > cap (4352) so every late row's candidate list is cut while streaming
    L, k = 6000, 2048
    inp = workloads.make_prefill(L, 64, 128, 16, k, seed=13)
    d = inp.to("cuda")
    idx = dsa.index_topk(d.q_I, d.q_scale, d.w, d.k_cache, d.k_scale, k).cpu().numpy()
    rows = np.array([0, 1, 127, 128, 2046, 2047, 2048, 4351, 4352, 4353, 5000, 5998, 5999])
    sc = dsa.index_scores(d.q_I, d.q_scale, d.w, d.k_cache, d.k_scale).cpu().numpy()
    dsa.check_device_error()
    all_rows = np.arange(L)
    assert np.array_equal(idx, cpu_topk_of(sc, all_rows, k))
    ref_sc = oracle.index_scores(inp.q_I, inp.q_scale, inp.w, inp.k_cache, inp.k_scale, rows)
    ok, worst = score_tolerance_ok(sc[rows], ref_sc, rows)
    assert ok, worst
    ref_idx = oracle.topk(ref_sc, rows, k)
    assert overlap_excluding_ties(idx[rows], ref_idx, ref_sc, rows, k) >= 0.999


def test_all_equal_keys_tie_break(dsa):
    L, k = 700, 64
    inp = workloads.make_prefill(L, 64, 128, 16, k, seed=14)
    d = inp.to("cuda")
    kc = d.k_cache[:1].expand(L, -1).contiguous()
    ks = d.k_scale[:1].expand(L).contiguous()
    idx = dsa.index_topk(d.q_I, d.q_scale, d.w, kc, ks, k).cpu().numpy()
    dsa.check_device_error()
    for t in range(L):
        n = min(k, t + 1)
        assert idx[t, :n].tolist() == list(range(n))


def test_repeat_runs_are_identical(dsa):
    inp = workloads.make_prefill(900, 64, 128, 16, 256, seed=15).to("cuda")
    a = dsa.index_topk(inp.q_I, inp.q_scale, inp.w, inp.k_cache, inp.k_scale, 256)
    b = dsa.index_topk(inp.q_I, inp.q_scale, inp.w, inp.k_cache, inp.k_scale, 256)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
