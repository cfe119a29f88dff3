"""Parity at the full workload sizes, on sampled outputs.

Each test runs the whole hot path on one of the method-shaped workloads
(L = 8192, L = 32768 with planted keys, L = 131072, and decode 64 x 65536)
through the same calls bench.py times, then checks sampled query rows /
sequences against the float64 oracle: scores within 1e-4 relative, the
selection bit-exact against a CPU top-k of the GPU's own scores and at least
99.9% overlap with the oracle's (exact ties excluded), and attention within
2e-2 max-abs / 1e-2 relative on the GPU's own selection.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_helpers import attn_close, cpu_topk_of, overlap_excluding_ties, score_tolerance_ok

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import long_context_03_b200 as m
    m.lib()
    return m


def _host(t):
    return t.detach().cpu()


def _check_prefill_rows(dsa, P, idx, out, rows, score_block_rows):
    """Oracle checks of sampled rows of a prefill run."""
    L, k = P.L, P.topk
    rows = np.asarray(sorted(set(int(r) for r in rows)), dtype=np.int64)
    h = {n: _host(getattr(P, n)) for n in ("q_I", "q_scale", "w", "k_cache", "k_scale", "kv")}
    ref_sc = oracle.index_scores(h["q_I"][rows], h["q_scale"][rows], h["w"][rows], h["k_cache"], h["k_scale"], rows,
                                 query_rows=np.arange(len(rows)))
    ref_idx = oracle.topk(ref_sc, rows, k)
    gidx = _host(idx[torch.as_tensor(rows, device=idx.device)]).numpy()
    assert overlap_excluding_ties(gidx, ref_idx, ref_sc, rows, k) >= 0.999
    for r, t in enumerate(rows):
        n = min(k, t + 1)
        assert np.all((gidx[r, :n] >= 0) & (gidx[r, :n] <= t)) and np.all(gidx[r, n:] == -1)
    # GPU scores (test hook) for a few contiguous row blocks: tolerance and bit-exact top-k
    for r0 in score_block_rows:
        nb = min(4, L - r0)
        sc = _host(dsa.index_scores(P.q_I, P.q_scale, P.w, P.k_cache, P.k_scale, r0, nb)).numpy()
        rr = np.arange(r0, r0 + nb)
        assert np.array_equal(_host(idx[r0:r0 + nb]).numpy(), cpu_topk_of(sc, rr, k))
        sel = [np.where(rows == t)[0][0] for t in rr if t in rows]
        if sel:
            ok, worst = score_tolerance_ok(sc[[int(t - r0) for t in rr if t in rows]], ref_sc[sel], rows[sel])
            assert ok, worst
    # attention on the GPU's own selection
    ref_o, _ = oracle.sparse_mla(_host(P.q[torch.as_tensor(rows, device=P.q.device)]), h["kv"], gidx, P.scale)
    ok, mx, rl = attn_close(out[torch.as_tensor(rows, device=out.device)], ref_o)
    assert ok, (mx, rl)


def _run_prefill(dsa, P):
    idx = dsa.index_topk(P.q_I, P.q_scale, P.w, P.k_cache, P.k_scale, P.topk)
    out, _ = dsa.sparse_mla_attn(P.q, P.kv, idx, P.scale)
    dsa.check_device_error()
    return idx, out


def test_prefill_L8192(dsa):
    P = workloads.make_config("prefill_L8192", device="cuda")
    idx, out = _run_prefill(dsa, P)
    rows = [0, 1, 2046, 2047, 2048, 4095, 5000, 8190, 8191]
    _check_prefill_rows(dsa, P, idx, out, rows, score_block_rows=[2044, 8188])


def test_prefill_L32768_planted(dsa):
    P = workloads.make_config("prefill_L32768_planted", device="cuda")
    idx, out = _run_prefill(dsa, P)
    rows = [0, 2047, 2048, 16383, 32766, 32767]
    _check_prefill_rows(dsa, P, idx, out, rows, score_block_rows=[32764])
    planted = set(_host(P.planted).tolist())
    last = _host(idx[-1]).tolist()
    assert np.mean([s in planted for s in last]) > 0.05


def test_prefill_L131072(dsa):
    P = workloads.make_config("prefill_L131072", device="cuda")
    idx, out = _run_prefill(dsa, P)
    g = np.random.default_rng(7)
    # rows from every class of row block: short rows (t < 2048, all keys
    # selected), the streamed range below the sampled starting thresholds,
    # the sampled range t >= 16384 (most of the work), the block edges around
    # the score-hook blocks, and the last block
    rows = ([0, 1, 2046, 2047, 2048, 2049] + g.choice(np.arange(2050, 16384), 8, replace=False).tolist()
            + g.choice(np.arange(16384, 131064), 40, replace=False).tolist()
            + [16383, 16384, 16385, 65535, 65536, 65537, 99999, 100000] + list(range(131064, 131072)))
    _check_prefill_rows(dsa, P, idx, out, rows, score_block_rows=[1024, 16384, 65536, 131068])
    del P, idx, out
    torch.cuda.empty_cache()


def test_decode_B64_L65536(dsa):
    D = workloads.make_config("decode_B64_L65536", device="cuda")
    idx = dsa.index_topk_decode(D.q_I, D.q_scale, D.w, D.k_cache, D.k_scale, D.lens, D.topk)
    out, lse = dsa.sparse_mla_attn_decode(D.q, D.kv, idx, D.scale, want_lse=True)
    sc = dsa.index_scores_decode(D.q_I, D.q_scale, D.w, D.k_cache, D.k_scale, D.lens)
    dsa.check_device_error()
    seqs = [0, 17, 63]
    sub = workloads.DecodeInputs(len(seqs), D.L, D.H_I, D.d_I, D.Hq, D.topk, D.scale,
                                 *[_host(getattr(D, n)[seqs]) for n in
                                   ("q_I", "q_scale", "w", "k_cache", "k_scale", "q", "kv", "lens")])
    res = oracle.decode_seqs(sub, range(len(seqs)))
    gidx = _host(idx).numpy()
    gsc = _host(sc).numpy()
    for i, b in enumerate(seqs):
        ref_sc, ref_idx, _, _ = res[i]
        t = D.L - 1
        ok, worst = score_tolerance_ok(gsc[b:b + 1], ref_sc[None], [t])
        assert ok, worst
        assert np.array_equal(gidx[b], cpu_topk_of(gsc[b:b + 1], [t], D.topk)[0])
        assert overlap_excluding_ties(gidx[b:b + 1], ref_idx[None], ref_sc[None], [t], D.topk) >= 0.999
        ref_o, ref_l = oracle.sparse_mla(oracle._bf16_bits(sub.q[i:i + 1]), sub.kv[i], gidx[b:b + 1], D.scale)
        ok, mx, rl = attn_close(out[b:b + 1], ref_o)
        assert ok, (b, mx, rl)
        np.testing.assert_allclose(_host(lse[b]).numpy(), ref_l[0], rtol=1e-4, atol=1e-4)


# ------------------------------------------------------------------ edges

def test_single_token_and_topk_above_length(dsa):
    for L, k in [(1, 64), (5, 2048), (130, 129)]:
        P = workloads.make_prefill(L, 64, 128, 16, k, seed=50 + L, device="cuda")
        idx, out = _run_prefill(dsa, P)
        gidx = _host(idx).numpy()
        for t in range(min(L, k)):  # t + 1 <= k: every causal key, then -1
            assert sorted(gidx[t, :t + 1].tolist()) == list(range(t + 1))
            assert np.all(gidx[t, t + 1:] == -1)
        if L > k:  # longer rows: the oracle's exact selection
            rows = np.arange(k, L)
            ref_sc = oracle.index_scores(_host(P.q_I), _host(P.q_scale), _host(P.w), _host(P.k_cache),
                                         _host(P.k_scale), rows)
            assert overlap_excluding_ties(gidx[rows], oracle.topk(ref_sc, rows, k), ref_sc, rows, k) >= 0.999
        ref_o, _ = oracle.sparse_mla(_host(P.q), _host(P.kv), gidx, P.scale)
        ok, mx, rl = attn_close(out, ref_o)
        assert ok, (L, k, mx, rl)


def test_empty_attention_batch_is_a_no_op(dsa):
    q = torch.empty((0, 16, 576), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((4, 576), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((0, 8), dtype=torch.int32, device="cuda")
    out, _ = dsa.sparse_mla_attn(q, kv, idx, 0.1)
    dsa.check_device_error()
    assert out.shape == (0, 16, 512)


def test_out_of_range_index_is_skipped_and_reported(dsa):
    P = workloads.make_prefill(64, 8, 64, 16, 8, seed=60, device="cuda")
    idx = torch.tensor([[0, 1, 2, 500, -1, -1, -1, -1]], dtype=torch.int32, device="cuda")
    out, _ = dsa.sparse_mla_attn(P.q[:1].contiguous(), P.kv, idx, P.scale)
    st, raw = dsa.device_error()
    assert st == -6  # DSA_ERR_BAD_INDEX
    ref_o, _ = oracle.sparse_mla(_host(P.q[:1]), _host(P.kv), np.array([[0, 1, 2, -1]], np.int32), P.scale)
    ok, mx, rl = attn_close(out, ref_o)
    assert ok, (mx, rl)
    assert dsa.device_error()[0] == 0  # the word was cleared
