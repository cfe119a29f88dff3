"""Decode indexer, top-k and attention on the GPU against the float64 oracle."""
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


@pytest.mark.parametrize("d_I", [128, 64])
def test_decode_path(dsa, d_I):
    B, L, k = 6, 5000, 2048
    lens = [5000, 4999, 1, 2048, 2049, 3333]
    inp = workloads.make_decode(B, L, 64, d_I, 128, k, seed=31, lens=lens)
    d = inp.to("cuda")
    sc = dsa.index_scores_decode(d.q_I, d.q_scale, d.w, d.k_cache, d.k_scale, d.lens).cpu().numpy()
    idx = dsa.index_topk_decode(d.q_I, d.q_scale, d.w, d.k_cache, d.k_scale, d.lens, k)
    out, lse = dsa.sparse_mla_attn_decode(d.q, d.kv, idx, inp.scale, want_lse=True)
    dsa.check_device_error()
    idx = idx.cpu().numpy()
    res = oracle.decode_seqs(inp, range(B))
    for b in range(B):
        n = lens[b]
        t = n - 1
        ref_sc, ref_idx, ref_out, ref_lse = res[b]
        ok, worst = score_tolerance_ok(sc[b:b + 1, :n], ref_sc[None], [t])
        assert ok, (b, worst)
        assert np.array_equal(idx[b], cpu_topk_of(sc[b:b + 1, :n], [t], k)[0])
        assert overlap_excluding_ties(idx[b:b + 1], ref_idx[None], ref_sc[None], [t], k) >= 0.999
        # attention over the GPU's own selection, checked against the oracle on that selection
        ref_o, ref_l = oracle.sparse_mla(oracle._bf16_bits(inp.q[b:b + 1]), inp.kv[b, :n], idx[b:b + 1], inp.scale)
        ok, mx, rl = attn_close(out[b:b + 1], ref_o)
        assert ok, (b, mx, rl)
        np.testing.assert_allclose(lse[b].cpu().numpy(), ref_l[0], rtol=1e-4, atol=1e-4)


def test_decode_selection_with_all_scores_tied(dsa):
    # one 11-bit bin holds every key: 40000 keys overflow the on-chip bin
    # buffer (global multi-pass path), 10000 keys fit it; ties go to the
    # lower index, so the answer is 0..k-1 in order
    B, L, k = 3, 40000, 2048
    lens = [40000, 10000, 3000]
    inp = workloads.make_decode(B, L, 64, 128, 16, k, seed=41, lens=lens)
    inp.k_cache[:] = inp.k_cache[:, :1]
    inp.k_scale[:] = inp.k_scale[:, :1]
    d = inp.to("cuda")
    sc = dsa.index_scores_decode(d.q_I, d.q_scale, d.w, d.k_cache, d.k_scale, d.lens).cpu().numpy()
    idx = dsa.index_topk_decode(d.q_I, d.q_scale, d.w, d.k_cache, d.k_scale, d.lens, k)
    dsa.check_device_error()
    idx = idx.cpu().numpy()
    for b in range(B):
        n = lens[b]
        assert np.all(sc[b, :n] == sc[b, 0])
        assert np.array_equal(idx[b], np.arange(k, dtype=np.int32))
        assert np.array_equal(idx[b], cpu_topk_of(sc[b:b + 1, :n], [n - 1], k)[0])


@pytest.mark.parametrize("B,Hq,lens", [
    (1, 128, [3001]),                      # one sequence over 16 clusters
    (3, 16, [2048, 1, 700]),               # a sequence with one row: its other parts are empty
    (30, 128, None),                       # pieces of about six chunks, sequences over two or three clusters
    (5, 17, [3000, 1, 2048, 999, 2500]),   # an odd head count: partial output boxes and a half-used combine block
    (100, 128, None),                      # a batch that fills the GPU: one cluster per sequence
])
def test_split_selections_match_the_oracle(dsa, B, Hq, lens):
    """Flash-decoding: the (sequence, chunk) work spread over every cluster and
    combined equals the oracle, and the unsplit call up to rounding."""
    L, k = 3072, 2048
    inp = workloads.make_decode(B, L, 64, 128, Hq, k, seed=57, lens=lens)
    d = inp.to("cuda")
    idx = dsa.index_topk_decode(d.q_I, d.q_scale, d.w, d.k_cache, d.k_scale, d.lens, k)
    ws = torch.empty(dsa.split_workspace_size(B, k), dtype=torch.uint8, device="cuda")
    out, lse = dsa.sparse_mla_attn_decode(d.q, d.kv, idx, inp.scale, want_lse=True, workspace=ws)
    out1, lse1 = dsa.sparse_mla_attn_decode(d.q, d.kv, idx, inp.scale, want_lse=True, split=False)
    dsa.check_device_error()
    ok, mx, rl = attn_close(out, out1.float().cpu().numpy().astype(np.float64), max_abs=8e-3, rel=4e-3)
    assert ok, (mx, rl)
    np.testing.assert_allclose(lse.cpu().numpy(), lse1.cpu().numpy(), rtol=1e-5, atol=1e-5)
    idx_h = idx.cpu().numpy()
    n_all = inp.lens.numpy() if hasattr(inp.lens, "numpy") else np.asarray(inp.lens)
    for b in sorted({0, B // 2, B - 1}):
        n = int(n_all[b])
        ref_o, ref_l = oracle.sparse_mla(oracle._bf16_bits(inp.q[b:b + 1]), inp.kv[b, :n], idx_h[b:b + 1],
                                         inp.scale)
        ok, mx, rl = attn_close(out[b:b + 1], ref_o)
        assert ok, (b, mx, rl)
        np.testing.assert_allclose(lse[b].cpu().numpy(), ref_l[0], rtol=1e-4, atol=1e-4)
