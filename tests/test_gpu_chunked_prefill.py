"""Chunked prefill: a chunk of query tokens at positions q0..q0+Tq-1 against
a key cache that already holds them. Row r must equal row q0 + r of the
whole-sequence selection (the selection is exact and the ranking total, so
the two must agree bit for bit), and sampled rows must match the float64
oracle at their positions; attention over the chunk's selection is checked
against the oracle too."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_helpers import attn_close, cpu_topk_of, overlap_excluding_ties

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import long_context_03_b200 as m
    m.lib()
    return m


def _chunk(dsa, P, q0, Tq, L_cache):
    return dsa.index_topk_chunk(P.q_I[q0:q0 + Tq].contiguous(), P.q_scale[q0:q0 + Tq].contiguous(),
                                P.w[q0:q0 + Tq].contiguous(), P.k_cache[:L_cache].contiguous(),
                                P.k_scale[:L_cache].contiguous(), q0, P.topk)


@pytest.mark.parametrize("cfg,q0,Tq", [("tiny", 300, 100), ("tiny", 0, 37), ("tiny", 511, 1),
                                       ("big", 16384, 4096), ("big", 5000, 3001)])
def test_chunk_equals_rows_of_the_whole_sequence(dsa, cfg, q0, Tq):
    if cfg == "tiny":
        P = workloads.make_config("tiny_L512", device="cuda")
    else:
        P = workloads.make_prefill(20480, 64, 128, 16, 2048, seed=13, device="cuda")
    end = q0 + Tq
    full = dsa.index_topk(P.q_I[:end].contiguous(), P.q_scale[:end].contiguous(), P.w[:end].contiguous(),
                          P.k_cache[:end].contiguous(), P.k_scale[:end].contiguous(), P.topk)
    # a cache that ends exactly at the chunk, and one that runs past it
    for L_cache in (end, min(P.L, end + 300)):
        idx = _chunk(dsa, P, q0, Tq, L_cache)
        dsa.check_device_error()
        assert torch.equal(idx, full[q0:end]), (cfg, q0, Tq, L_cache)


def test_chunk_rows_against_the_oracle(dsa):
    P = workloads.make_prefill(8192, 64, 128, 16, 2048, seed=17, device="cuda")
    q0, Tq = 6000, 2192
    idx = _chunk(dsa, P, q0, Tq, P.L).cpu().numpy()
    rows = np.array([q0, q0 + 1, q0 + 1000, P.L - 1])
    h = {k: getattr(P, k).cpu() for k in ("q_I", "q_scale", "w", "k_cache", "k_scale", "q", "kv")}
    ref_sc = oracle.index_scores(h["q_I"], h["q_scale"], h["w"], h["k_cache"], h["k_scale"], rows)
    ref_idx = oracle.topk(ref_sc, rows, P.topk)
    got = idx[rows - q0]
    assert overlap_excluding_ties(got, ref_idx, ref_sc, rows, P.topk) >= 0.999
    for r, t in enumerate(rows):
        sc = dsa.index_scores(P.q_I, P.q_scale, P.w, P.k_cache, P.k_scale, int(t), 1).cpu().numpy()
        assert np.array_equal(got[r], cpu_topk_of(sc, [t], P.topk)[0])
    # attention of the chunk's queries over their selections
    q = P.q[q0:q0 + Tq].contiguous()
    out, _ = dsa.sparse_mla_attn(q, P.kv, torch.from_numpy(idx).cuda(), P.scale)
    ref_o, _ = oracle.sparse_mla(h["q"][rows], h["kv"], got, P.scale)
    ok, mx, rl = attn_close(out[torch.as_tensor(rows - q0, device="cuda")], ref_o)
    assert ok, (mx, rl)
