"""Short-sequence dense fallback: causal MQA over the latent rows without the
indexer, checked against the float64 oracle over the selection {0..t} and
against the sparse path whose selection covers every causal key."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_helpers import attn_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import long_context_03_b200 as m
    m.lib()
    return m


def _causal_idx(rows, width):
    idx = np.full((len(rows), width), -1, dtype=np.int32)
    for r, t in enumerate(rows):
        idx[r, :t + 1] = np.arange(t + 1)
    return idx


def test_dense_tiny_all_tokens(dsa):
    P = workloads.make_config("tiny_L512", device="cuda")
    out, lse = dsa.dense_mla_attn_causal(P.q, P.kv, P.scale, want_lse=True)
    dsa.check_device_error()
    rows = np.arange(P.L)
    ref_o, ref_l = oracle.sparse_mla(P.q.cpu(), P.kv.cpu(), _causal_idx(rows, P.L), P.scale)
    ok, mx, rl = attn_close(out, ref_o)
    assert ok, (mx, rl)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_l, rtol=1e-4, atol=1e-4)


def test_dense_chunk_offset(dsa):
    P = workloads.make_config("tiny_L512", device="cuda")
    q0, T = 300, 100
    out, _ = dsa.dense_mla_attn_causal(P.q[q0:q0 + T].contiguous(), P.kv, P.scale, q0=q0)
    rows = np.arange(q0, q0 + T)
    ref_o, _ = oracle.sparse_mla(P.q[q0:q0 + T].cpu(), P.kv.cpu(), _causal_idx(rows, P.L), P.scale)
    ok, mx, rl = attn_close(out, ref_o)
    assert ok, (mx, rl)


def test_dense_2048_matches_oracle_and_sparse_path(dsa):
    P = workloads.make_prefill(2048, 64, 128, 128, 2048, seed=23, device="cuda")
    out, _ = dsa.dense_mla_attn_causal(P.q, P.kv, P.scale)
    idx = dsa.index_topk(P.q_I, P.q_scale, P.w, P.k_cache, P.k_scale, 2048)  # every causal key, ranked
    sp, _ = dsa.sparse_mla_attn(P.q, P.kv, idx, P.scale)
    dsa.check_device_error()
    rows = np.array([0, 1, 127, 128, 1000, 2047])
    ref_o, _ = oracle.sparse_mla(P.q[torch.as_tensor(rows, device="cuda")].cpu(), P.kv.cpu(),
                                 _causal_idx(rows, 2048), P.scale)
    sel = torch.as_tensor(rows, device="cuda")
    for got in (out, sp):
        ok, mx, rl = attn_close(got[sel], ref_o)
        assert ok, (mx, rl)
