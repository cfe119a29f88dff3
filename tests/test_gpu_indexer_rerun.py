"""The prefill selection's sampled starting threshold and its recovery path.

Long rows start their threshold at a score taken from 8 sampled key tiles
(the middle tile of each of 8 equal strata of the row block's key range). If
the sample is unrepresentative, a row ends with fewer than topk admitted keys
and its row block is recomputed with plain streaming inside the same call.
These tests make the sample unrepresentative on purpose (the sampled tiles
of the last row blocks get keys far above the rest) and check that the
result is still the exact top-k, and that ordinary inputs need no recovery.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_helpers import cpu_topk_of, overlap_excluding_ties, score_tolerance_ok

pytestmark = pytest.mark.gpu

NSAMPLE, BM, RB = 8, 128, 8


@pytest.fixture(scope="module")
def dsa():
    import long_context_03_b200 as m
    m.lib()
    return m


def _sample_tiles(nkt):
    return [((2 * i + 1) * nkt) // (2 * NSAMPLE) for i in range(NSAMPLE)]


def _bias_keys(P, positions, bias=3.0):
    """Add `bias` to every dimension of the indexer keys at `positions`, requantised per token."""
    pos = torch.as_tensor(sorted(positions), dtype=torch.long, device=P.k_cache.device)
    k8 = P.k_cache[pos].view(torch.float8_e4m3fn).float() * P.k_scale[pos, None]
    codes, scale = workloads.quantize_e4m3_per_token(k8 + bias)
    P.k_cache[pos] = codes
    P.k_scale[pos] = scale


def _run(dsa, P):
    ws = torch.empty(dsa.index_topk_workspace_size(P.L, P.H_I, P.d_I, P.topk), dtype=torch.uint8, device="cuda")
    idx = dsa.index_topk(P.q_I, P.q_scale, P.w, P.k_cache, P.k_scale, P.topk, workspace=ws)
    n = dsa.index_topk_rerun_count(ws, P.L, P.H_I, P.d_I, P.topk)
    dsa.check_device_error()
    return idx, n


def _check_rows(dsa, P, idx, rows):
    rows = np.asarray(rows, dtype=np.int64)
    h = {k: getattr(P, k).cpu() for k in ("q_I", "q_scale", "w", "k_cache", "k_scale")}
    ref_sc = oracle.index_scores(h["q_I"], h["q_scale"], h["w"], h["k_cache"], h["k_scale"], rows)
    gidx = idx[torch.as_tensor(rows, device="cuda")].cpu().numpy()
    assert overlap_excluding_ties(gidx, oracle.topk(ref_sc, rows, P.topk), ref_sc, rows, P.topk) >= 0.999
    for r, t in enumerate(rows):
        sc = dsa.index_scores(P.q_I, P.q_scale, P.w, P.k_cache, P.k_scale, int(t), 1).cpu().numpy()
        assert np.array_equal(gidx[r], cpu_topk_of(sc, [t], P.topk)[0])
        ok, worst = score_tolerance_ok(sc, ref_sc[r:r + 1], [t])
        assert ok, worst


def test_unrepresentative_sample_is_recomputed(dsa):
    L = 20480
    P = workloads.make_prefill(L, 64, 128, 16, 2048, seed=11, device="cuda")
    # the last row block spans rows 20472..20479 and keys in 160 tiles
    nkt = (L - 1) // BM + 1
    biased = [tile * BM + c for tile in _sample_tiles(nkt) for c in range(BM)]
    _bias_keys(P, biased)
    idx, n = _run(dsa, P)
    assert n >= 1  # the last row blocks sampled only biased keys: 1024 < topk admitted
    _check_rows(dsa, P, idx, [L - 1, L - 8, L - 129, 16400])


def test_representative_inputs_need_no_recompute(dsa):
    P = workloads.make_config("prefill_L32768_planted", device="cuda")
    idx, n = _run(dsa, P)
    nrb = (P.L + RB - 1) // RB
    assert n <= nrb // 1000  # at most 0.1% of row blocks
    _check_rows(dsa, P, idx, [P.L - 1, 20000])
    Q = workloads.make_prefill(32768, 64, 128, 16, 2048, seed=5, device="cuda")
    idx, n = _run(dsa, Q)
    assert n <= nrb // 1000
    _check_rows(dsa, Q, idx, [32767, 17000])
