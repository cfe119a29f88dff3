"""The synthetic inputs follow the recipe the benchmark and the tests state:
distributions, per-token E4M3 scaling, the planted structure and the fixed
draw order (CPU only; small sizes)."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads


@pytest.fixture(scope="module")
def P():
    return workloads.make_prefill(2048, 64, 128, 16, 2048, seed=0, device="cpu")


def _deq(codes, scale):
    return oracle.e4m3_to_f64(codes.numpy().reshape(codes.shape[0], -1)) * scale.numpy().astype(np.float64)[:, None]


def test_indexer_queries_and_keys_are_standard_normal_per_token_e4m3(P):
    for codes, scale in ((P.q_I, P.q_scale), (P.k_cache, P.k_scale)):
        x = _deq(codes, scale)
        assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.02
        # the largest magnitude of every token lands exactly on the largest finite code
        top = np.abs(oracle.e4m3_to_f64(codes.numpy().reshape(codes.shape[0], -1))).max(axis=1)
        assert np.all(top == 448.0)


def test_weights_queries_and_latent_rows(P):
    w = P.w.numpy()
    assert w.min() >= 0.0 and w.max() < 1.0 / 64 and abs(w.mean() - 0.5 / 64) < 2e-4
    q = P.q.float().numpy()
    assert P.q.dtype == torch.bfloat16 and abs(q.std() - 1.0) < 0.01
    kv = P.kv.float().numpy()
    assert P.kv.dtype == torch.bfloat16 and abs(kv.std() * math.sqrt(576) - 1.0) < 0.02
    assert P.scale == pytest.approx(1 / math.sqrt(576))


def test_planted_rows_carry_the_bias():
    Q = workloads.make_prefill(4096, 64, 128, 1, 2048, seed=0, device="cpu", plant_frac=0.05)
    pl = Q.planted.numpy()
    assert len(pl) == round(0.05 * 4096) and len(set(pl.tolist())) == len(pl)
    x = _deq(Q.k_cache, Q.k_scale)
    rest = np.setdiff1d(np.arange(4096), pl)
    assert abs(x[pl].mean() - 3.0) < 0.05 and abs(x[rest].mean()) < 0.02


def test_draws_are_seeded_and_ordered():
    a = workloads.make_prefill(256, 8, 64, 4, 64, seed=3, device="cpu")
    b = workloads.make_prefill(256, 8, 64, 4, 64, seed=3, device="cpu")
    c = workloads.make_prefill(256, 8, 64, 4, 64, seed=4, device="cpu")
    for f in ("q_I", "q_scale", "w", "k_cache", "k_scale", "q", "kv"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f
        assert not torch.equal(getattr(a, f), getattr(c, f)), f
    # q_I is the first draw: the first query row depends on the seed only, not on the shapes after it
    d = workloads.make_prefill(256, 8, 64, 16, 64, seed=3, device="cpu")
    assert torch.equal(a.q_I, d.q_I) and torch.equal(a.k_cache, d.k_cache)


def test_decode_lengths_default_to_the_cache_length():
    D = workloads.make_decode(3, 300, 64, 128, 8, 64, seed=1, device="cpu")
    assert D.lens.tolist() == [300, 300, 300]
    E = workloads.make_decode(3, 300, 64, 128, 8, 64, seed=1, device="cpu", lens=[1, 150, 300])
    assert E.lens.dtype == torch.int32 and E.lens.tolist() == [1, 150, 300]
