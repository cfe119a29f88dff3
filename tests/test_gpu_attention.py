"""Sparse MQA attention on the GPU against the float64 oracle, same index set."""
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


def _oracle_idx(inp, rows):
    sc = oracle.index_scores(inp.q_I, inp.q_scale, inp.w, inp.k_cache, inp.k_scale, rows)
    return oracle.topk(sc, rows, inp.topk)


def test_tiny_all_rows(dsa, tiny):
    rows = np.arange(tiny.L)
    idx = _oracle_idx(tiny, rows)
    d = tiny.to("cuda")
    out, lse = dsa.sparse_mla_attn(d.q, d.kv, torch.from_numpy(idx).cuda(), tiny.scale, want_lse=True)
    dsa.check_device_error()
    ref, ref_lse = oracle.sparse_mla(oracle._bf16_bits(tiny.q)[rows], tiny.kv, idx, tiny.scale)
    ok, mx, rl = attn_close(out, ref)
    assert ok, (mx, rl)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("Hq,k", [(128, 2048), (128, 96), (64, 256), (1, 32), (17, 200), (100, 2048)])
def test_heads_and_chunks(dsa, Hq, k):
    L = 3000
    inp = workloads.make_prefill(L, 8, 64, Hq, k, seed=21)
    rows = np.array([0, 5, 31, 32, 33, 1000, 2047, 2048, 2999])
    T = len(rows)
    idx = _oracle_idx(inp, rows)
    q_rows = inp.q[rows].contiguous()
    out, lse = dsa.sparse_mla_attn(q_rows.cuda(), inp.kv.cuda(), torch.from_numpy(idx).cuda(), inp.scale,
                                   want_lse=True)
    dsa.check_device_error()
    ref, ref_lse = oracle.sparse_mla(q_rows, inp.kv, idx, inp.scale)
    ok, mx, rl = attn_close(out, ref)
    assert ok, (mx, rl)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=1e-4, atol=1e-4)


def test_many_tokens_per_cluster_and_permutation(dsa):
    # more tokens than clusters: each cluster loops; permuting a row's entries
    # leaves its output unchanged within rounding
    L, k, T = 4096, 512, 400
    inp = workloads.make_prefill(L, 8, 64, 128, k, seed=22)
    g = torch.Generator().manual_seed(5)
    idx = torch.stack([torch.randperm(L, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    idx[3, 100:] = -1
    q = inp.q[:T].contiguous()
    out, _ = dsa.sparse_mla_attn(q.cuda(), inp.kv.cuda(), idx.cuda(), inp.scale)
    dsa.check_device_error()
    sample = [0, 1, 2, 3, 150, 399]
    ref, _ = oracle.sparse_mla(q[sample], inp.kv, idx[sample].numpy(), inp.scale)
    ok, mx, rl = attn_close(out[sample], ref)
    assert ok, (mx, rl)


def test_large_logits_force_rescaling(dsa):
    # scaled-up queries make later chunks exceed the running max by far more
    # than 2^8, exercising the accumulator rescale path
    L, k, T = 2048, 1024, 16
    inp = workloads.make_prefill(L, 8, 64, 128, k, seed=23)
    idx = torch.stack([torch.arange(k, dtype=torch.int32) * 2 for _ in range(T)])
    q = (inp.q[:T].float() * 24.0).to(torch.bfloat16)
    out, lse = dsa.sparse_mla_attn(q.cuda(), inp.kv.cuda(), idx.cuda(), inp.scale, want_lse=True)
    dsa.check_device_error()
    ref, ref_lse = oracle.sparse_mla(q, inp.kv, idx.numpy(), inp.scale)
    ok, mx, rl = attn_close(out, ref)
    assert ok, (mx, rl)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=1e-4, atol=1e-3)


def test_row_with_no_valid_entry_is_zero(dsa):
    inp = workloads.make_prefill(256, 8, 64, 16, 64, seed=24)
    idx = torch.full((2, 64), -1, dtype=torch.int32)
    idx[1, 0] = 7
    out, lse = dsa.sparse_mla_attn(inp.q[:2].cuda(), inp.kv.cuda(), idx.cuda(), inp.scale, want_lse=True)
    dsa.check_device_error()
    assert torch.all(out[0] == 0)
    assert torch.all(torch.isneginf(lse[0]))
    assert torch.equal(out[1].cpu(), inp.kv[7, :512].expand(16, -1))
