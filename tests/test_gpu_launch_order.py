"""The attention and the decode selection are launched as programmatic
dependents of the previous kernel in the stream: they may start before it
ends, and must not read its outputs early. Here the inputs are produced by
ordinary kernels (torch elementwise ops) right before each call, several
times over; every result must equal the one computed on settled inputs."""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import long_context_03_b200 as m
    m.lib()
    return m


def test_inputs_written_just_before_the_call_are_read_after_they_land(dsa):
    B, L, k = 8, 5000, 2048
    D = workloads.make_decode(B, L, 64, 128, 128, k, seed=71, lens=[5000, 4000, 3000, 2049, 2048, 1000, 17, 1],
                              device="cuda")
    idx = dsa.index_topk_decode(D.q_I, D.q_scale, D.w, D.k_cache, D.k_scale, D.lens, k)
    out, lse = dsa.sparse_mla_attn_decode(D.q, D.kv, idx, D.scale, want_lse=True)
    out1, lse1 = dsa.sparse_mla_attn_decode(D.q, D.kv, idx, D.scale, want_lse=True, split=False)
    torch.cuda.synchronize()
    dsa.check_device_error()
    for _ in range(4):
        # each input comes out of a kernel launched just before the call
        q2 = D.q * 1.0
        idx2 = idx + 0
        o2, l2 = dsa.sparse_mla_attn_decode(q2, D.kv, idx2, D.scale, want_lse=True)
        q3 = D.q * 1.0
        o3, l3 = dsa.sparse_mla_attn_decode(q3, D.kv, idx + 0, D.scale, want_lse=True, split=False)
        s2 = D.q_scale * 1.0
        i2 = dsa.index_topk_decode(D.q_I, s2, D.w * 1.0, D.k_cache, D.k_scale, D.lens, k)
        torch.cuda.synchronize()
        dsa.check_device_error()
        assert torch.equal(o2, out) and torch.equal(l2, lse)
        assert torch.equal(o3, out1) and torch.equal(l3, lse1)
        assert torch.equal(i2, idx)
