"""The on-device E4M3 quantiser for appended tokens, bit for bit against the
oracle's definition (scale = absmax/448 in fp32, RNE codes saturating at
+-448)."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import long_context_03_b200 as m
    m.lib()
    return m


@pytest.mark.parametrize("n,d", [(300, 8192), (20000, 128), (257, 100), (1, 1)])
def test_quantiser_matches_the_oracle(dsa, n, d):
    g = torch.Generator().manual_seed(n + d)
    mags = torch.logspace(-6, 3, n)[torch.randperm(n, generator=g)]
    x = torch.randn((n, d), generator=g) * mags[:, None]
    if n > 2:
        x[1] = 0.0  # all-zero row: scale 1
        x[2, :] = 1e-3
        x[2, 0] = 448.0  # one large value: the rest land on subnormal codes
    codes, scale = dsa.quantize_e4m3_rows(x.cuda())
    dsa.check_device_error()
    ref_codes, ref_scale = oracle.quantize_e4m3(x)
    assert np.array_equal(scale.cpu().numpy(), ref_scale)
    assert np.array_equal(codes.cpu().numpy(), ref_codes)


def test_quantised_keys_feed_the_indexer(dsa):
    # keys quantised on the device score exactly like keys quantised by the oracle
    import workloads
    P = workloads.make_prefill(1024, 64, 128, 16, 64, seed=3, device="cuda")
    k_raw = torch.randn((1024, 128), generator=torch.Generator().manual_seed(9))
    codes, scale = dsa.quantize_e4m3_rows(k_raw.cuda())
    ref_codes, ref_scale = oracle.quantize_e4m3(k_raw)
    idx = dsa.index_topk(P.q_I, P.q_scale, P.w, codes, scale, 64)
    idx_ref = dsa.index_topk(P.q_I, P.q_scale, P.w, torch.from_numpy(ref_codes).cuda(),
                             torch.from_numpy(ref_scale).cuda(), 64)
    assert torch.equal(idx, idx_ref)
