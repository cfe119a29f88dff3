"""RoPE + FP8 quantiser for appended indexer queries and keys, against the oracle.

The rotated fp32 rows lie within one fp32 ulp of the oracle's float64
rotation, plus 1e-9 of the pair's norm: the kernel rounds its float64
rotation once, and the device's pow and sincos may differ from the host's in
the last float64 ulps, which positions up to 131071 turn into angle
differences of ~1e-11 rad, so a rotated value that nearly cancels can move by
more than one ulp of itself while staying within ~1e-10 of the pair's norm
(a wrong pairing or sign would be off by the norm itself). The codes and scales are
bit-exact against the oracle's quantiser applied to the kernel's own rotated
rows, and at position 0 the whole call equals the plain quantiser bit for bit.
"""
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


def _inputs(n, heads, d, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((n, heads, d), generator=g) * 2.5
    x[3] = 0.0  # an all-zero row: scale 1, zero codes
    pos = torch.randint(0, 131072, (n,), generator=g, dtype=torch.int32)
    pos[0], pos[1], pos[2] = 0, 1, 131071
    return x, pos


@pytest.mark.parametrize("heads,d,rope_dim,interleaved", [(64, 128, 64, True), (64, 128, 64, False),
                                                          (1, 128, 64, True), (8, 64, 64, True),
                                                          (4, 96, 32, False)])
def test_rope_quantiser_matches_the_oracle(dsa, heads, d, rope_dim, interleaved):
    n = 67
    x, pos = _inputs(n, heads, d, seed=heads * 1000 + d + rope_dim + int(interleaved))
    codes, scale, rot = dsa.rope_quantize_e4m3_rows(x.cuda(), pos.cuda(), rope_dim=rope_dim,
                                                    interleaved=interleaved, want_rotated=True)
    rot = rot.cpu().numpy().astype(np.float64)
    ref = oracle.rope(x.numpy(), pos.numpy(), rope_dim=rope_dim, interleaved=interleaved)
    ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
    xn = x.numpy().astype(np.float64)
    norm = np.abs(xn).copy()  # the pair norm on rotated dims, the value itself elsewhere
    half = rope_dim // 2
    for i in range(half):
        a, b = (2 * i, 2 * i + 1) if interleaved else (i, i + half)
        norm[..., a] = norm[..., b] = np.hypot(xn[..., a], xn[..., b])
    err = np.abs(rot - ref)
    assert np.all(err <= ulp + 1e-9 * norm), (err / (ulp + 1e-9 * norm)).max()
    assert np.array_equal(rot[..., rope_dim:], x.numpy()[..., rope_dim:].astype(np.float64))
    c_ref, s_ref = oracle.quantize_e4m3(rot.astype(np.float32).reshape(n, -1))
    assert np.array_equal(codes.cpu().numpy().reshape(n, -1), c_ref)
    assert np.array_equal(scale.cpu().numpy(), s_ref)
    # and against the oracle's own rotation end to end: equal codes except where an fp32 rounding of
    # the rotation differs, which moves a value across a code boundary only when it sits on one
    c_end, s_end = oracle.rope_quantize_e4m3(x.numpy(), pos.numpy(), rope_dim=rope_dim, interleaved=interleaved)
    same = np.mean(codes.cpu().numpy().reshape(n, -1) == c_end.reshape(n, -1))
    assert same >= 0.999


def test_position_zero_is_the_plain_quantiser(dsa):
    x, _ = _inputs(40, 64, 128, seed=9)
    pos = torch.zeros(40, dtype=torch.int32)
    codes, scale, _ = dsa.rope_quantize_e4m3_rows(x.cuda(), pos.cuda())
    c0, s0 = dsa.quantize_e4m3_rows(x.reshape(40, -1).cuda())
    assert torch.equal(codes.reshape(40, -1), c0) and torch.equal(scale, s0)


def test_empty_batch_is_a_no_op(dsa):
    x = torch.empty((0, 64, 128), device="cuda")
    pos = torch.empty((0,), dtype=torch.int32, device="cuda")
    codes, scale, _ = dsa.rope_quantize_e4m3_rows(x, pos)
    assert codes.shape == (0, 64, 128) and scale.shape == (0,)
