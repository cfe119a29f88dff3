"""Pins of the float64 oracle against things other than itself.

Each test names what fixes the expected value: a library routine (torch's
fp8 / bf16 conversions, numpy einsum and lexsort, torch's float64 scaled dot
product attention), a hand-worked example (tests/golden/hand_examples.json), a
closed form, or an invariant of the method.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")


def _torch_dequant(codes, scale):
    """Library dequantisation: torch's own e4m3 decoder, times the per-token scale."""
    c = torch.as_tensor(np.asarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn).to(torch.float64)
    s = torch.as_tensor(np.asarray(scale, dtype=np.float32)).to(torch.float64)
    return (c * s.view(-1, *([1] * (c.dim() - 1)))).numpy()


# --- number formats -------------------------------------------------------

def test_e4m3_decoder_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert set(np.nonzero(nan)[0]) == {0x7F, 0xFF}
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])
    assert mine[0x7E] == 448.0 and mine[0x01] == 2.0 ** -9


def test_bf16_decoder_matches_torch():
    bits = np.arange(65536, dtype=np.uint16)
    mine = oracle.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])


def test_input_quantiser_round_trip_rne_and_saturation():
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = oracle.e4m3_to_f64(finite)
    # decode(encode(decode(c))) == decode(c): one row per value, scale forced to 1
    x = torch.tensor(np.stack([vals, np.full_like(vals, 448.0)], 1), dtype=torch.float32)
    codes, scale = workloads.quantize_e4m3_per_token(x)
    assert torch.all(scale == 1.0)
    assert np.array_equal(oracle.e4m3_to_f64(codes[:, 0].numpy()), vals)
    # round to nearest even at midpoints: 1 + 1/16 lies between 1 (even code) and 1.125
    mid = torch.tensor([[1.0625, 448.0], [1.1875, 448.0], [-1.0625, 448.0]], dtype=torch.float32)
    c, _ = workloads.quantize_e4m3_per_token(mid)
    assert list(oracle.e4m3_to_f64(c[:, 0].numpy())) == [1.0, 1.25, -1.0]
    # the per-token scale maps the absmax to exactly 448
    big = torch.tensor([[1000.0, -250.0, 0.0]], dtype=torch.float32)
    c, s = workloads.quantize_e4m3_per_token(big)
    assert s.item() == pytest.approx(1000.0 / 448.0, rel=1e-7)
    assert oracle.e4m3_to_f64(c[0, 0].item()) == 448.0
    z, sz = workloads.quantize_e4m3_per_token(torch.zeros(1, 4))
    assert sz.item() == 1.0 and int(z.sum()) == 0


# --- hand-worked examples -------------------------------------------------

def test_hand_example_indexer_and_topk():
    g = json.load(open(GOLDEN))["indexer"]
    q8 = np.array(g["q_codes"], dtype=np.uint8)
    k8 = np.array(g["k_codes"], dtype=np.uint8)
    rows = g["q_rows_are_positions"]
    sc = oracle.index_scores(q8, np.array(g["q_scale"], np.float32), np.array(g["w"], np.float32),
                             k8, np.array(g["k_scale"], np.float32), rows,
                             query_rows=list(range(len(rows))))
    for r, exp_row in enumerate(g["scores"]):
        for s, v in enumerate(exp_row):
            if v is None:
                assert sc[r, s] == -np.inf
            else:
                assert sc[r, s] == v
    assert oracle.topk(sc, rows, 2).tolist() == g["top2"]
    assert oracle.topk(sc, rows, 3).tolist() == g["top3"]


def test_hand_example_attention():
    g = json.load(open(GOLDEN))["attention"]
    q = torch.tensor(g["q"], dtype=torch.bfloat16)
    kv = torch.tensor(g["kv"], dtype=torch.bfloat16)
    out, lse = oracle.sparse_mla(q, kv, np.array(g["idx"], np.int32), g["scale"], Dv=g["Dv"])
    np.testing.assert_allclose(out, np.array(g["out"]), rtol=1e-15, atol=0)
    np.testing.assert_allclose(lse, np.array(g["lse"]), rtol=1e-15, atol=0)
    # the closed form behind the fixture
    e = math.e
    assert out[0, 0, 0] == pytest.approx(e / (1 + e), rel=1e-15)


# --- library routines on the tiny workload --------------------------------

def test_scores_match_numpy_einsum(tiny):
    L = tiny.L
    rows = np.arange(L)
    sc = oracle.index_scores(tiny.q_I, tiny.q_scale, tiny.w, tiny.k_cache, tiny.k_scale, rows)
    q = _torch_dequant(tiny.q_I.numpy(), tiny.q_scale.numpy())          # [L, H, D]
    k = _torch_dequant(tiny.k_cache.numpy(), tiny.k_scale.numpy())      # [L, D]
    dots = np.einsum("thd,sd->tsh", q, k)
    ref = np.einsum("tsh,th->ts", np.maximum(dots, 0.0), tiny.w.numpy().astype(np.float64))
    causal = np.tril(np.ones((L, L), dtype=bool))
    np.testing.assert_allclose(sc[causal], ref[causal], rtol=1e-12, atol=1e-12)
    assert np.all(sc[~causal] == -np.inf)


def test_scores_nonnegative_with_nonnegative_weights(tiny):
    rows = np.arange(0, tiny.L, 7)
    sc = oracle.index_scores(tiny.q_I, tiny.q_scale, tiny.w, tiny.k_cache, tiny.k_scale, rows)
    assert np.all(tiny.w.numpy() >= 0)
    for r, t in enumerate(rows):
        assert np.all(sc[r, :t + 1] >= 0.0)


def test_topk_matches_numpy_lexsort(tiny):
    rows = np.arange(tiny.L)
    sc = oracle.index_scores(tiny.q_I, tiny.q_scale, tiny.w, tiny.k_cache, tiny.k_scale, rows)
    ix = oracle.topk(sc, rows, tiny.topk)
    for r, t in enumerate(rows):
        s = np.arange(t + 1)
        order = np.lexsort((s, -sc[r, :t + 1]))[:tiny.topk]
        n = min(tiny.topk, t + 1)
        assert np.array_equal(ix[r, :n], order[:n])
        assert np.all(ix[r, n:] == -1)


def test_topk_all_equal_keys_breaks_ties_by_lower_index():
    L, H, D, k = 300, 8, 64, 64
    inp = workloads.make_prefill(L, H, D, 16, k, seed=3)
    k8 = np.tile(inp.k_cache[:1].numpy(), (L, 1))
    ks = np.full((L,), float(inp.k_scale[0]), np.float32)
    rows = np.array([0, 10, 63, 64, 299])
    sc = oracle.index_scores(inp.q_I, inp.q_scale, inp.w, k8, ks, rows)
    ix = oracle.topk(sc, rows, k)
    for r, t in enumerate(rows):
        n = min(k, t + 1)
        assert ix[r, :n].tolist() == list(range(n))
        assert np.all(ix[r, n:] == -1)


def test_doubling_key_scales_doubles_scores_and_keeps_selection(tiny):
    rows = np.arange(0, tiny.L, 5)
    a = oracle.index_scores(tiny.q_I, tiny.q_scale, tiny.w, tiny.k_cache, tiny.k_scale, rows)
    b = oracle.index_scores(tiny.q_I, tiny.q_scale, tiny.w, tiny.k_cache, tiny.k_scale * 2, rows)
    fin = np.isfinite(a)
    assert np.array_equal(b[fin], 2.0 * a[fin])
    assert np.array_equal(oracle.topk(a, rows, tiny.topk), oracle.topk(b, rows, tiny.topk))


def test_relu_is_applied_per_head_before_the_weighted_sum():
    # One key, two heads with dots +1 and -1: ReLU per head gives w0, summing
    # first would give w0 - w1. Codes: 0x38 = 1.0, 0xB8 = -1.0.
    q8 = np.array([[[0x38], [0xB8]]], dtype=np.uint8)
    k8 = np.array([[0x38]], dtype=np.uint8)
    sc = oracle.index_scores(q8, np.ones(1, np.float32), np.array([[0.25, 0.5]], np.float32),
                             k8, np.ones(1, np.float32), [0])
    assert sc[0, 0] == 0.25


def test_causality_and_padding(tiny):
    rows = np.arange(tiny.L)
    sc = oracle.index_scores(tiny.q_I, tiny.q_scale, tiny.w, tiny.k_cache, tiny.k_scale, rows)
    ix = oracle.topk(sc, rows, tiny.topk)
    for r, t in enumerate(rows):
        n = min(tiny.topk, t + 1)
        valid = ix[r, :n]
        assert np.all((valid >= 0) & (valid <= t))
        assert len(set(valid.tolist())) == n
        assert np.all(ix[r, n:] == -1)


# --- attention ------------------------------------------------------------

def _dense_causal_mqa(q_bf16, kv_bf16, scale, Dv=512):
    """torch float64 scaled_dot_product_attention, is_causal, K/V shared by all heads."""
    q = q_bf16.to(torch.float64).permute(1, 0, 2)[None]          # [1, Hq, L, 576]
    Hq = q.shape[1]
    kv = kv_bf16.to(torch.float64)
    k = kv[None, None].expand(1, Hq, -1, -1)
    v = kv[None, None, :, :Dv].expand(1, Hq, -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale)
    return o[0].permute(1, 0, 2).numpy()                         # [L, Hq, Dv]


def test_sparse_equals_dense_when_topk_covers_every_candidate():
    L, k = 96, 128                      # k >= t+1 for every row
    inp = workloads.make_prefill(L, 8, 64, 16, k, seed=5)
    rows = np.arange(L)
    _, ix, out, _ = oracle.prefill_rows(inp, rows)
    ref = _dense_causal_mqa(inp.q, inp.kv, inp.scale)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_sparse_equals_dense_on_tiny_rows_below_topk(tiny):
    rows = np.arange(tiny.topk)         # t < 64 = topk
    _, _, out, _ = oracle.prefill_rows(tiny, rows)
    ref = _dense_causal_mqa(tiny.q[:tiny.topk], tiny.kv[:tiny.topk], tiny.scale)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_softmax_special_cases(tiny):
    # t = 0 selects only row 0: the output is that row's value part, exactly
    _, ix, out, _ = oracle.prefill_rows(tiny, [0])
    assert ix[0, 0] == 0 and np.all(ix[0, 1:] == -1)
    v0 = oracle.bf16_to_f64(tiny.kv[0, :512])
    assert np.array_equal(out[0, 0], v0)
    # Q = 0: uniform weights, the output is the mean of the selected value rows
    sel = np.array([[5, 17, 300, 2, -1, 511]], np.int32)
    qz = torch.zeros((1, tiny.Hq, 576), dtype=torch.bfloat16)
    o, lse = oracle.sparse_mla(qz, tiny.kv, sel, tiny.scale)
    vals = oracle.bf16_to_f64(tiny.kv[[5, 17, 300, 2, 511], :512])
    np.testing.assert_allclose(o[0, 3], vals.mean(0), rtol=1e-13, atol=1e-15)
    assert lse[0, 0] == pytest.approx(math.log(5.0), rel=1e-15)
    # permuting the selection leaves the output unchanged
    q1 = tiny.q[100:101]
    a, _ = oracle.sparse_mla(q1, tiny.kv, np.array([[1, 50, 99, 7]], np.int32), tiny.scale)
    b, _ = oracle.sparse_mla(q1, tiny.kv, np.array([[99, 7, 1, 50]], np.int32), tiny.scale)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-16)


def test_planted_keys_are_over_selected():
    inp = workloads.make_prefill(2048, 64, 128, 16, 256, seed=0, plant_frac=0.05)
    planted = set(inp.planted.tolist())
    assert len(planted) == round(0.05 * 2048)
    rows = np.array([511, 1023, 2047])
    sc = oracle.index_scores(inp.q_I, inp.q_scale, inp.w, inp.k_cache, inp.k_scale, rows)
    ix = oracle.topk(sc, rows, inp.topk)
    frac = np.mean([s in planted for s in ix[ix >= 0].tolist()])
    assert frac > 0.05


def test_decode_matches_last_prefill_row():
    # a decode query is the last row of its sequence: same keys, same scores
    dec = workloads.make_decode(2, 700, 64, 128, 16, 256, seed=1)
    (sc, ix, out, lse), = oracle.decode_seqs(dec, [1])
    b = 1
    q8 = np.zeros((700, 64, 128), np.uint8)
    q8[699] = dec.q_I[b].numpy()
    qs = np.ones(700, np.float32)
    qs[699] = float(dec.q_scale[b])
    w = np.zeros((700, 64), np.float32)
    w[699] = dec.w[b].numpy()
    sc2 = oracle.index_scores(q8, qs, w, dec.k_cache[b], dec.k_scale[b], [699])
    assert np.array_equal(sc, sc2[0])
    assert np.array_equal(ix, oracle.topk(sc2, [699], 256)[0])


# ---------------------------------------------------------------- FP8 encoder

def _finite_codes():
    return [c for c in range(256) if (c & 0x7F) != 0x7F]


def test_e4m3_encoder_round_trips_every_finite_code():
    for c in _finite_codes():
        assert oracle.double_to_e4m3(oracle.e4m3_to_f64(np.array([c], np.uint8))[0]) == c, c


def test_e4m3_encoder_ties_go_to_the_even_code():
    vals = oracle.e4m3_to_f64(np.arange(0x7F, dtype=np.uint8))  # 0 .. 448, increasing
    for c in range(0x7E):
        lo, hi = vals[c], vals[c + 1]
        mid = (lo + hi) / 2
        even = c if c % 2 == 0 else c + 1
        assert oracle.double_to_e4m3(mid) == even, c
        assert oracle.double_to_e4m3(-mid) == even | 0x80, c
        assert oracle.double_to_e4m3(np.nextafter(mid, 0)) == c
        assert oracle.double_to_e4m3(np.nextafter(mid, 1e9)) == c + 1
    assert oracle.double_to_e4m3(1e6) == 0x7E and oracle.double_to_e4m3(-1e6) == 0xFE  # saturation


def test_e4m3_encoder_matches_torch_conversion():
    g = torch.Generator().manual_seed(3)
    x = torch.cat([torch.randn(20000, generator=g) * s for s in (1e-4, 1e-2, 1.0, 30.0, 300.0)])
    x = x.clamp(-448, 448)
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.double_to_e4m3(float(v)) for v in x.tolist()], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_row_quantiser_matches_the_input_recipe():
    g = torch.Generator().manual_seed(4)
    x = torch.randn((64, 128), generator=g) * torch.logspace(-3, 2, 64)[:, None]
    x[5] = 0.0  # an all-zero row takes scale 1
    codes, scale = oracle.quantize_e4m3(x)
    ref_codes, ref_scale = workloads.quantize_e4m3_per_token(x)
    assert np.array_equal(scale, ref_scale.numpy())
    assert np.array_equal(codes, ref_codes.numpy())


# --- rotary position encoding of appended tokens ---------------------------

def _rope_inputs(n=5, H=3, d=128, seed=3):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((n, H, d)), rng.integers(0, 131072, size=n)


def test_rope_position_zero_is_the_identity():
    x, _ = _rope_inputs()
    assert np.array_equal(oracle.rope(x, np.zeros(len(x), dtype=np.int64)), x)


def test_rope_first_pair_turns_by_the_position_in_radians():
    # theta_0 = base^0 = 1: the unit vector (1, 0) at position p becomes (cos p, sin p)
    x = np.zeros((4, 128))
    x[:, 0] = 1.0
    pos = np.array([1, 2, 7, 100000])
    r = oracle.rope(x, pos)
    assert np.allclose(r[:, 0], [math.cos(p) for p in pos], rtol=0, atol=1e-12)
    assert np.allclose(r[:, 1], [math.sin(p) for p in pos], rtol=0, atol=1e-12)  # counter-clockwise


def test_rope_equals_complex_multiplication():
    # each pair as the complex number a + ib, multiplied by exp(i * p * theta_i)
    x, pos = _rope_inputs()
    r = oracle.rope(x, pos)
    z = x[..., 0:64:2] + 1j * x[..., 1:64:2]
    rz = r[..., 0:64:2] + 1j * r[..., 1:64:2]
    # the frequencies, recovered from a rotation at position 1 of the vector (1, 0)
    e = np.zeros((1, 128))
    e[0, 0:64:2] = 1.0
    r1 = oracle.rope(e, [1])[0]
    theta = np.arctan2(r1[1:64:2], r1[0:64:2])
    want = z * np.exp(1j * pos[:, None, None] * theta[None, None, :])
    assert np.abs(rz - want).max() < 1e-9
    assert np.array_equal(r[..., 64:], x[..., 64:])  # the rest of each head is untouched


def test_rope_frequencies_fall_geometrically_from_one_to_nearly_one_over_base():
    e = np.zeros((1, 64))
    e[0, 0::2] = 1.0
    r1 = oracle.rope(e, [1], rope_dim=64, base=10000.0)[0]
    theta = np.arctan2(r1[1::2], r1[0::2])
    assert theta[0] == pytest.approx(1.0, abs=1e-15)
    ratios = theta[1:] / theta[:-1]
    assert np.allclose(ratios, 10000.0 ** (-1 / 32), rtol=1e-12)  # 32 pairs span base^(-31/32)
    assert theta[-1] == pytest.approx(10000.0 ** (-31 / 32), rel=1e-12)


def test_rope_scores_depend_on_the_relative_position_only():
    rng = np.random.default_rng(5)
    q, k = rng.standard_normal((1, 128)), rng.standard_normal((1, 128))
    for m, n in [(5, 2), (1000, 10), (70000, 69999)]:
        base_dot = float(oracle.rope(q, [m])[0] @ oracle.rope(k, [n])[0])
        for c in (1, 333, 40000):
            shifted = float(oracle.rope(q, [m + c])[0] @ oracle.rope(k, [n + c])[0])
            assert shifted == pytest.approx(base_dot, rel=1e-9, abs=1e-9)


def test_rope_rotations_compose_and_keep_pair_norms():
    x, _ = _rope_inputs(n=3)
    a, b = np.array([3, 500, 60000]), np.array([4, 12345, 7])
    twice = oracle.rope(oracle.rope(x, a), b)
    once = oracle.rope(x, a + b)
    assert np.abs(twice - once).max() < 1e-9
    norms = x[..., 0:64:2] ** 2 + x[..., 1:64:2] ** 2
    rn = once[..., 0:64:2] ** 2 + once[..., 1:64:2] ** 2
    assert np.allclose(rn, norms, rtol=1e-12)


def test_rope_pair_layouts_are_one_permutation_apart():
    # split-half pairs (i, i+32) are consecutive pairs after moving dim i to 2i and i+32 to 2i+1
    x, pos = _rope_inputs()
    perm = np.arange(128)
    perm[0:64:2], perm[1:64:2] = np.arange(32), np.arange(32, 64)
    inter = oracle.rope(x[..., perm], pos, interleaved=True)
    half = oracle.rope(x, pos, interleaved=False)
    assert np.abs(inter - half[..., perm]).max() < 1e-12


def test_rope_quantiser_at_position_zero_is_the_plain_quantiser():
    x, _ = _rope_inputs(n=4, H=2)
    x32 = x.astype(np.float32)
    codes, scale = oracle.rope_quantize_e4m3(x32, np.zeros(4, dtype=np.int64))
    c0, s0 = oracle.quantize_e4m3(x32.reshape(4, -1))
    assert np.array_equal(codes.reshape(4, -1), c0) and np.array_equal(scale, s0)
    # and the codes stay within half a step of the rotated row (torch's decoder)
    pos = np.array([1, 99, 4096, 131071])
    codes, scale = oracle.rope_quantize_e4m3(x32, pos)
    deq = _torch_dequant(codes.reshape(4, -1), scale)
    ref = oracle.rope(x32, pos).reshape(4, -1)
    step = np.where(np.abs(ref) >= 2.0 ** -6 * scale[:, None], np.abs(ref) / 8, 2.0 ** -9 * scale[:, None])
    assert np.all(np.abs(deq - ref) <= 0.5 * step * 1.0001 + 1e-7 * np.abs(ref))
