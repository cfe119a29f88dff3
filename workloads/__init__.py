"""Seeded synthetic inputs for the DeepSeek Sparse Attention (DSA) hot path.

This module is shared by the tests, the benchmark and the smoke run. It feeds
both the CUDA library and the float64 oracle, so it holds none of the method's
arithmetic: it only draws random numbers in a fixed order and converts them to
the storage formats of the input contract.

Input contract (the indexer's FP8 cache, "Lightning Indexer 的计算过程" step 2
<2> on adg.csdn.net/695234...: act_quant produces FP8 values plus a scale
factor, cached as k_cache / k_scale_cache):

* q_I  [L, H_I, d_I]  e4m3 bytes, one fp32 scale per token (absmax over all
  H_I*d_I values / 448; a token of zeros gets scale 1).
* k_cache [L, d_I]    e4m3 bytes, one fp32 scale per token (absmax over d_I).
* w    [L, H_I]       fp32 per-head indexer weights.
* q    [L, Hq, 576]   bf16 main-attention queries (512 latent + 64 RoPE dims).
* kv   [L, 576]       bf16 MLA latent cache rows, N(0,1)/sqrt(576).

fp32 -> e4m3 is round-to-nearest-even after clamping to +-448 (the largest
finite e4m3 value); fp32 -> bf16 is round-to-nearest-even. Both conversions are
torch's own.

Draw order, from one torch.Generator seeded with `seed` on `device`:
q_I, k_I, w, [planted positions], q, kv. Large tensors are drawn in row
chunks from the same generator, so the stream is fixed for a given device.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

E4M3_MAX = 448.0
D_QK = 576      # latent (512) + RoPE (64) dims of an MLA cache row
D_V = 512       # value dims: the latent part of the same row

_CHUNK_ELEMS = 1 << 26   # draw big tensors 64M elements at a time


def _randn(shape, gen, device, dtype=torch.float32):
    return torch.randn(shape, generator=gen, device=device, dtype=dtype)


def quantize_e4m3_per_token(x: torch.Tensor):
    """x [n, m] fp32 -> (codes uint8 [n, m], scale fp32 [n]).

    scale = absmax/448 per row (1 for an all-zero row); codes = RNE(x/scale)
    saturated to +-448.
    """
    absmax = x.abs().amax(dim=1)
    scale = torch.where(absmax > 0, absmax / E4M3_MAX, torch.ones_like(absmax))
    y = (x / scale[:, None]).clamp_(-E4M3_MAX, E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, scale.to(torch.float32)


def _draw_bf16_rows(rows: int, cols: int, gen, device, div: float = 1.0):
    out = torch.empty((rows, cols), dtype=torch.bfloat16, device=device)
    step = max(1, _CHUNK_ELEMS // cols)
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        x = _randn((r1 - r0, cols), gen, device)
        if div != 1.0:
            x /= div
        out[r0:r1] = x.to(torch.bfloat16)
    return out


def _draw_quantized_rows(rows: int, cols: int, gen, device, plant=None, plant_bias=3.0):
    codes = torch.empty((rows, cols), dtype=torch.uint8, device=device)
    scale = torch.empty((rows,), dtype=torch.float32, device=device)
    step = max(1, _CHUNK_ELEMS // cols)
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        x = _randn((r1 - r0, cols), gen, device)
        if plant is not None:
            sel = plant[(plant >= r0) & (plant < r1)] - r0
            x[sel] += plant_bias
        c, s = quantize_e4m3_per_token(x)
        codes[r0:r1] = c
        scale[r0:r1] = s
    return codes, scale


@dataclass
class PrefillInputs:
    L: int
    H_I: int
    d_I: int
    Hq: int
    topk: int
    scale: float
    q_I: torch.Tensor        # uint8 [L, H_I, d_I]
    q_scale: torch.Tensor    # f32 [L]
    w: torch.Tensor          # f32 [L, H_I]
    k_cache: torch.Tensor    # uint8 [L, d_I]
    k_scale: torch.Tensor    # f32 [L]
    q: torch.Tensor          # bf16 [L, Hq, 576]
    kv: torch.Tensor         # bf16 [L, 576]
    planted: Optional[torch.Tensor] = None   # int64 positions with the +3 bias

    def to(self, device):
        kw = {}
        for f in ("q_I", "q_scale", "w", "k_cache", "k_scale", "q", "kv", "planted"):
            v = getattr(self, f)
            kw[f] = None if v is None else v.to(device)
        return PrefillInputs(self.L, self.H_I, self.d_I, self.Hq, self.topk, self.scale, **kw)


@dataclass
class DecodeInputs:
    B: int
    L: int                   # tokens cached per sequence (the new token included)
    H_I: int
    d_I: int
    Hq: int
    topk: int
    scale: float
    q_I: torch.Tensor        # uint8 [B, H_I, d_I]
    q_scale: torch.Tensor    # f32 [B]
    w: torch.Tensor          # f32 [B, H_I]
    k_cache: torch.Tensor    # uint8 [B, L, d_I]
    k_scale: torch.Tensor    # f32 [B, L]
    q: torch.Tensor          # bf16 [B, Hq, 576]
    kv: torch.Tensor         # bf16 [B, L, 576]
    lens: torch.Tensor       # int32 [B]

    def to(self, device):
        kw = {f: getattr(self, f).to(device) for f in
              ("q_I", "q_scale", "w", "k_cache", "k_scale", "q", "kv", "lens")}
        return DecodeInputs(self.B, self.L, self.H_I, self.d_I, self.Hq, self.topk, self.scale, **kw)


def make_prefill(L: int, H_I: int, d_I: int, Hq: int, topk: int, *, seed: int = 0,
                 plant_frac: float = 0.0, signed_w: bool = False,
                 device="cpu") -> PrefillInputs:
    """One causal prefill sequence of length L.

    q_I, k_I ~ N(0,1) quantised per token; w ~ U(0,1)/H_I (U(-1,1)/H_I when
    signed_w); q ~ N(0,1) bf16; kv ~ N(0,1)/sqrt(576) bf16. With plant_frac > 0,
    round(plant_frac*L) distinct positions drawn without replacement get +3.0 on
    every indexer-key dim before quantisation.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    qi_codes, q_scale = _draw_quantized_rows(L, H_I * d_I, gen, device)
    # k_I is drawn before the plant positions so the stream order stays
    # q_I, k_I, w, plant; the bias is added after the draw, before quantising.
    k_raw = _randn((L, d_I), gen, device)
    if signed_w:
        w = (torch.rand((L, H_I), generator=gen, device=device) * 2.0 - 1.0) / H_I
    else:
        w = torch.rand((L, H_I), generator=gen, device=device) / H_I
    planted = None
    if plant_frac > 0:
        n = int(round(plant_frac * L))
        planted = torch.randperm(L, generator=gen, device=device)[:n].sort().values
        k_raw[planted] += 3.0
    k_codes, k_scale = quantize_e4m3_per_token(k_raw)
    del k_raw
    q = _draw_bf16_rows(L * Hq, D_QK, gen, device).view(L, Hq, D_QK)
    kv = _draw_bf16_rows(L, D_QK, gen, device, div=math.sqrt(D_QK))
    return PrefillInputs(L, H_I, d_I, Hq, topk, 1.0 / math.sqrt(D_QK),
                         qi_codes.view(L, H_I, d_I), q_scale, w.float().contiguous(),
                         k_codes, k_scale, q, kv, planted)


def make_decode(B: int, L: int, H_I: int, d_I: int, Hq: int, topk: int, *, seed: int = 0,
                device="cpu", lens=None) -> DecodeInputs:
    """B sequences of L cached tokens each, one new query per sequence.

    The cache already holds the new token's key and latent row, so the query
    sits at position lens[b]-1 (lens defaults to L for every sequence).
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    qi_codes, q_scale = _draw_quantized_rows(B, H_I * d_I, gen, device)
    k_codes, k_scale = _draw_quantized_rows(B * L, d_I, gen, device)
    w = torch.rand((B, H_I), generator=gen, device=device) / H_I
    q = _draw_bf16_rows(B * Hq, D_QK, gen, device).view(B, Hq, D_QK)
    kv = _draw_bf16_rows(B * L, D_QK, gen, device, div=math.sqrt(D_QK)).view(B, L, D_QK)
    if lens is None:
        lens_t = torch.full((B,), L, dtype=torch.int32, device=device)
    else:
        lens_t = torch.as_tensor(lens, dtype=torch.int32, device=device)
    return DecodeInputs(B, L, H_I, d_I, Hq, topk, 1.0 / math.sqrt(D_QK),
                        qi_codes.view(B, H_I, d_I), q_scale, w.float().contiguous(),
                        k_codes.view(B, L, d_I), k_scale.view(B, L), q, kv, lens_t)


# The five workloads of the method's shapes (k = 2048 selected tokens, 64
# indexer heads of dim 128, 128 query heads over 576-d latent rows).
CONFIGS = {
    "tiny_L512": dict(kind="prefill", L=512, H_I=8, d_I=64, Hq=16, topk=64),
    "prefill_L8192": dict(kind="prefill", L=8192, H_I=64, d_I=128, Hq=128, topk=2048),
    "prefill_L32768_planted": dict(kind="prefill", L=32768, H_I=64, d_I=128, Hq=128, topk=2048,
                                   plant_frac=0.05),
    "prefill_L131072": dict(kind="prefill", L=131072, H_I=64, d_I=128, Hq=128, topk=2048),
    "decode_B64_L65536": dict(kind="decode", B=64, L=65536, H_I=64, d_I=128, Hq=128, topk=2048),
}


def make_config(name: str, *, seed: int = 0, device="cpu"):
    c = dict(CONFIGS[name])
    kind = c.pop("kind")
    if kind == "prefill":
        return make_prefill(seed=seed, device=device, **c)
    return make_decode(seed=seed, device=device, **c)
