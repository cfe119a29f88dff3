"""Comparison helpers shared by the GPU parity tests (CPU-side numpy only)."""
import numpy as np
import torch

import oracle


def to_dev(inp, device="cuda"):
    return inp.to(device)


def score_tolerance_ok(gpu, ref, rows):
    """Index scores within 1e-4 relative of the oracle.

    |gpu - ref| <= 1e-4 * max(|ref|, 1e-3 * max_s ref[t, s]) on every causal
    entry, and exact zeros (every head ReLU'd away) must be exactly zero.
    Returns (ok, worst ratio of error to allowance).
    """
    worst = 0.0
    ok = True
    for r, t in enumerate(rows):
        g = gpu[r, :t + 1].astype(np.float64)
        f = ref[r, :t + 1]
        floor = 1e-3 * np.max(np.abs(f)) if f.size else 0.0
        allow = 1e-4 * np.maximum(np.abs(f), floor)
        err = np.abs(g - f)
        zero = f == 0.0
        if np.any(g[zero] != 0.0):
            ok = False
        nz = ~zero
        if np.any(nz):
            ratio = float(np.max(err[nz] / allow[nz]))
            worst = max(worst, ratio)
            if ratio > 1.0:
                ok = False
    return ok, worst


def overlap_excluding_ties(idx_gpu, idx_ref, scores_ref, rows, k):
    """Selected-set overlap with the oracle, dropping every s whose oracle score
    equals the oracle's k-th score (exact ties), over rows with t+1 > k."""
    hit = tot = 0
    for r, t in enumerate(rows):
        if t + 1 <= k:
            continue
        ref = idx_ref[r]
        theta = scores_ref[r, ref[k - 1]]
        tie = lambda s: scores_ref[r, s] == theta
        a = {int(s) for s in idx_gpu[r] if s >= 0 and not tie(s)}
        b = {int(s) for s in ref if s >= 0 and not tie(s)}
        hit += len(a & b)
        tot += len(b)
    return (hit / tot) if tot else 1.0


def cpu_topk_of(scores_f32, rows, k):
    """The oracle's ranking rule applied to the GPU's own fp32 scores."""
    return oracle.topk(scores_f32.astype(np.float64), rows, k)


def attn_close(gpu_bf16, ref, max_abs=2e-2, rel=1e-2):
    """Attention within 2e-2 max-abs and 1e-2 relative (L2) of the oracle."""
    g = gpu_bf16.float().cpu().numpy().astype(np.float64) if isinstance(gpu_bf16, torch.Tensor) else gpu_bf16
    d = np.abs(g - ref)
    mx = float(d.max()) if d.size else 0.0
    rl = float(np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-300))
    return (mx <= max_abs and rl <= rel), mx, rl
