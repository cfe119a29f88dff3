"""Run one hot-path call repeatedly on seeded synthetic inputs, for profiling a
single kernel (e.g. under ncu with -k and -s/-c) without the rest of the
benchmark's allocations.

    python -m long_context_03_b200.run_kernel indexer --L 65536
    python -m long_context_03_b200.run_kernel attention --L 16384
    python -m long_context_03_b200.run_kernel decode --B 64 --L 65536
    python -m long_context_03_b200.run_kernel decode_paged --B 64 --L 65536 --page 64
    python -m long_context_03_b200.run_kernel rope --B 64        # RoPE + E4M3 of B appended query rows

Prints the mean CUDA-event time of the calls after the warm-up ones. Inputs come from the seeded
generators of the benchmark (`workloads`); the indexer case uses a single
query head for the attention inputs, which the indexer never reads.
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if _ROOT not in sys.path:
    sys.path.insert(0, _ROOT)

import long_context_03_b200 as dsa  # noqa: E402
import workloads  # noqa: E402


def _time(fn, repeat):
    """Mean CUDA-event time of the calls after the first min(3, repeat - 1)."""
    warm = min(3, repeat - 1)
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(repeat - warm):
        fn()
    e1.record()
    torch.cuda.synchronize()
    dsa.check_device_error()
    return e0.elapsed_time(e1) / (repeat - warm)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("op", choices=["indexer", "attention", "decode", "decode_paged", "rope"])
    ap.add_argument("--L", type=int, default=65536)
    ap.add_argument("--B", type=int, default=64)
    ap.add_argument("--topk", type=int, default=2048)
    ap.add_argument("--repeat", type=int, default=3)
    ap.add_argument("--page", type=int, default=64)
    a = ap.parse_args(argv)
    dev = torch.device("cuda", 0)
    if a.op == "indexer":
        P = workloads.make_prefill(a.L, 64, 128, 1, a.topk, seed=0, device=dev)
        ws = torch.empty(dsa.index_topk_workspace_size(a.L, 64, 128, a.topk), dtype=torch.uint8, device=dev)
        idx = torch.empty((a.L, a.topk), dtype=torch.int32, device=dev)
        ms = _time(lambda: dsa.index_topk(P.q_I, P.q_scale, P.w, P.k_cache, P.k_scale, a.topk, idx=idx,
                                          workspace=ws), a.repeat)
    elif a.op == "attention":
        P = workloads.make_prefill(a.L, 64, 128, 128, a.topk, seed=0, device=dev)
        idx = dsa.index_topk(P.q_I, P.q_scale, P.w, P.k_cache, P.k_scale, a.topk)
        out = torch.empty((a.L, 128, 512), dtype=torch.bfloat16, device=dev)
        ms = _time(lambda: dsa.sparse_mla_attn(P.q, P.kv, idx, P.scale, out=out), a.repeat)
    elif a.op == "rope":
        # B appended tokens: indexer queries [B, 64, 128] and keys [B, 128], rotated and quantised
        g = torch.Generator(device=dev).manual_seed(0)
        xq = torch.randn((a.B, 64, 128), generator=g, device=dev)
        xk = torch.randn((a.B, 128), generator=g, device=dev)
        pos = torch.randint(0, a.L, (a.B,), generator=g, device=dev, dtype=torch.int32)

        def step():
            dsa.rope_quantize_e4m3_rows(xq, pos)
            dsa.rope_quantize_e4m3_rows(xk, pos)

        ms = _time(step, a.repeat)
    elif a.op == "decode_paged":
        # both caches in one shuffled pool of pages (every sequence full length)
        D = workloads.make_decode(a.B, a.L, 64, 128, 128, a.topk, seed=0, device=dev)
        npg = a.L // a.page
        perm = torch.randperm(a.B * npg, device=dev)
        k_pool = torch.empty((a.B * a.L, 128), dtype=torch.uint8, device=dev)
        k_pool.view(-1, a.page, 128)[perm] = D.k_cache.view(torch.uint8).reshape(-1, a.page, 128)
        ks_pool = torch.empty((a.B * a.L,), dtype=torch.float32, device=dev)
        ks_pool.view(-1, a.page)[perm] = D.k_scale.reshape(-1, a.page)
        kv_pool = torch.empty((a.B * a.L, 576), dtype=torch.bfloat16, device=dev)
        kv_pool.view(-1, a.page, 576)[perm] = D.kv.reshape(-1, a.page, 576)
        table = perm.to(torch.int32).view(a.B, npg)
        ws = torch.empty(dsa.index_topk_decode_workspace_size(a.B, a.L, a.topk), dtype=torch.uint8, device=dev)
        idx = torch.empty((a.B, a.topk), dtype=torch.int32, device=dev)
        out = torch.empty((a.B, 128, 512), dtype=torch.bfloat16, device=dev)

        def step():
            dsa.index_topk_decode_paged(D.q_I, D.q_scale, D.w, k_pool, ks_pool, table, D.lens, a.topk,
                                        page_size=a.page, idx=idx, workspace=ws)
            dsa.sparse_mla_attn_paged(D.q, kv_pool, table, idx, a.L, D.scale, page_size=a.page, out=out)

        ms = _time(step, a.repeat)
    else:
        D = workloads.make_decode(a.B, a.L, 64, 128, 128, a.topk, seed=0, device=dev)
        ws = torch.empty(dsa.index_topk_decode_workspace_size(a.B, a.L, a.topk), dtype=torch.uint8, device=dev)
        idx = torch.empty((a.B, a.topk), dtype=torch.int32, device=dev)
        out = torch.empty((a.B, 128, 512), dtype=torch.bfloat16, device=dev)

        def step():
            dsa.index_topk_decode(D.q_I, D.q_scale, D.w, D.k_cache, D.k_scale, D.lens, a.topk, idx=idx, workspace=ws)
            dsa.sparse_mla_attn_decode(D.q, D.kv, idx, D.scale, out=out)

        ms = _time(step, a.repeat)
    print(f"{a.op} L={a.L} B={a.B} topk={a.topk}: {ms:.3f} ms (mean of the last {a.repeat - min(3, a.repeat - 1)}"
          f" of {a.repeat} calls)")


if __name__ == "__main__":
    main()
