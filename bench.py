"""Benchmark of the DSA hot path on B200: prefill tokens/s at L = 131072 and
decode tokens/s for 64 sequences x 65536 cached tokens.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the whole hot path over one batch of synthetic input:
a 131072-token causal prefill (indexer + top-2048 selection + sparse MQA over
the latent cache) and one decode batch (64 queries, each against its own
65536-token caches). Inputs are seeded, generated on the device and resident
in HBM before timing; they are far larger than L2 (the queries alone are
19 GB), so no flush is needed between steps. `value` is prefill tokens/s
summed over ranks; decode tokens/s is reported beside it.

With N > 1 (torchrun), every rank runs the same workload independently on
its own GPU (replicas: the path has no exchange step); times are the max over
ranks and `value` counts every rank's tokens.

--impl reference times the float64 CPU oracle (the checker, not a competing
system) on a bounded sample of the same workload on this host's cores.

--kernel OP runs one hot-path call repeatedly on seeded inputs instead (for
timing or profiling a single kernel, e.g. under ncu with -k and -s/-c) and
prints its mean CUDA-event time as one JSON line:

    python bench.py --kernel indexer --prefill-L 65536 --repeat 5
    python bench.py --kernel attention --prefill-L 16384
    python bench.py --kernel attention_chunk --chunk-T 2048   # last 2048 rows of the 128K prefill
    python bench.py --kernel decode --decode-B 64 --decode-L 65536
    python bench.py --kernel decode_paged --decode-B 64 --decode-L 65536 --page 64
    python bench.py --kernel rope --decode-B 64      # RoPE + E4M3 of B appended indexer rows
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "DSA prefill tokens/s @128K & decode tok/s, % of FP8/BF16/HBM roofline"

# DRAM bytes (read + write) per timed unit of the default workload, from one
# single-pass ncu capture (dram__bytes_read.sum + dram__bytes_write.sum) of
# this benchmark on B200. Valid only for the kernels they were taken on: an
# entry is None until the current kernels are captured. Units: the prefill
# indexer entry covers its main and re-run passes; decode entries cover one
# decode batch.
MEASURED_TRAFFIC = {
    "prefill_indexer": 1.2733e9 + 3.0800e9 + 0.0001e9,  # main pass + re-run pass
    "prefill_attention": None,  # measured on a 2048-row chunk only; does not scale with the token count
    "decode_step": 0.5542e9 + 0.0027e9 + 0.0174e9 + 0.1611e9 + 0.0002e9,
    "decode_indexer": 0.5542e9 + 0.0027e9 + 0.0174e9,
}
DEFAULT_SIZES = (131072, 64, 65536)  # prefill L, decode B, decode L the traffic was measured on
D_QK, D_V = 576, 512


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--prefill-L", type=int, default=131072)
    ap.add_argument("--decode-B", type=int, default=64)
    ap.add_argument("--decode-L", type=int, default=65536)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-chunks", type=int, default=8,
                    help="query-row chunks whose copies overlap the compute in the e2e leg (1: no overlap)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-rows", type=int, default=240)
    ap.add_argument("--kernel", default=None,
                    choices=["indexer", "attention", "attention_chunk", "decode", "decode_paged", "rope"],
                    help="time one hot-path call instead of the whole step (see the module docstring)")
    ap.add_argument("--repeat", type=int, default=5, help="calls in --kernel mode (the first min(3, repeat-1) warm up)")
    ap.add_argument("--page", type=int, default=64, help="page size of --kernel decode_paged")
    ap.add_argument("--chunk-T", type=int, default=2048,
                    help="--kernel attention_chunk: the last T query rows of the prefill attend over its whole cache")
    ap.add_argument("--no-fp8-probe", action="store_true",
                    help="skip the library FP8 GEMM measured after the timed work (context for the indexer's peak)")
    return ap.parse_args(argv)


# ----------------------------------------------------------------- helpers

def measure_fp8_gemm(dev, seconds=3.0, n=8192):
    """Context for the indexer's roofline: a library FP8 GEMM (torch._scaled_mm,
    e4m3 8192^3, bf16 out) as a burst (best of 10) and back to back for
    `seconds`. Runs after every timed region; the reported peak stays twice the
    measured bf16 figure. Any failure is reported, never raised."""
    try:
        g = torch.Generator(device=dev).manual_seed(0)
        a = torch.randn((n, n), generator=g, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn((n, n), generator=g, device=dev).to(torch.float8_e4m3fn).t()  # column-major operand
        one = torch.ones((), dtype=torch.float32, device=dev)

        def mm():
            return torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)

        for _ in range(3):
            mm()
        torch.cuda.synchronize()
        flop = 2.0 * n ** 3
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            mm()
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        calls = 0
        e0.record()
        t_end = time.perf_counter() + seconds
        while time.perf_counter() < t_end:
            for _ in range(20):
                mm()
            calls += 20
            torch.cuda.synchronize()
        e1.record()
        torch.cuda.synchronize()
        sustained = flop * calls / (e0.elapsed_time(e1) * 1e-3) / 1e12
        return {"burst_tflops": flop / (best * 1e-3) / 1e12, "sustained_tflops": sustained,
                "method": f"torch._scaled_mm e4m3 {n}^3, bf16 out: best of 10, then {calls} calls back to back"}
    except Exception as e:  # informational only
        return {"error": f"{type(e).__name__}: {e}"[:300]}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        m = json.load(open(p))
        return {"hbm_gbs": m["hbm_gbs"], "bf16_tflops": m["bf16_tflops"],
                "bf16_tflops_sustained": m["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def prefill_work(L, H_I, d_I, Hq, topk):
    """Algorithmic work of one prefill pass (causal pairs only)."""
    pairs = L * (L + 1) // 2
    idx_flop = 2.0 * H_I * d_I * pairs
    sel = sum(min(topk, t + 1) for t in range(min(L, topk))) + max(0, L - topk) * topk
    attn_flop = sel * Hq * 2.0 * (D_QK + D_V)
    return idx_flop, attn_flop


def decode_bytes(B, L, H_I, d_I, Hq, topk):
    """Compulsory HBM bytes of one decode step."""
    keys = B * L * (d_I + 4)
    gather = B * min(topk, L) * D_QK * 2
    small = B * (H_I * d_I + 4 + H_I * 4 + Hq * D_QK * 2 + Hq * D_V * 2 + topk * 4)
    return keys, gather, small


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(5)
        except Exception:
            self.p.kill()
        self.f.flush()
        rows = []
        for line in open(self.f.name):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.f.name)
        if not rows:
            return None
        sm = [r[0] for r in rows]
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[2]) if v.lower() == "active"})
        return {"sm_mhz": float(np.median(loaded)), "sm_max_mhz": rows[0][1], "reasons": reasons,
                "samples": len(rows)}


def dist_setup(gpus):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


def max_over_ranks(x, ws):
    if ws == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_totals(seg_ms, ws, L, B):
    """Whole-job rates of N independent replicas.

    seg_ms = this rank's mean step time (ms) of the four launches in step
    order (prefill indexer, prefill attention, decode indexer, decode
    attention). Each is replaced by its max over ranks, so the job is as
    fast as its slowest GPU; every rank processes L prefill tokens and B
    decode tokens per step. Returns (segment maxima, prefill tokens/s,
    decode tokens/s), all ranks' tokens counted.
    """
    t = [max_over_ranks(float(x), ws) for x in seg_ms]
    t_prefill, t_decode = t[0] + t[1], t[2] + t[3]
    return t, ws * L / (t_prefill * 1e-3), ws * B / (t_decode * 1e-3)


# ---------------------------------------------------------- CPU baseline

def cpu_oracle_prefill(inp_dev, n_rows, seed=1):
    """Oracle on a uniform sample of query rows of the prefill workload.

    Returns (tokens/s estimate for the whole prefill, seconds, rows, threads).
    The per-row cost grows with t, so rows are drawn uniformly over [0, L).
    """
    import oracle
    L = inp_dev.L
    n_rows = max(n_rows, oracle.num_threads())
    g = np.random.default_rng(seed)
    rows = np.sort(g.choice(L, size=n_rows, replace=False))
    host = dict(q_I=inp_dev.q_I[rows].cpu(), q_scale=inp_dev.q_scale[rows].cpu(), w=inp_dev.w[rows].cpu(),
                k_cache=inp_dev.k_cache.cpu(), k_scale=inp_dev.k_scale.cpu(), q=inp_dev.q[rows].cpu(),
                kv=inp_dev.kv.cpu())
    t0 = time.perf_counter()
    sc = oracle.index_scores(host["q_I"], host["q_scale"], host["w"], host["k_cache"], host["k_scale"], rows,
                             query_rows=np.arange(n_rows))
    ix = oracle.topk(sc, rows, inp_dev.topk)
    oracle.sparse_mla(host["q"], host["kv"], ix, inp_dev.scale)
    dt = time.perf_counter() - t0
    return n_rows / dt, dt, rows, min(n_rows, oracle.num_threads())


def cpu_oracle_decode(dec_dev, n_seq):
    import oracle
    sub = workloads.DecodeInputs(n_seq, dec_dev.L, dec_dev.H_I, dec_dev.d_I, dec_dev.Hq, dec_dev.topk, dec_dev.scale,
                                 dec_dev.q_I[:n_seq].cpu(), dec_dev.q_scale[:n_seq].cpu(), dec_dev.w[:n_seq].cpu(),
                                 dec_dev.k_cache[:n_seq].cpu(), dec_dev.k_scale[:n_seq].cpu(),
                                 dec_dev.q[:n_seq].cpu(), dec_dev.kv[:n_seq].cpu(), dec_dev.lens[:n_seq].cpu())
    t0 = time.perf_counter()
    oracle.decode_seqs(sub, range(n_seq))
    dt = time.perf_counter() - t0
    return n_seq / dt, dt


# -------------------------------------------------------------- our path

def workload_config(a, ws):
    """The `config` both arms report: the benchmark workload, named by its sizes."""
    cP = workloads.CONFIGS["prefill_L131072"]
    cD = workloads.CONFIGS["decode_B64_L65536"]
    return {"workload": f"prefill L={a.prefill_L} (H_I={cP['H_I']}, d_I={cP['d_I']}, topk={cP['topk']}, "
                        f"Hq={cP['Hq']}) + decode B={a.decode_B} x L={a.decode_L}",
            "parallelism": "replicas" if ws > 1 else "single",
            "l2": "inputs larger than L2 (no flush needed)", "seed": "rank"}


def run_ours(a, ws, rank):
    import long_context_03_b200 as dsa
    dev = torch.device("cuda", torch.cuda.current_device())
    cfgP = dict(workloads.CONFIGS["prefill_L131072"])
    cfgP["L"] = a.prefill_L
    cfgD = dict(workloads.CONFIGS["decode_B64_L65536"])
    cfgD["B"], cfgD["L"] = a.decode_B, a.decode_L
    P = workloads.make_prefill(cfgP["L"], cfgP["H_I"], cfgP["d_I"], cfgP["Hq"], cfgP["topk"], seed=rank,
                               device=dev)
    D = workloads.make_decode(cfgD["B"], cfgD["L"], cfgD["H_I"], cfgD["d_I"], cfgD["Hq"], cfgD["topk"], seed=rank,
                              device=dev)
    L, k = P.L, P.topk
    idx = torch.empty((L, k), dtype=torch.int32, device=dev)
    out = torch.empty((L, P.Hq, D_V), dtype=torch.bfloat16, device=dev)
    ws_p = torch.empty(dsa.index_topk_workspace_size(L, P.H_I, P.d_I, k), dtype=torch.uint8, device=dev)
    didx = torch.empty((D.B, k), dtype=torch.int32, device=dev)
    dout = torch.empty((D.B, D.Hq, D_V), dtype=torch.bfloat16, device=dev)
    ws_d = torch.empty(dsa.index_topk_decode_workspace_size(D.B, D.L, k), dtype=torch.uint8, device=dev)
    ws_a = torch.empty(dsa.split_workspace_size(D.B, k), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        dsa.index_topk(P.q_I, P.q_scale, P.w, P.k_cache, P.k_scale, k, idx=idx, workspace=ws_p)
        if ev:
            ev[1].record(stream)
        dsa.sparse_mla_attn(P.q, P.kv, idx, P.scale, out=out)
        if ev:
            ev[2].record(stream)
        dsa.index_topk_decode(D.q_I, D.q_scale, D.w, D.k_cache, D.k_scale, D.lens, k, idx=didx, workspace=ws_d)
        if ev:
            ev[3].record(stream)
        dsa.sparse_mla_attn_decode(D.q, D.kv, didx, D.scale, out=dout, workspace=ws_a)
        if ev:
            ev[4].record(stream)

    for _ in range(a.warmup):
        step()
    torch.cuda.synchronize()
    dsa.check_device_error()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(a.steps)]
    clk = ClockSampler(dev.index)
    barrier(ws)
    torch.cuda.synchronize()
    clk.start()
    t_wall = time.perf_counter()
    for s in range(a.steps):
        step(evs[s])
    torch.cuda.synchronize()
    barrier(ws)
    t_wall = time.perf_counter() - t_wall
    clocks = clk.stop()
    dsa.check_device_error()
    seg = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(4)] for e in evs])  # ms
    (t_idx, t_attn, t_didx, t_dattn), value, dec_tps = replica_totals(seg.mean(axis=0), ws, L, D.B)
    t_prefill = t_idx + t_attn
    t_decode = t_didx + t_dattn

    pk = peaks()
    fp8_peak = 2.0 * pk["bf16_tflops_sustained"]
    idx_flop, attn_flop = prefill_work(L, P.H_I, P.d_I, P.Hq, k)
    keys_b, gather_b, small_b = decode_bytes(D.B, D.L, D.H_I, D.d_I, D.Hq, k)
    idx_tf = idx_flop / (t_idx * 1e-3) / 1e12
    attn_tf = attn_flop / (t_attn * 1e-3) / 1e12
    dec_gbs = (keys_b + gather_b + small_b) / (t_decode * 1e-3) / 1e9
    dec_idx_gbs = (keys_b + D.B * (D.H_I * D.d_I + 8 + D.H_I * 4)) / (t_didx * 1e-3) / 1e9
    rl = {
        "prefill_indexer": {"bound": "tensor", "achieved": idx_tf, "peak": fp8_peak, "unit": "TFLOP/s",
                            "frac": idx_tf / fp8_peak, "traffic": None,
                            "note": "FP8 peak = 2 x measured sustained bf16 (nominal fp8:bf16 ratio); time includes the in-kernel ranking"},
        "prefill_attention": {"bound": "tensor", "achieved": attn_tf, "peak": pk["bf16_tflops_sustained"],
                              "unit": "TFLOP/s", "frac": attn_tf / pk["bf16_tflops_sustained"], "traffic": None},
        "decode_step": {"bound": "hbm", "achieved": dec_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                        "frac": dec_gbs / pk["hbm_gbs"], "traffic": None},
        "decode_indexer": {"bound": "hbm", "achieved": dec_idx_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                           "frac": dec_idx_gbs / pk["hbm_gbs"], "traffic": None},
    }
    if (L, D.B, D.L) == DEFAULT_SIZES:
        for key, val in MEASURED_TRAFFIC.items():
            if val is not None:
                rl[key]["traffic"] = val
    dom = "prefill_indexer" if t_idx >= t_attn else "prefill_attention"
    res = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": t_prefill + t_decode, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8-e4m3 indexer / bf16 attention (fp32 accumulate)", "data": "synthetic",
        "config": workload_config(a, ws),
        "prefill": {"tokens_per_s": value, "ms": t_prefill, "indexer_ms": t_idx, "attention_ms": t_attn},
        "decode": {"tokens_per_s": dec_tps, "ms": t_decode, "indexer_ms": t_didx, "attention_ms": t_dattn},
        "roofline": dict(rl[dom], kernel=dom),
        "roofline_all": rl,
        "peaks": {"source": pk["source"], "fp8": "2 x bf16_tflops_sustained"},
        "gpu_launches": 6 * a.steps,  # prefill: indexer (main + re-run pass), attention; decode: scores, select, attention (64 sequences fill the GPU: no split, no combine step)
        "clocks": clocks,
        "wall_s_timed": t_wall,
    }
    res["decode_steady"] = run_decode_steady(a, dsa, D, didx, dout, ws_d, ws_a, ws, dev, keys_b + gather_b + small_b,
                                             pk["hbm_gbs"])
    if not a.no_e2e:
        res["e2e"] = run_e2e(a, dsa, P, idx, out, ws_p, ws, dev)
        res["e2e"]["decode"] = run_e2e_decode(a, dsa, D, didx, dout, ws_d, ws, dev)
    if rank == 0 and not a.no_cpu_baseline:
        tps, dt, rows, cores = cpu_oracle_prefill(P, a.cpu_sample_rows)
        dtps, ddt = cpu_oracle_decode(D, 2)
        res["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                               "sample": f"{len(rows)} query rows drawn uniformly from the L={L} prefill "
                                         f"({dt:.1f} s; tokens/s = rows / time, the per-row cost tracks t)",
                               "decode_tokens_per_s": dtps,
                               "decode_sample": f"2 of the {D.B} decode sequences ({ddt:.1f} s)"}
    if ws == 1 and not a.no_fp8_probe:
        m = measure_fp8_gemm(dev)
        res["fp8_gemm_measured"] = m
        if "sustained_tflops" in m:
            ri = res["roofline_all"]["prefill_indexer"]
            ri["frac_of_measured_fp8_gemm_sustained"] = ri["achieved"] / m["sustained_tflops"]
    return res


def run_decode_steady(a, dsa, D, didx, dout, ws_d, ws_a, ws, dev, step_bytes, hbm_peak):
    """Decode steps back to back, as a serving loop runs them: the decode step
    (indexer + top-k + attention, every kernel of it) captured once in a CUDA
    graph and replayed, timed with CUDA events on the replay stream. Inside the
    combined benchmark step the decode instead follows a 75 ms prefill (L2
    full of its output, clocks lowered by the power cap)."""
    def one():
        dsa.index_topk_decode(D.q_I, D.q_scale, D.w, D.k_cache, D.k_scale, D.lens, D.topk, idx=didx, workspace=ws_d)
        dsa.sparse_mla_attn_decode(D.q, D.kv, didx, D.scale, out=dout, workspace=ws_a)
    try:
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            one()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize()
        n_in = 20
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(n_in):
                one()
        for _ in range(max(1, a.warmup)):
            g.replay()
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(a.steps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        dsa.check_device_error()
        ms_local, err = e0.elapsed_time(e1) / (a.steps * n_in), None
        del g
    except Exception as e:
        ms_local, err = 1e30, f"{type(e).__name__}: {e}"
    ms = max_over_ranks(ms_local, ws)  # every rank takes part, failed or not
    if err is not None or ms >= 1e30:
        return {"value": None, "unit": "tokens/s", "error": err or "failed on another rank"}
    gbs = step_bytes / (ms * 1e-3) / 1e9
    return {"value": ws * D.B / (ms * 1e-3), "unit": "tokens/s", "ms": ms,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak},
            "method": f"CUDA graph of {n_in} decode steps replayed {a.steps} times"}


def run_e2e(a, dsa, P, idx, out, ws_p, ws, dev):
    """Same prefill metric through the public API with pinned host buffers:
    every step copies the inputs host->device and the output back."""
    need = sum(getattr(P, n).numel() * getattr(P, n).element_size()
               for n in ("q_I", "q_scale", "w", "k_cache", "k_scale", "q", "kv")) + out.numel() * out.element_size()
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        avail = None
    if avail is not None and avail < 2 * need:
        return {"value": None, "unit": "tokens/s", "error": f"host memory: {avail} bytes free, {need} needed pinned"}
    try:
        host = {n: getattr(P, n).cpu().pin_memory() for n in ("q_I", "q_scale", "w", "k_cache", "k_scale", "q", "kv")}
        out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    except Exception as e:  # host memory too small to pin
        return {"value": None, "unit": "tokens/s", "error": f"{type(e).__name__}: {e}"}
    dev_bufs = {n: getattr(P, n) for n in host}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out.numel() * out.element_size()
    # Query rows in nch chunks: chunk c's inputs copy in on s_in while chunk
    # c-1 computes on s_cmp and chunk c-2's output copies out on s_out. The
    # chunked selection equals the whole-sequence one row for row, so the
    # result is the same as one call over all rows.
    nch = max(1, min(a.e2e_chunks, P.L))
    bounds = [(P.L * c) // nch for c in range(nch + 1)]
    per_row = ("q_I", "q_scale", "w", "q")  # the cache-wide inputs copy first
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    tq_max = max(bounds[c + 1] - bounds[c] for c in range(nch))
    ws_c = torch.empty(max(dsa.index_topk_workspace_size(tq_max, P.H_I, P.d_I, P.topk), 16), dtype=torch.uint8,
                       device=dev)
    times = []
    for s in range(a.warmup + a.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(s_in)
        with torch.cuda.stream(s_in):
            for n in ("k_cache", "k_scale", "kv"):
                dev_bufs[n].copy_(host[n], non_blocking=True)
        for c in range(nch):
            r0, r1 = bounds[c], bounds[c + 1]
            with torch.cuda.stream(s_in):
                for n in per_row:
                    dev_bufs[n][r0:r1].copy_(host[n][r0:r1], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev)
                dsa.index_topk_chunk(P.q_I[r0:r1], P.q_scale[r0:r1], P.w[r0:r1], P.k_cache[:r1], P.k_scale[:r1],
                                     r0, P.topk, idx=idx[r0:r1], workspace=ws_c)
                dsa.sparse_mla_attn(P.q[r0:r1], P.kv[:r1], idx[r0:r1], P.scale, out=out[r0:r1])
                done = torch.cuda.Event()
                done.record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done)
                out_h[r0:r1].copy_(out[r0:r1], non_blocking=True)
        e1.record(s_out)  # s_out waited on every chunk's compute, which waited on its inputs
        torch.cuda.synchronize()
        if s >= a.warmup:
            times.append(e0.elapsed_time(e1))
    t = max_over_ranks(float(np.mean(times)), ws)
    return {"value": ws * P.L / (t * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": t, "scope": "prefill (the headline metric)",
            "pipeline": f"{nch} query-row chunks; copies in, compute and copies out on three streams"}


def run_e2e_decode(a, dsa, D, didx, dout, ws_d, ws, dev):
    """Decode tokens/s through the public API with host buffers: every step
    copies the step's new-token inputs (indexer query, its scale and head
    weights, the attention query) host->device and the output back; the key
    and latent caches stay resident on the device, as in serving."""
    names = ("q_I", "q_scale", "w", "q")
    try:
        host = {n: getattr(D, n).cpu().pin_memory() for n in names}
        out_h = torch.empty(dout.shape, dtype=dout.dtype).pin_memory()
    except Exception as e:
        return {"value": None, "unit": "tokens/s", "error": f"{type(e).__name__}: {e}"}
    dev_bufs = {n: getattr(D, n) for n in names}
    ws_a = torch.empty(dsa.split_workspace_size(D.B, D.topk), dtype=torch.uint8, device=dev)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = dout.numel() * dout.element_size()
    stream = torch.cuda.current_stream(dev)
    times = []
    for s in range(a.warmup + 4 * a.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for n, t in host.items():
            dev_bufs[n].copy_(t, non_blocking=True)
        dsa.index_topk_decode(D.q_I, D.q_scale, D.w, D.k_cache, D.k_scale, D.lens, D.topk, idx=didx, workspace=ws_d)
        dsa.sparse_mla_attn_decode(D.q, D.kv, didx, D.scale, out=dout, workspace=ws_a)
        out_h.copy_(dout, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        if s >= a.warmup:
            times.append(e0.elapsed_time(e1))
    t = max_over_ranks(float(np.mean(times)), ws)
    return {"value": ws * D.B / (t * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": t,
            "scope": "decode: new-token inputs in, output out; caches resident"}


# ------------------------------------------------------- reference (oracle)

def run_reference(a, ws, rank):
    """The float64 oracle on host cores, a bounded sample per step."""
    cfgP = dict(workloads.CONFIGS["prefill_L131072"])
    cfgP["L"] = a.prefill_L
    # inputs drawn on the CPU with the same recipe (a CPU generator stream)
    P = workloads.make_prefill(cfgP["L"], cfgP["H_I"], cfgP["d_I"], 1, cfgP["topk"], seed=0, device="cpu")
    # the sample needs only a few query rows of the 128-head queries
    g = torch.Generator().manual_seed(7)
    import oracle
    # eight rows per host thread and step keep every core busy while the
    # per-row cost varies with t (rows are drawn uniformly over the prefill)
    rows_per_step = 8 * max(1, oracle.num_threads())
    q_rows = torch.randn((rows_per_step * (a.warmup + a.steps), 128, D_QK), generator=g).to(torch.bfloat16)
    times = []
    rng = np.random.default_rng(1)
    for s in range(a.warmup + a.steps):
        rows = np.sort(rng.choice(P.L, size=rows_per_step, replace=False))
        t0 = time.perf_counter()
        sc = oracle.index_scores(P.q_I, P.q_scale, P.w, P.k_cache, P.k_scale, rows)
        ix = oracle.topk(sc, rows, P.topk)
        oracle.sparse_mla(q_rows[s * rows_per_step:(s + 1) * rows_per_step], P.kv, ix, P.scale)
        dt = time.perf_counter() - t0
        if s >= a.warmup:
            times.append(dt)
    per_row = float(np.mean(times)) / rows_per_step
    value = 1.0 / per_row
    cores = min(rows_per_step, oracle.num_threads())
    sample = (f"{rows_per_step} query rows per step drawn uniformly from the L={P.L} prefill (indexer, top-k and "
              f"attention for each; tokens/s = rows / time; the decode part of the workload is not timed here)")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": float(np.mean(times)) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(a, ws),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def _time_calls(fn, repeat, dsa):
    """Mean CUDA-event time (ms) of the calls after the first min(3, repeat - 1)."""
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
    return e0.elapsed_time(e1) / (repeat - warm), repeat - warm


def run_kernel(a):
    """One hot-path call, repeated on seeded synthetic inputs of the benchmark's shapes."""
    import long_context_03_b200 as dsa
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    L, B, DL, k = a.prefill_L, a.decode_B, a.decode_L, 2048
    if a.kernel == "indexer":
        # the indexer never reads the attention queries: one query head keeps the inputs small
        P = workloads.make_prefill(L, 64, 128, 1, k, seed=0, device=dev)
        ws = torch.empty(dsa.index_topk_workspace_size(L, 64, 128, k), dtype=torch.uint8, device=dev)
        idx = torch.empty((L, k), dtype=torch.int32, device=dev)
        fn = lambda: dsa.index_topk(P.q_I, P.q_scale, P.w, P.k_cache, P.k_scale, k, idx=idx, workspace=ws)
        shape = {"L": L}
    elif a.kernel == "attention":
        P = workloads.make_prefill(L, 64, 128, 128, k, seed=0, device=dev)
        idx = dsa.index_topk(P.q_I, P.q_scale, P.w, P.k_cache, P.k_scale, k)
        out = torch.empty((L, 128, D_V), dtype=torch.bfloat16, device=dev)
        fn = lambda: dsa.sparse_mla_attn(P.q, P.kv, idx, P.scale, out=out)
        shape = {"L": L}
    elif a.kernel == "attention_chunk":
        # the attention of the last T rows of an L-token prefill: their real
        # selections (the chunked indexer) over the whole latent cache, with
        # queries only for those rows (the full query tensor would be 19 GB)
        T = min(a.chunk_T, L)
        P = workloads.make_prefill(L, 64, 128, 1, k, seed=0, device=dev)
        q0 = L - T
        idx = dsa.index_topk_chunk(P.q_I[q0:].contiguous(), P.q_scale[q0:].contiguous(), P.w[q0:].contiguous(),
                                   P.k_cache, P.k_scale, q0, k)
        g = torch.Generator(device=dev).manual_seed(1)
        q = torch.randn((T, 128, D_QK), generator=g, device=dev).to(torch.bfloat16)
        out = torch.empty((T, 128, D_V), dtype=torch.bfloat16, device=dev)
        fn = lambda: dsa.sparse_mla_attn(q, P.kv, idx, P.scale, out=out)
        shape = {"L": L, "T": T}
    elif a.kernel == "rope":
        g = torch.Generator(device=dev).manual_seed(0)
        xq = torch.randn((B, 64, 128), generator=g, device=dev)
        xk = torch.randn((B, 128), generator=g, device=dev)
        pos = torch.randint(0, L, (B,), generator=g, device=dev, dtype=torch.int32)

        def fn():
            dsa.rope_quantize_e4m3_rows(xq, pos)
            dsa.rope_quantize_e4m3_rows(xk, pos)
        shape = {"B": B}
    elif a.kernel == "decode_paged":
        # both caches in one shuffled pool of pages (every sequence full length)
        D = workloads.make_decode(B, DL, 64, 128, 128, k, seed=0, device=dev)
        npg = DL // a.page
        perm = torch.randperm(B * npg, device=dev)
        k_pool = torch.empty((B * DL, 128), dtype=torch.uint8, device=dev)
        k_pool.view(-1, a.page, 128)[perm] = D.k_cache.view(torch.uint8).reshape(-1, a.page, 128)
        ks_pool = torch.empty((B * DL,), dtype=torch.float32, device=dev)
        ks_pool.view(-1, a.page)[perm] = D.k_scale.reshape(-1, a.page)
        kv_pool = torch.empty((B * DL, D_QK), dtype=torch.bfloat16, device=dev)
        kv_pool.view(-1, a.page, D_QK)[perm] = D.kv.reshape(-1, a.page, D_QK)
        table = perm.to(torch.int32).view(B, npg)
        ws = torch.empty(dsa.index_topk_decode_workspace_size(B, DL, k), dtype=torch.uint8, device=dev)
        ws_a = torch.empty(dsa.split_workspace_size(B, k), dtype=torch.uint8, device=dev)
        idx = torch.empty((B, k), dtype=torch.int32, device=dev)
        out = torch.empty((B, 128, D_V), dtype=torch.bfloat16, device=dev)

        def fn():
            dsa.index_topk_decode_paged(D.q_I, D.q_scale, D.w, k_pool, ks_pool, table, D.lens, k,
                                        page_size=a.page, idx=idx, workspace=ws)
            dsa.sparse_mla_attn_paged(D.q, kv_pool, table, idx, DL, D.scale, page_size=a.page, out=out,
                                      split=True, workspace=ws_a)
        shape = {"B": B, "L": DL, "page": a.page}
    else:
        D = workloads.make_decode(B, DL, 64, 128, 128, k, seed=0, device=dev)
        ws = torch.empty(dsa.index_topk_decode_workspace_size(B, DL, k), dtype=torch.uint8, device=dev)
        ws_a = torch.empty(dsa.split_workspace_size(B, k), dtype=torch.uint8, device=dev)
        idx = torch.empty((B, k), dtype=torch.int32, device=dev)
        out = torch.empty((B, 128, D_V), dtype=torch.bfloat16, device=dev)

        def fn():
            dsa.index_topk_decode(D.q_I, D.q_scale, D.w, D.k_cache, D.k_scale, D.lens, k, idx=idx, workspace=ws)
            dsa.sparse_mla_attn_decode(D.q, D.kv, idx, D.scale, out=out, workspace=ws_a)
        shape = {"B": B, "L": DL}
    ms, n = _time_calls(fn, a.repeat, dsa)
    return {"kernel": a.kernel, "ms": ms, "calls_timed": n, "calls": a.repeat, **shape}


def main():
    a = parse()
    if a.kernel is not None:
        print(json.dumps(run_kernel(a)))
        return
    if a.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        ws = int(os.environ.get("WORLD_SIZE", "1"))
        if rank != 0:
            return
        print(json.dumps(run_reference(a, ws, rank)))
        return
    ws, rank, _ = dist_setup(a.gpus)
    try:
        res = run_ours(a, ws, rank)
        if rank == 0:
            print(json.dumps(res))
    finally:
        if ws > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
