"""The N > 1 path of bench.py on CPU: two `gloo` ranks as separate processes.

The path has no exchange step, so N GPUs run N independent replicas; what
must hold across ranks is the timing rule (each launch's time is the max over
ranks, the job is as fast as its slowest replica) and the token count (every
rank's tokens). The reference arm under torchrun runs on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, seg_by_rank, q):
    import datetime

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=ws,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(ws)
        t, value, dec = bench.replica_totals(seg_by_rank[rank], ws, L=131072, B=64)
        bench.barrier(ws)
        q.put((rank, t, value, dec))
    finally:
        torch.distributed.destroy_process_group()


def test_replica_totals_take_the_slowest_rank():
    ws = 2
    seg = [[140.0, 130.0, 0.25, 0.10], [150.0, 120.0, 0.20, 0.12]]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, seg, q)) for r in range(ws)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(ws)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want_t = [150.0, 130.0, 0.25, 0.12]
    for rank, t, value, dec in res:
        assert t == want_t
        assert value == pytest.approx(2 * 131072 / (280.0e-3))
        assert dec == pytest.approx(2 * 64 / (0.37e-3))


def test_single_rank_totals_need_no_process_group():
    import bench
    t, value, dec = bench.replica_totals([1.0, 1.0, 0.5, 0.5], 1, L=1000, B=10)
    assert t == [1.0, 1.0, 0.5, 0.5]
    assert value == pytest.approx(1000 / 2e-3) and dec == pytest.approx(10 / 1e-3)


def _run_ref(env_extra, *args):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", *args],
                          capture_output=True, text=True, env=env, timeout=600, cwd=ROOT)


def test_reference_arm_other_ranks_exit_without_work():
    r = _run_ref({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, "--gpus", "2", "--steps", "1",
                 "--warmup", "3")
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_prints_one_contract_line():
    import oracle
    oracle.build()
    r = _run_ref({"RANK": "0", "WORLD_SIZE": "1"}, "--steps", "1", "--warmup", "3", "--prefill-L", "1024")
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["value"] > 0
    # the same workload description as the GPU arm's line, so the two lines compare
    import bench
    assert d["config"] == bench.workload_config(bench.parse(["--prefill-L", "1024"]), 1)


def test_fp8_gemm_probe_reports_instead_of_raising():
    # on a host without a GPU the probe's library call runs (small n) and the event timing fails:
    # the failure comes back as a field, the benchmark line is never lost
    import bench
    r = bench.measure_fp8_gemm(torch.device("cpu"), seconds=0.01, n=32)
    assert isinstance(r, dict) and ("error" in r or "burst_tflops" in r)


def test_roofline_work_counts():
    # the algorithmic work behind `achieved`: causal pairs for the indexer, min(k, t+1) rows per
    # query for the attention, compulsory bytes for a decode step
    import bench
    for L, k in [(1, 4), (5, 4), (37, 8), (300, 64)]:
        pairs = sum(t + 1 for t in range(L))
        sel = sum(min(k, t + 1) for t in range(L))
        idx_flop, attn_flop = bench.prefill_work(L, 8, 64, 16, k)
        assert idx_flop == 2 * 8 * 64 * pairs
        assert attn_flop == sel * 16 * 2 * (576 + 512)
    idx_flop, attn_flop = bench.prefill_work(131072, 64, 128, 128, 2048)
    assert idx_flop == pytest.approx(1.407e14, rel=1e-3) and attn_flop == pytest.approx(7.42e13, rel=1e-3)
    keys, gather, small = bench.decode_bytes(64, 65536, 64, 128, 128, 2048)
    assert keys == 64 * 65536 * 132 and gather == 64 * 2048 * 1152
    assert (keys + gather + small) / 1e6 == pytest.approx(723.5, abs=0.1)
