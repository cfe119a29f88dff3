"""Failure detection without a GPU fault: a kernel whose bounded wait runs
out (a barrier that nothing completes) records a timeout that the host reads
and clears, and the context stays usable for the next calls."""
import time

import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import long_context_03_b200 as m
    m.lib()
    return m


@pytest.mark.parametrize("cycles", [1 << 20, 0])
def test_a_wait_that_runs_out_is_reported_and_the_context_survives(dsa, cycles):
    dsa.check_device_error()
    P = workloads.make_config("tiny_L512", device="cuda")
    before = dsa.index_topk(P.q_I, P.q_scale, P.w, P.k_cache, P.k_scale, P.topk)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    dsa.selftest_wait_timeout(cycles)
    st, raw = dsa.device_error()
    waited = time.perf_counter() - t0
    assert st == -4 and (raw & 0xFF) == 1 and (raw >> 8) == 99  # timeout, self-test site
    if cycles:
        assert waited < 0.5  # 2^20 cycles are about half a millisecond
    else:
        assert 0.2 < waited < 10.0  # the library's own bound, ~2^31 SM cycles
    assert dsa.device_error()[0] == 0  # read and cleared
    after = dsa.index_topk(P.q_I, P.q_scale, P.w, P.k_cache, P.k_scale, P.topk)
    dsa.check_device_error()
    assert torch.equal(before, after)
