"""The decode step captured in a CUDA graph (as a serving loop replays it):
every call of it can be captured, and a replay gives bit for bit what the
eager calls give, for a batch that splits its selections over the clusters
(with the combine step) and for one that does not."""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import long_context_03_b200 as m
    m.lib()
    return m


@pytest.mark.parametrize("B,lens", [(6, [5000, 4999, 1, 2048, 2049, 3333]), (64, None)])
def test_replayed_decode_step_equals_eager(dsa, B, lens):
    L, k = 5000, 2048
    D = workloads.make_decode(B, L, 64, 128, 128, k, seed=61, lens=lens, device="cuda")
    ws = torch.empty(dsa.index_topk_decode_workspace_size(B, L, k), dtype=torch.uint8, device="cuda")
    ws_a = torch.empty(dsa.split_workspace_size(B, k), dtype=torch.uint8, device="cuda")
    idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
    out = torch.empty((B, 128, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 128), dtype=torch.float32, device="cuda")

    def step():
        dsa.index_topk_decode(D.q_I, D.q_scale, D.w, D.k_cache, D.k_scale, D.lens, k, idx=idx, workspace=ws)
        dsa.sparse_mla_attn_decode(D.q, D.kv, idx, D.scale, out=out, lse=lse, workspace=ws_a)

    step()
    torch.cuda.synchronize()
    dsa.check_device_error()
    ref = (idx.clone(), out.clone(), lse.clone())
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for t in (idx, out, lse):
        t.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    dsa.check_device_error()
    assert torch.equal(idx, ref[0])
    assert torch.equal(out, ref[1]) and torch.equal(lse, ref[2])
    del g
