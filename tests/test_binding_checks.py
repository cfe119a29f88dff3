"""The Python binding refuses host tensors and foreign workspaces before any
pointer reaches the library (runs without a GPU)."""
import pytest
import torch

import workloads


@pytest.fixture(scope="module")
def dsa():
    from long_context_03_b200 import build
    build.build()
    import long_context_03_b200 as m
    return m


def test_host_tensors_are_refused(dsa):
    P = workloads.make_config("tiny_L512", device="cpu")
    with pytest.raises(ValueError, match="CUDA tensor"):
        dsa.index_topk(P.q_I, P.q_scale, P.w, P.k_cache, P.k_scale, P.topk)
    with pytest.raises(ValueError, match="CUDA tensor"):
        dsa.sparse_mla_attn(P.q, P.kv, torch.zeros((P.L, P.topk), dtype=torch.int32), P.scale)
    D = workloads.make_decode(2, 64, 64, 128, 8, 16, seed=0, device="cpu")
    with pytest.raises(ValueError, match="CUDA tensor"):
        dsa.index_topk_decode(D.q_I, D.q_scale, D.w, D.k_cache, D.k_scale, D.lens, 16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        dsa.quantize_e4m3_rows(torch.zeros((2, 8)))


def test_host_workspace_is_refused(dsa):
    with pytest.raises(ValueError, match="workspace must be a CUDA tensor"):
        dsa._ws(torch.empty(64, dtype=torch.uint8), 64, torch.device("cuda", 0))
    with pytest.raises(ValueError, match="workspace must be a CUDA tensor"):
        dsa.index_topk_rerun_count(torch.empty(64, dtype=torch.uint8), 512, 8, 64, 64)
