"""Packed batches of sequences (cu_seqlens form): each sequence's rows of
the batched selection must equal the single-sequence selection bit for bit
(same exact selection and total ranking), for full prefills, mid-cache
chunks and single decode-like queries mixed in one call."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import long_context_03_b200 as m
    m.lib()
    return m


def test_packed_batch_equals_per_sequence_calls(dsa):
    # (keys, queries, first query position): a long full prefill that takes
    # the sampled-threshold path, a chunk in the middle of its cache, a
    # single query at the end of its cache, a short full prefill
    shapes = [(20000, 20000, 0), (6000, 700, 3000), (9000, 1, 8999), (1500, 1500, 0)]
    seqs = [workloads.make_prefill(lk, 64, 128, 1, 2048, seed=70 + i, device="cuda") for i, (lk, _, _) in enumerate(shapes)]
    q_parts, qs_parts, w_parts, k_parts, ks_parts, cu_q, cu_k, pos0 = [], [], [], [], [], [0], [0], []
    for P, (lk, tq, q0) in zip(seqs, shapes):
        q_parts.append(P.q_I[q0:q0 + tq]); qs_parts.append(P.q_scale[q0:q0 + tq]); w_parts.append(P.w[q0:q0 + tq])
        k_parts.append(P.k_cache); ks_parts.append(P.k_scale)
        cu_q.append(cu_q[-1] + tq); cu_k.append(cu_k[-1] + lk); pos0.append(q0)
    cat = lambda xs: torch.cat(xs).contiguous()
    idx = dsa.index_topk_varlen(cat(q_parts), cat(qs_parts), cat(w_parts), cat(k_parts), cat(ks_parts),
                                cu_q, cu_k, 2048, q_pos0=pos0)
    dsa.check_device_error()
    for b, (P, (lk, tq, q0)) in enumerate(zip(seqs, shapes)):
        ref = dsa.index_topk_chunk(P.q_I[q0:q0 + tq].contiguous(), P.q_scale[q0:q0 + tq].contiguous(),
                                   P.w[q0:q0 + tq].contiguous(), P.k_cache, P.k_scale, q0, 2048)
        assert torch.equal(idx[cu_q[b]:cu_q[b + 1]], ref), b
    # default positions: the queries are the last tokens of each cache
    idx2 = dsa.index_topk_varlen(cat(q_parts[2:3]), cat(qs_parts[2:3]), cat(w_parts[2:3]), cat(k_parts[2:3]),
                                 cat(ks_parts[2:3]), [0, 1], [0, 9000], 2048)
    assert torch.equal(idx2, idx[cu_q[2]:cu_q[3]])
