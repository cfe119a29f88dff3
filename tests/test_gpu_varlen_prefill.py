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


def _packed(shapes, seed0, Hq=1):
    seqs = [workloads.make_prefill(lk, 64, 128, Hq, 2048, seed=seed0 + i, device="cuda")
            for i, (lk, _, _) in enumerate(shapes)]
    parts = {n: [] for n in ("q_I", "q_scale", "w", "q", "k_cache", "k_scale", "kv")}
    cu_q, cu_k, pos0 = [0], [0], []
    for P, (lk, tq, q0) in zip(seqs, shapes):
        for n in ("q_I", "q_scale", "w", "q"):
            parts[n].append(getattr(P, n)[q0:q0 + tq])
        for n in ("k_cache", "k_scale", "kv"):
            parts[n].append(getattr(P, n))
        cu_q.append(cu_q[-1] + tq)
        cu_k.append(cu_k[-1] + lk)
        pos0.append(q0)
    cat = {n: torch.cat(v).contiguous() for n, v in parts.items()}
    return seqs, cat, cu_q, cu_k, pos0


def test_packed_batch_rows_match_the_oracle(dsa):
    """Sampled rows of every packed sequence against the oracle on that
    sequence's own keys (positions q0 + local row), and bit-exact against a
    CPU top-k of the GPU's own scores for the same rows."""
    import oracle
    from gpu_helpers import cpu_topk_of, overlap_excluding_ties, score_tolerance_ok
    shapes = [(20000, 20000, 0), (6000, 700, 3000), (9000, 1, 8999), (1500, 1500, 0)]
    seqs, c, cu_q, cu_k, pos0 = _packed(shapes, 70)
    idx = dsa.index_topk_varlen(c["q_I"], c["q_scale"], c["w"], c["k_cache"], c["k_scale"], cu_q, cu_k, 2048,
                                q_pos0=pos0)
    dsa.check_device_error()
    g = np.random.default_rng(3)
    for b, (P, (lk, tq, q0)) in enumerate(zip(seqs, shapes)):
        local = sorted(set([0, tq - 1] + g.choice(tq, min(tq, 6), replace=False).tolist()))
        rows = np.asarray([q0 + r for r in local], dtype=np.int64)
        h = {n: getattr(P, n).cpu() for n in ("q_I", "q_scale", "w", "k_cache", "k_scale")}
        ref_sc = oracle.index_scores(h["q_I"][rows], h["q_scale"][rows], h["w"][rows], h["k_cache"], h["k_scale"],
                                     rows, query_rows=np.arange(len(rows)))
        gidx = idx[[cu_q[b] + r for r in local]].cpu().numpy()
        assert overlap_excluding_ties(gidx, oracle.topk(ref_sc, rows, 2048), ref_sc, rows, 2048) >= 0.999, b
        for r, t in enumerate(rows):
            n = min(2048, int(t) + 1)
            assert np.all((gidx[r, :n] >= 0) & (gidx[r, :n] <= t)) and np.all(gidx[r, n:] == -1)
            sc = dsa.index_scores(P.q_I, P.q_scale, P.w, P.k_cache, P.k_scale, int(t), 1).cpu().numpy()
            assert np.array_equal(gidx[r], cpu_topk_of(sc, [int(t)], 2048)[0]), (b, int(t))
            ok, worst = score_tolerance_ok(sc, ref_sc[r:r + 1], [int(t)])
            assert ok, (b, int(t), worst)


def test_packed_attention_matches_per_sequence_calls_and_the_oracle(dsa):
    """Attention over a packed batch (sequence-local indices from the varlen
    selection): every token equals the single-sequence call bit for bit, and
    sampled tokens of every sequence match the oracle."""
    import oracle
    from gpu_helpers import attn_close
    shapes = [(3000, 3000, 0), (6000, 700, 3000), (9000, 1, 8999), (1500, 1500, 0), (2100, 37, 2063)]
    seqs, c, cu_q, cu_k, pos0 = _packed(shapes, 80, Hq=16)
    idx = dsa.index_topk_varlen(c["q_I"], c["q_scale"], c["w"], c["k_cache"], c["k_scale"], cu_q, cu_k, 2048,
                                q_pos0=pos0)
    out, lse = dsa.sparse_mla_attn_varlen(c["q"], c["kv"], idx, cu_q, cu_k, seqs[0].scale, want_lse=True)
    dsa.check_device_error()
    g = np.random.default_rng(4)
    for b, (P, (lk, tq, q0)) in enumerate(zip(seqs, shapes)):
        sl = slice(cu_q[b], cu_q[b + 1])
        ref, ref_lse = dsa.sparse_mla_attn(P.q[q0:q0 + tq].contiguous(), P.kv, idx[sl].contiguous(), P.scale,
                                           want_lse=True)
        assert torch.equal(out[sl], ref) and torch.equal(lse[sl], ref_lse), b
        local = sorted(set([0, tq - 1] + g.choice(tq, min(tq, 3), replace=False).tolist()))
        rows = [cu_q[b] + r for r in local]
        ref_o, _ = oracle.sparse_mla(P.q[[q0 + r for r in local]].cpu(), P.kv.cpu(), idx[rows].cpu().numpy(), P.scale)
        ok, mx, rl = attn_close(out[rows], ref_o)
        assert ok, (b, mx, rl)


def test_packed_attention_reports_an_index_past_its_sequence(dsa):
    shapes = [(300, 300, 0), (500, 10, 490)]
    seqs, c, cu_q, cu_k, pos0 = _packed(shapes, 90, Hq=16)
    idx = dsa.index_topk_varlen(c["q_I"], c["q_scale"], c["w"], c["k_cache"], c["k_scale"], cu_q, cu_k, 2048,
                                q_pos0=pos0)
    dsa.check_device_error()
    bad = idx.clone()
    bad[0, 0] = 300  # local row 300 is past the first sequence's 300 rows (it would be the second's row 0)
    out, _ = dsa.sparse_mla_attn_varlen(c["q"], c["kv"], bad, cu_q, cu_k, seqs[0].scale)
    st, _ = dsa.device_error()
    assert st == -6  # DSA_ERR_BAD_INDEX
    skip = idx.clone()
    skip[0, 0] = -1
    ref, _ = dsa.sparse_mla_attn_varlen(c["q"], c["kv"], skip, cu_q, cu_k, seqs[0].scale)
    assert torch.equal(out, ref)
