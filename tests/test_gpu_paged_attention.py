"""Attention over a paged latent cache equals attention over the contiguous
cache bit for bit (the same rows are gathered in the same order), for
per-token tables (decode) and one shared table (prefill); a page entry
outside the pool skips its rows and is reported."""
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


def _page(kv_rows, page, gen):
    """Scatter [n, 576] rows into a shuffled pool of pages; return (pool, table [n_pages])."""
    n = kv_rows.shape[0]
    npg = (n + page - 1) // page
    perm = torch.randperm(npg + 3, generator=gen)[:npg]  # a few spare pages in the pool
    pool = torch.zeros(((npg + 3) * page, 576), dtype=torch.bfloat16, device=kv_rows.device)
    for i in range(npg):
        rows = kv_rows[i * page:(i + 1) * page]
        pool[perm[i] * page:perm[i] * page + rows.shape[0]] = rows
    return pool, perm.to(torch.int32)


def test_decode_tables_match_contiguous(dsa):
    B, L, page = 6, 5000, 64
    D = workloads.make_decode(B, L, 64, 128, 128, 2048, seed=31, lens=[5000, 4999, 1, 2048, 2049, 3333], device="cuda")
    idx = dsa.index_topk_decode(D.q_I, D.q_scale, D.w, D.k_cache, D.k_scale, D.lens, 2048)
    ref, ref_lse = dsa.sparse_mla_attn_decode(D.q, D.kv, idx, D.scale, want_lse=True)
    gen = torch.Generator().manual_seed(5)
    pools, tables = [], []
    base = 0
    for b in range(B):
        pool, table = _page(D.kv[b], page, gen)
        pools.append(pool)
        tables.append(table + base)
        base += pool.shape[0] // page
    pool = torch.cat(pools)
    table = torch.stack(tables).cuda()
    out, lse = dsa.sparse_mla_attn_paged(D.q, pool, table, idx, L, D.scale, page_size=page, want_lse=True)
    dsa.check_device_error()
    assert torch.equal(out, ref) and torch.equal(lse, ref_lse)


def test_prefill_shared_table_and_bad_page(dsa):
    P = workloads.make_config("tiny_L512", device="cuda")
    idx = dsa.index_topk(P.q_I, P.q_scale, P.w, P.k_cache, P.k_scale, P.topk)
    ref, _ = dsa.sparse_mla_attn(P.q, P.kv, idx, P.scale)
    pool, table = _page(P.kv, 16, torch.Generator().manual_seed(6))
    table = table.cuda()[None]
    out, _ = dsa.sparse_mla_attn_paged(P.q, pool, table, idx, P.L, P.scale, page_size=16)
    dsa.check_device_error()
    assert torch.equal(out, ref)
    # page 3 (rows 48..63) leads outside the pool: those rows are skipped and reported
    bad = table.clone()
    bad[0, 3] = 10 ** 6
    out_bad, _ = dsa.sparse_mla_attn_paged(P.q, pool, bad, idx, P.L, P.scale, page_size=16)
    st, _ = dsa.device_error()
    assert st == -6  # DSA_ERR_BAD_INDEX
    idx_skip = idx.clone()
    idx_skip[(idx_skip >= 48) & (idx_skip < 64)] = -1
    ref_skip, _ = dsa.sparse_mla_attn(P.q, P.kv, idx_skip, P.scale)
    assert torch.equal(out_bad, ref_skip)
