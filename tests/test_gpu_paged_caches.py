"""Paged caches equal the contiguous ones bit for bit.

Attention over a paged latent cache gathers the same rows in the same order
as over the contiguous cache, for per-token tables (decode) and one shared
table (prefill); a page entry outside the pool skips its rows and is
reported. The decode indexer over a paged FP8 key cache computes the same
scores (same codes, same scales, same arithmetic), so its top-k equals the
contiguous call's exactly; a bad page entry is reported."""
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
    out, lse = dsa.sparse_mla_attn_paged(D.q, pool, table, idx, L, D.scale, page_size=page, want_lse=True,
                                         split=True)
    dsa.check_device_error()
    assert torch.equal(out, ref) and torch.equal(lse, ref_lse)
    # one cluster per sequence (no split) in both forms
    ref1, ref1_lse = dsa.sparse_mla_attn_decode(D.q, D.kv, idx, D.scale, want_lse=True, split=False)
    out1, lse1 = dsa.sparse_mla_attn_paged(D.q, pool, table, idx, L, D.scale, page_size=page, want_lse=True)
    dsa.check_device_error()
    assert torch.equal(out1, ref1) and torch.equal(lse1, ref1_lse)


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


def _page_keys(k_cache, k_scale, lens, page, gen, spare=5):
    """Scatter every sequence's key pages into one shuffled pool.

    Returns (k_pool [pool_rows, d], ks_pool [pool_rows], table [B, max_blocks]);
    table entries of pages past a sequence's length are -1 (never read)."""
    B, L, d = k_cache.shape
    max_blocks = (L + page - 1) // page
    Lp = max_blocks * page
    kc = torch.zeros((B, Lp, d), dtype=torch.uint8, device=k_cache.device)
    kc[:, :L] = k_cache.view(torch.uint8)
    ks = torch.zeros((B, Lp), dtype=torch.float32, device=k_cache.device)
    ks[:, :L] = k_scale
    used = [(int(n) + page - 1) // page for n in lens.tolist()]
    total = sum(used)
    perm = torch.randperm(total + spare, generator=gen)[:total].to(k_cache.device)
    k_pool = torch.zeros(((total + spare) * page, d), dtype=torch.uint8, device=k_cache.device)
    ks_pool = torch.full(((total + spare) * page,), 7.0, dtype=torch.float32, device=k_cache.device)
    table = torch.full((B, max_blocks), -1, dtype=torch.int32)
    i = 0
    for b in range(B):
        dst = perm[i:i + used[b]]
        rows = (dst[:, None] * page + torch.arange(page, device=k_cache.device)[None]).reshape(-1)
        k_pool[rows] = kc[b, :used[b] * page].reshape(-1, d)
        ks_pool[rows] = ks[b, :used[b] * page].reshape(-1)
        table[b, :used[b]] = dst.cpu().to(torch.int32)
        i += used[b]
    return k_pool, ks_pool, table.to(k_cache.device)


@pytest.mark.parametrize("page", [16, 64, 128, 256])
def test_decode_indexer_paged_keys_match_contiguous(dsa, page):
    B, L = 6, 5000
    D = workloads.make_decode(B, L, 64, 128, 128, 2048, seed=41, lens=[5000, 4999, 1, 2048, 2049, 3333],
                              device="cuda")
    ref = dsa.index_topk_decode(D.q_I, D.q_scale, D.w, D.k_cache, D.k_scale, D.lens, 2048)
    k_pool, ks_pool, table = _page_keys(D.k_cache, D.k_scale, D.lens, page, torch.Generator().manual_seed(page))
    idx = dsa.index_topk_decode_paged(D.q_I, D.q_scale, D.w, k_pool, ks_pool, table, D.lens, 2048, page_size=page)
    dsa.check_device_error()
    assert torch.equal(idx, ref)


def test_paged_decode_step_matches_contiguous(dsa):
    """A whole decode step (indexer + attention) with both caches paged, at 64K."""
    B, L, page = 16, 65536, 64
    lens = [65536, 65535, 40000, 2049, 1, 30001, 65472, 12345, 65536, 777, 50000, 64, 65, 2048, 33333, 60000]
    D = workloads.make_decode(B, L, 64, 128, 128, 2048, seed=43, lens=lens, device="cuda")
    ref_idx = dsa.index_topk_decode(D.q_I, D.q_scale, D.w, D.k_cache, D.k_scale, D.lens, 2048)
    ref_out, ref_lse = dsa.sparse_mla_attn_decode(D.q, D.kv, ref_idx, D.scale, want_lse=True)
    gen = torch.Generator().manual_seed(9)
    k_pool, ks_pool, table = _page_keys(D.k_cache, D.k_scale, D.lens, page, gen)
    # the latent rows use the same page numbers as the keys (one page table per sequence)
    kv_pool = torch.zeros((k_pool.shape[0], 576), dtype=torch.bfloat16, device="cuda")
    for b in range(B):
        n = (lens[b] + page - 1) // page
        rows = (table[b, :n].long()[:, None] * page + torch.arange(page, device="cuda")[None]).reshape(-1)
        src = torch.zeros((n * page, 576), dtype=torch.bfloat16, device="cuda")
        m = min(n * page, L)
        src[:m] = D.kv[b, :m]
        kv_pool[rows] = src
    idx = dsa.index_topk_decode_paged(D.q_I, D.q_scale, D.w, k_pool, ks_pool, table, D.lens, 2048, page_size=page)
    out, lse = dsa.sparse_mla_attn_paged(D.q, kv_pool, table, idx, L, D.scale, page_size=page, want_lse=True,
                                         split=True)
    dsa.check_device_error()
    assert torch.equal(idx, ref_idx)
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)


def test_decode_indexer_bad_page_is_reported(dsa):
    B, L, page = 2, 3000, 64
    D = workloads.make_decode(B, L, 64, 128, 128, 2048, seed=47, lens=[3000, 2500], device="cuda")
    k_pool, ks_pool, table = _page_keys(D.k_cache, D.k_scale, D.lens, page, torch.Generator().manual_seed(3))
    dsa.check_device_error()
    bad = table.clone()
    bad[1, 5] = 10 ** 6
    dsa.index_topk_decode_paged(D.q_I, D.q_scale, D.w, k_pool, ks_pool, bad, D.lens, 2048, page_size=page)
    st, _ = dsa.device_error()
    assert st == -6  # DSA_ERR_BAD_INDEX
    # the good sequence is unaffected
    ref = dsa.index_topk_decode(D.q_I, D.q_scale, D.w, D.k_cache, D.k_scale, D.lens, 2048)
    idx = dsa.index_topk_decode_paged(D.q_I, D.q_scale, D.w, k_pool, ks_pool, bad, D.lens, 2048, page_size=page)
    dsa.device_error()
    assert torch.equal(idx[0], ref[0])


def _page_one(k_cache, k_scale, page, gen, spare=3):
    """One sequence's keys [L, d] and scales [L] in a shuffled pool; table [max_blocks]."""
    L, d = k_cache.shape
    npg = (L + page - 1) // page
    perm = torch.randperm(npg + spare, generator=gen)[:npg].to(k_cache.device)
    k_pool = torch.zeros(((npg + spare) * page, d), dtype=torch.uint8, device=k_cache.device)
    ks_pool = torch.full(((npg + spare) * page,), 5.0, dtype=torch.float32, device=k_cache.device)
    kc = torch.zeros((npg * page, d), dtype=torch.uint8, device=k_cache.device)
    kc[:L] = k_cache.view(torch.uint8)
    ks = torch.zeros((npg * page,), dtype=torch.float32, device=k_cache.device)
    ks[:L] = k_scale
    rows = (perm[:, None] * page + torch.arange(page, device=k_cache.device)[None]).reshape(-1)
    k_pool[rows] = kc
    ks_pool[rows] = ks
    return k_pool, ks_pool, perm.to(torch.int32)


@pytest.mark.parametrize("page", [16, 64, 256])
def test_prefill_chunk_paged_keys_match_contiguous(dsa, page):
    L = 20480  # long enough for the sampled starting thresholds
    P = workloads.make_prefill(L, 64, 128, 1, 2048, seed=51, device="cuda")
    k_pool, ks_pool, table = _page_one(P.k_cache, P.k_scale, page, torch.Generator().manual_seed(page))
    for q0, Tq in [(0, L), (17000, 3000), (4095, 1)]:
        sl = slice(q0, q0 + Tq)
        ref = dsa.index_topk_chunk(P.q_I[sl], P.q_scale[sl], P.w[sl], P.k_cache[:q0 + Tq], P.k_scale[:q0 + Tq],
                                   q0, 2048)
        idx = dsa.index_topk_chunk_paged(P.q_I[sl], P.q_scale[sl], P.w[sl], k_pool, ks_pool, table, q0, q0 + Tq,
                                         2048, page_size=page)
        dsa.check_device_error()
        assert torch.equal(idx, ref), (q0, Tq)


def test_prefill_chunk_bad_page_is_reported(dsa):
    L = 4096
    P = workloads.make_prefill(L, 64, 128, 1, 2048, seed=53, device="cuda")
    k_pool, ks_pool, table = _page_one(P.k_cache, P.k_scale, 64, torch.Generator().manual_seed(1))
    dsa.check_device_error()
    bad = table.clone()
    bad[10] = -7
    dsa.index_topk_chunk_paged(P.q_I, P.q_scale, P.w, k_pool, ks_pool, bad, 0, L, 2048, page_size=64)
    st, _ = dsa.device_error()
    assert st == -6  # DSA_ERR_BAD_INDEX
    # rows before the bad page never read it
    ref = dsa.index_topk_chunk(P.q_I[:640], P.q_scale[:640], P.w[:640], P.k_cache[:640], P.k_scale[:640], 0, 2048)
    idx = dsa.index_topk_chunk_paged(P.q_I[:640], P.q_scale[:640], P.w[:640], k_pool, ks_pool, bad, 0, 640, 2048,
                                     page_size=64)
    assert dsa.device_error()[0] == 0
    assert torch.equal(idx, ref)


def test_paged_decode_step_matches_the_oracle(dsa):
    """Paged decode (keys and latent rows in one shuffled pool) against the
    oracle on the logical caches: selection bit-exact against a CPU top-k of
    the GPU's own scores and >= 99.9% overlap with the oracle's, attention
    within tolerance, for ragged lengths."""
    import oracle
    from gpu_helpers import attn_close, cpu_topk_of, overlap_excluding_ties
    B, L, page = 5, 20000, 64
    lens = [20000, 2049, 1, 13333, 2048]
    D = workloads.make_decode(B, L, 64, 128, 128, 2048, seed=45, lens=lens, device="cuda")
    k_pool, ks_pool, table = _page_keys(D.k_cache, D.k_scale, D.lens, page, torch.Generator().manual_seed(11))
    kv_pool = torch.zeros((k_pool.shape[0], 576), dtype=torch.bfloat16, device="cuda")
    for b in range(B):
        n = (lens[b] + page - 1) // page
        rows = (table[b, :n].long()[:, None] * page + torch.arange(page, device="cuda")[None]).reshape(-1)
        src = torch.zeros((n * page, 576), dtype=torch.bfloat16, device="cuda")
        m = min(n * page, L)
        src[:m] = D.kv[b, :m]
        kv_pool[rows] = src
    idx = dsa.index_topk_decode_paged(D.q_I, D.q_scale, D.w, k_pool, ks_pool, table, D.lens, 2048, page_size=page)
    out, lse = dsa.sparse_mla_attn_paged(D.q, kv_pool, table, idx, L, D.scale, page_size=page, want_lse=True,
                                         split=True)
    sc = dsa.index_scores_decode(D.q_I, D.q_scale, D.w, D.k_cache, D.k_scale, D.lens)
    dsa.check_device_error()
    host = workloads.DecodeInputs(B, L, 64, 128, 128, 2048, D.scale,
                                  *[getattr(D, n).cpu() for n in ("q_I", "q_scale", "w", "k_cache", "k_scale", "q",
                                                                  "kv", "lens")])
    res = oracle.decode_seqs(host, range(B))
    gidx = idx.cpu().numpy()
    gsc = sc.cpu().numpy()
    for b in range(B):
        ref_sc, ref_idx, _, _ = res[b]
        t = lens[b] - 1
        assert np.array_equal(gidx[b], cpu_topk_of(gsc[b:b + 1, :t + 1], [t], 2048)[0]), b
        assert overlap_excluding_ties(gidx[b:b + 1], ref_idx[None], ref_sc[None], [t], 2048) >= 0.999, b
        ref_o, ref_l = oracle.sparse_mla(oracle._bf16_bits(host.q[b:b + 1]), host.kv[b, :lens[b]], gidx[b:b + 1],
                                         D.scale)
        ok, mx, rl = attn_close(out[b:b + 1], ref_o)
        assert ok, (b, mx, rl)
        np.testing.assert_allclose(lse[b].cpu().numpy(), ref_l[0], rtol=1e-4, atol=1e-4)


def test_paged_prefill_keys_and_latent_rows_match_the_oracle(dsa):
    """A chunk of a prefill over a paged FP8 key cache, then attention over a
    paged latent cache (one shared table), against the oracle on sampled rows."""
    import oracle
    from gpu_helpers import attn_close, overlap_excluding_ties
    L, page, q0, Tq = 20480, 64, 16000, 2000
    P = workloads.make_prefill(L, 64, 128, 16, 2048, seed=57, device="cuda")
    k_pool, ks_pool, table = _page_one(P.k_cache, P.k_scale, page, torch.Generator().manual_seed(12))
    sl = slice(q0, q0 + Tq)
    idx = dsa.index_topk_chunk_paged(P.q_I[sl], P.q_scale[sl], P.w[sl], k_pool, ks_pool, table, q0, q0 + Tq, 2048,
                                     page_size=page)
    kv_pool, kv_table = _page(P.kv[:q0 + Tq], page, torch.Generator().manual_seed(13))
    out, _ = dsa.sparse_mla_attn_paged(P.q[sl].contiguous(), kv_pool, kv_table.cuda()[None], idx, q0 + Tq, P.scale,
                                       page_size=page)
    dsa.check_device_error()
    local = [0, 1, 999, 1998, 1999]
    rows = np.asarray([q0 + r for r in local], dtype=np.int64)
    h = {n: getattr(P, n).cpu() for n in ("q_I", "q_scale", "w", "k_cache", "k_scale")}
    ref_sc = oracle.index_scores(h["q_I"][rows], h["q_scale"][rows], h["w"][rows], h["k_cache"], h["k_scale"], rows,
                                 query_rows=np.arange(len(rows)))
    gidx = idx[local].cpu().numpy()
    assert overlap_excluding_ties(gidx, oracle.topk(ref_sc, rows, 2048), ref_sc, rows, 2048) >= 0.999
    ref_o, _ = oracle.sparse_mla(P.q[rows.tolist()].cpu(), P.kv.cpu(), gidx, P.scale)
    ok, mx, rl = attn_close(out[local], ref_o)
    assert ok, (mx, rl)
