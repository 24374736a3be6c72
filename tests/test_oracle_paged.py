"""Pins of the paged-cache oracle (oracle.attn_fwd_paged), no GPU.

The cache is built here from dense per-request sequences by scattering their
rows into randomly placed pages (the unused rows and spare pages hold a large
poison value), and the oracle's result is checked against fp64 torch
scaled_dot_product_attention on the dense sequences with the bottom-right
causal mask.  Invariants: the page size and the physical placement of the
pages do not change the result at all; an empty request gives O = 0 and
lse = -inf; with one query the causal flag changes nothing.
"""
import numpy as np
import pytest
import torch

import oracle

POISON = 1.0e3


def dense_requests(seed, lens, H, d):
    rng = np.random.default_rng(seed)
    ks = [rng.standard_normal((L, H, d)) for L in lens]
    vs = [rng.standard_normal((L, H, d)) for L in lens]
    return ks, vs


def scatter_to_pages(ks, vs, page_size, seed, spare=2, max_blocks=None):
    """Store each request's rows page by page in randomly chosen physical pages."""
    H, d = ks[0].shape[1:] if ks[0].size else (ks[-1].shape[1], ks[-1].shape[2])
    npages = [-(-k.shape[0] // page_size) for k in ks]
    max_blocks = max(max(npages), 1) if max_blocks is None else max_blocks
    num_blocks = sum(npages) + spare
    place = np.random.default_rng(seed).permutation(num_blocks)
    k_cache = np.full((num_blocks, page_size, H, d), POISON)
    v_cache = np.full((num_blocks, page_size, H, d), -POISON)
    table = np.full((len(ks), max_blocks), -1, dtype=np.int32)
    nxt = 0
    for b, (k, v) in enumerate(zip(ks, vs)):
        for pg in range(npages[b]):
            phys = place[nxt]
            nxt += 1
            table[b, pg] = phys
            rows = slice(pg * page_size, min((pg + 1) * page_size, k.shape[0]))
            n = rows.stop - rows.start
            k_cache[phys, :n] = k[rows]
            v_cache[phys, :n] = v[rows]
    seq_lens = np.array([k.shape[0] for k in ks], dtype=np.int32)
    return k_cache, v_cache, table, seq_lens


def sdpa_dense(q, k, v, causal, scale):
    """fp64 torch SDPA of one request: q [Lq, H, d] over k, v [L, H, d], bottom-right mask."""
    Lq, L = q.shape[0], k.shape[0]
    H, d = q.shape[1:]
    o = np.zeros((Lq, H, d))
    lse = np.full((H, Lq), -np.inf)
    if L == 0:
        return o, lse
    i = np.arange(Lq)[:, None]
    j = np.arange(L)[None, :]
    allowed = (j <= i + L - Lq) if causal else np.ones((Lq, L), dtype=bool)
    rows = allowed.any(axis=1)
    qt = torch.from_numpy(q).permute(1, 0, 2)[:, rows]
    kt = torch.from_numpy(k).permute(1, 0, 2)
    vt = torch.from_numpy(v).permute(1, 0, 2)
    mask = torch.from_numpy(allowed[rows])
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    o[rows] = out.permute(1, 0, 2).numpy()
    s = torch.matmul(qt, kt.transpose(1, 2)) * scale
    s = s.masked_fill(~mask, float("-inf"))
    lse[:, rows] = torch.logsumexp(s, dim=-1).numpy()
    return o, lse


CASES = [
    # Lq, causal, page_size, lens
    (1, False, 16, [37, 300, 16]),
    (4, True, 16, [37, 64, 5]),
    (3, True, 8, [2, 9, 24]),
    (2, False, 4, [0, 7, 12]),
]


@pytest.mark.parametrize("Lq,causal,page_size,lens", CASES)
def test_matches_sdpa_on_the_dense_sequences(Lq, causal, page_size, lens):
    H, d, scale = 2, 8, 0.4
    ks, vs = dense_requests(1, lens, H, d)
    q = np.random.default_rng(2).standard_normal((len(lens), Lq, H, d))
    kc, vc, table, seq_lens = scatter_to_pages(ks, vs, page_size, seed=3)
    o, lse = oracle.attn_fwd_paged(q, kc, vc, table, seq_lens, causal=causal, scale=scale)
    for b in range(len(lens)):
        exp_o, exp_lse = sdpa_dense(q[b], ks[b], vs[b], causal, scale)
        np.testing.assert_allclose(o[b], exp_o, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse[b], exp_lse, rtol=1e-12, atol=1e-13)
    assert np.abs(o).max() < 10.0  # no poison row was read


def test_page_size_and_placement_do_not_change_the_result():
    H, d, Lq = 2, 8, 3
    lens = [50, 129, 1]
    ks, vs = dense_requests(4, lens, H, d)
    q = np.random.default_rng(5).standard_normal((len(lens), Lq, H, d))
    ref = None
    for page_size, seed in [(1, 0), (4, 1), (16, 2), (16, 3), (64, 4), (256, 5)]:
        kc, vc, table, seq_lens = scatter_to_pages(ks, vs, page_size, seed=seed)
        got = oracle.attn_fwd_paged(q, kc, vc, table, seq_lens, causal=True, scale=0.3)
        if ref is None:
            ref = got
        else:
            np.testing.assert_array_equal(got[0], ref[0])
            np.testing.assert_array_equal(got[1], ref[1])


def test_single_query_ignores_the_causal_flag_and_empty_requests():
    H, d = 3, 4
    lens = [0, 20, 33]
    ks, vs = dense_requests(6, lens, H, d)
    q = np.random.default_rng(7).standard_normal((3, 1, H, d))
    kc, vc, table, seq_lens = scatter_to_pages(ks, vs, 8, seed=8)
    a = oracle.attn_fwd_paged(q, kc, vc, table, seq_lens, causal=False, scale=0.5)
    b = oracle.attn_fwd_paged(q, kc, vc, table, seq_lens, causal=True, scale=0.5)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    assert np.all(a[0][0] == 0.0) and np.all(a[1][0] == -np.inf)


def test_single_key_gives_its_value_row():
    H, d = 2, 5
    ks, vs = dense_requests(9, [1, 1], H, d)
    q = np.random.default_rng(10).standard_normal((2, 2, H, d))
    kc, vc, table, seq_lens = scatter_to_pages(ks, vs, 4, seed=11)
    o, lse = oracle.attn_fwd_paged(q, kc, vc, table, seq_lens, causal=False, scale=0.7)
    for b in range(2):
        for i in range(2):
            np.testing.assert_allclose(o[b, i], vs[b][0], rtol=1e-15)
            np.testing.assert_allclose(lse[b, :, i], 0.7 * (q[b, i] * ks[b][0]).sum(-1), rtol=1e-13)


def test_bad_metadata_is_rejected():
    H, d = 1, 4
    ks, vs = dense_requests(12, [9], H, d)
    q = np.zeros((1, 1, H, d))
    kc, vc, table, seq_lens = scatter_to_pages(ks, vs, 4, seed=13)
    bad = table.copy()
    bad[0, 2] = kc.shape[0]
    with pytest.raises(RuntimeError):
        oracle.attn_fwd_paged(q, kc, vc, bad, seq_lens)
    with pytest.raises(RuntimeError):
        oracle.attn_fwd_paged(q, kc, vc, table, np.array([13], dtype=np.int32))
