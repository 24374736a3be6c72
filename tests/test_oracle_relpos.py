"""Pins of the relative-position-score oracle (oracle.attn_fwd_relpos), no GPU.

The term scale * q_i . emb[dist[i, j]] added to the scores (the Granite-Speech
attention of the vLLM page "PR #42933": einsum("bnhid,ijd->bnhij", q, rel_pos_emb)
* scale fed to SDPA with the scores) is pinned by things other than the oracle:
  * emb = 0: plain attention, fp64 torch SDPA;
  * every embedding row the same vector c: a per-row constant shift, so O is plain
    attention and lse grows by scale * q_i . c (softmax shift invariance);
  * emb = the keys, dist[i, j] = j: the term equals the key term, i.e. plain
    attention at twice the scale;
  * fp64 torch SDPA with an additive mask built by torch.einsum from emb[dist],
    causal masks included;
  * a 1 x 2 case worked by hand.
"""
import math

import numpy as np
import pytest
import torch

import oracle



def sdpa(q, k, v, scale, bias=None, causal=False):
    """fp64 torch reference: q, k, v [B, N, H, d] numpy; bias [B, H, Nq, Nk] or None."""
    qt, kt, vt = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    Nq, Nk = q.shape[1], k.shape[1]
    mask = torch.zeros(Nq, Nk, dtype=torch.float64)
    if causal:
        allowed = torch.arange(Nk)[None, :] <= torch.arange(Nq)[:, None] + (Nk - Nq)
        mask = mask.masked_fill(~allowed, -math.inf)
    if bias is not None:
        mask = mask + torch.from_numpy(bias)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    s = torch.einsum("bhid,bhjd->bhij", qt, kt) * scale + mask
    return o.permute(0, 2, 1, 3).numpy(), torch.logsumexp(s, dim=-1).numpy()


def rnd(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


def test_zero_embedding_is_plain_attention():
    q, k, v = rnd(1, 2, 7, 3, 16), rnd(2, 2, 9, 3, 16), rnd(3, 2, 9, 3, 16)
    dist = np.random.default_rng(4).integers(0, 5, size=(7, 9)).astype(np.int32)
    o, lse = oracle.attn_fwd_relpos(q, k, v, np.zeros((5, 16)), dist, scale=0.3)
    o_ref, lse_ref = sdpa(q, k, v, 0.3)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12)


def test_constant_embedding_shifts_lse_only():
    q, k, v = rnd(5, 1, 6, 2, 8), rnd(6, 1, 11, 2, 8), rnd(7, 1, 11, 2, 8)
    c = rnd(8, 8)
    emb = np.tile(c, (4, 1))
    dist = np.random.default_rng(9).integers(0, 4, size=(6, 11)).astype(np.int32)
    scale = 0.4
    o, lse = oracle.attn_fwd_relpos(q, k, v, emb, dist, causal=True, scale=scale)
    o_ref, lse_ref = sdpa(q, k, v, scale, causal=True)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    shift = scale * np.einsum("bihd,d->bhi", q, c)
    np.testing.assert_allclose(lse, lse_ref + shift, atol=1e-11)


def test_key_embedding_doubles_the_scale():
    q, k, v = rnd(10, 1, 5, 1, 8), rnd(11, 1, 7, 1, 8), rnd(12, 1, 7, 1, 8)
    emb = k[0, :, 0, :].copy()                            # one row per key
    dist = np.tile(np.arange(7, dtype=np.int32), (5, 1))  # dist[i, j] = j
    o, lse = oracle.attn_fwd_relpos(q, k, v, emb, dist, scale=0.25)
    o_ref, lse_ref = sdpa(q, k, v, 0.5)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12)


@pytest.mark.parametrize("causal,Nq,Nk", [(False, 9, 13), (True, 13, 13), (True, 6, 10)])
def test_matches_torch_with_einsum_bias(causal, Nq, Nk):
    B, H, d, R = 2, 3, 16, 4
    q, k, v = rnd(13, B, Nq, H, d), rnd(14, B, Nk, H, d), rnd(15, B, Nk, H, d)
    emb = rnd(16, 2 * R + 1, d)
    rel = np.arange(Nq)[:, None] + (Nk - Nq) - np.arange(Nk)[None, :]   # i - j, diagonal-aligned
    dist = (np.clip(rel, -R, R) + R).astype(np.int32)
    scale = 1 / math.sqrt(d)
    o, lse = oracle.attn_fwd_relpos(q, k, v, emb, dist, causal=causal, scale=scale)
    rel_pos_emb = torch.from_numpy(emb)[torch.from_numpy(dist).long()]          # [Nq, Nk, d]
    bias = torch.einsum("bihd,ijd->bhij", torch.from_numpy(q), rel_pos_emb) * scale
    o_ref, lse_ref = sdpa(q, k, v, scale, bias=bias.numpy(), causal=causal)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12)


def test_two_keys_by_hand():
    # one query q = (1, 0), keys (0, 0) and (1, 0), values 0 and 1, scale 1;
    # emb rows (2, 0) and (0, 0), dist = [[0, 1]]: scores 0 + 2 = 2 and 1 + 0 = 1
    q = np.array([1.0, 0.0]).reshape(1, 1, 1, 2)
    k = np.array([[0.0, 0.0], [1.0, 0.0]]).reshape(1, 2, 1, 2)
    v = np.array([[0.0, 0.0], [1.0, 1.0]]).reshape(1, 2, 1, 2)
    emb = np.array([[2.0, 0.0], [0.0, 0.0]])
    dist = np.array([[0, 1]], dtype=np.int32)
    o, lse = oracle.attn_fwd_relpos(q, k, v, emb, dist, scale=1.0)
    p1 = math.exp(1) / (math.exp(2) + math.exp(1))
    np.testing.assert_allclose(o.reshape(2), [p1, p1], atol=1e-15)
    np.testing.assert_allclose(lse.reshape(()), math.log(math.exp(2) + math.exp(1)), atol=1e-15)


def test_rejects_out_of_range_distance():
    q = rnd(17, 1, 2, 1, 4)
    with pytest.raises(RuntimeError):
        oracle.attn_fwd_relpos(q, q, q, np.zeros((2, 4)), np.array([[0, 2], [1, 0]], dtype=np.int32))
