"""Pins of the backward oracle (oracle.attn_bwd), no GPU.

Checked against things other than itself: central finite differences of the
(separately pinned) forward oracle, fp64 torch autograd through
scaled_dot_product_attention, and two sums fixed by the softmax: the key
gradients of a row sum to zero and the value gradients sum to the upstream
gradients of the rows that see a key.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def rnd(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("causal,Nq,Nk", [(False, 3, 4), (True, 4, 4), (True, 5, 3)])
def test_finite_differences_of_the_forward(causal, Nq, Nk):
    B, H, d, scale = 1, 2, 3, 0.7
    q, k, v, do = rnd(1, B, Nq, H, d), rnd(2, B, Nk, H, d), rnd(3, B, Nk, H, d), rnd(4, B, Nq, H, d)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, causal=causal, scale=scale)

    def loss(q_, k_, v_):
        o, _ = oracle.attn_fwd(q_, k_, v_, causal=causal, scale=scale)
        return float((o * do).sum())

    eps = 1e-6
    for x, g, slot in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p, args_m = [q, k, v], [q, k, v]
            args_p[slot], args_m[slot] = xp, xm
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        np.testing.assert_allclose(g, num, atol=1e-7, rtol=1e-6)


@pytest.mark.parametrize("causal,Nq,Nk", [(False, 7, 9), (True, 9, 9), (True, 6, 10)])
def test_matches_torch_autograd(causal, Nq, Nk):
    B, H, d = 2, 3, 16
    scale = 1 / math.sqrt(d)
    q, k, v, do = rnd(5, B, Nq, H, d), rnd(6, B, Nk, H, d), rnd(7, B, Nk, H, d), rnd(8, B, Nq, H, d)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, causal=causal, scale=scale)
    qt, kt, vt = (torch.tensor(x.transpose(0, 2, 1, 3), dtype=torch.float64, requires_grad=True)
                  for x in (q, k, v))
    mask = torch.zeros(Nq, Nk, dtype=torch.float64)
    if causal:
        allowed = torch.arange(Nk)[None, :] <= torch.arange(Nq)[:, None] + (Nk - Nq)
        mask = mask.masked_fill(~allowed, -math.inf)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    o.backward(torch.tensor(do.transpose(0, 2, 1, 3), dtype=torch.float64))
    for g, t in ((dq, qt), (dk, kt), (dv, vt)):
        np.testing.assert_allclose(g, t.grad.numpy().transpose(0, 2, 1, 3), atol=1e-12)


def test_softmax_sums():
    B, H, Nq, Nk, d = 1, 2, 6, 8, 4
    q, k, v, do = rnd(9, B, Nq, H, d), rnd(10, B, Nk, H, d), rnd(11, B, Nk, H, d), rnd(12, B, Nq, H, d)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, causal=True, scale=0.5)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)          # sum_j dS_ij = 0 per row
    np.testing.assert_allclose(dv.sum(axis=1), do.sum(axis=1), atol=1e-12)  # rows of P sum to 1
