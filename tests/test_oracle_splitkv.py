"""Pins of the split-KV oracle (oracle.attn_fwd_splitkv), the decode path's ordering, no GPU.

Cutting the keys into ranges, keeping (m, l, o) per range and combining them
must give the definition's result: checked against the (separately pinned)
definition-order oracle and against fp64 torch SDPA to 1e-12, on a two-key case
worked by hand, with empty ranges (more splits than keys, causal rows that see
few keys) and rows that see no key at all.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def rnd(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("Nq,Nk,causal,splits", [
    (1, 300, False, 1), (1, 300, False, 2), (1, 300, False, 7), (1, 37, False, 37),
    (1, 37, False, 50), (5, 64, True, 3), (9, 9, True, 4), (4, 2, True, 3), (3, 130, False, 8),
])
def test_agrees_with_the_definition(Nq, Nk, causal, splits):
    B, H, d, scale = 2, 3, 16, 0.3
    q, k, v = rnd(1, B, Nq, H, d), rnd(2, B, Nk, H, d) * 2.0, rnd(3, B, Nk, H, d)
    o, lse = oracle.attn_fwd_splitkv(q, k, v, splits, causal=causal, scale=scale)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, causal=causal, scale=scale)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


def test_agrees_with_torch_sdpa():
    B, H, Nk, d, scale = 2, 4, 517, 32, 1 / math.sqrt(32)
    q, k, v = rnd(4, B, 1, H, d), rnd(5, B, Nk, H, d), rnd(6, B, Nk, H, d)
    o, lse = oracle.attn_fwd_splitkv(q, k, v, 5, scale=scale)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=scale)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=1e-12, atol=1e-12)
    s = torch.matmul(tq, tk.transpose(-1, -2)) * scale
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), rtol=1e-12, atol=1e-12)


def test_two_keys_by_hand():
    # q = (1, 0), k0 = (1, 0), k1 = (3, 0), scale 1: scores 1 and 3, one key per split.
    # per split: m = s_j, l = 1, o = v_j; combine: M = 3, L = e^-2 + 1,
    # O = (e^-2 v0 + v1) / (e^-2 + 1), lse = 3 + ln(1 + e^-2)
    q = np.array([[[[1.0, 0.0]]]])
    k = np.array([[[[1.0, 0.0]], [[3.0, 0.0]]]])
    v = np.array([[[[2.0, -1.0]], [[4.0, 1.0]]]])
    o, lse = oracle.attn_fwd_splitkv(q, k, v, 2, scale=1.0)
    w0 = math.exp(-2.0) / (1.0 + math.exp(-2.0))
    np.testing.assert_allclose(o[0, 0, 0], [w0 * 2.0 + (1 - w0) * 4.0, -w0 + (1 - w0)], rtol=1e-15)
    np.testing.assert_allclose(lse[0, 0, 0], 3.0 + math.log1p(math.exp(-2.0)), rtol=1e-15)


def test_rows_without_keys():
    q, k, v = rnd(7, 1, 6, 2, 8), rnd(8, 1, 3, 2, 8), rnd(9, 1, 3, 2, 8)
    o, lse = oracle.attn_fwd_splitkv(q, k, v, 2, causal=True, scale=0.5)
    # bottom-right alignment: query i sees keys j <= i - 3, so rows 0..2 see none
    assert np.all(o[0, :3] == 0.0) and np.all(lse[0, :, :3] == -np.inf)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, causal=True, scale=0.5)
    np.testing.assert_allclose(o[0, 3:], o_ref[0, 3:], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse[0, :, 3:], lse_ref[0, :, 3:], rtol=1e-12, atol=1e-12)
