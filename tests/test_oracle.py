"""Pins for the fp64 CPU oracle (no GPU).

Each test checks the oracle against something other than itself: closed forms
derived by hand (tests/golden), invariants the softmax definition fixes, special
cases that reduce to a textbook or library routine, and the blocked online
ordering the FlashAttention article describes ("FlashAttention的核心逻辑").
A plausible slip in the oracle -- a dropped scale, a wrong mask corner or sign,
a transposed operand, a missing max-subtraction term -- fails at least one of
them (test_oracle_mutants.py plants such slips and checks exactly that).
"""
import glob
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from attention_forward_tiled_b200.inputs import make_inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _ev(expr):
    """Evaluate a golden-fixture number: rationals, log(...), inf only."""
    env = {"__builtins__": {}, "log": math.log, "inf": math.inf}
    if "log" in expr or "inf" in expr:
        return float(eval(expr, env))  # noqa: S307 - fixed, committed fixtures
    return float(Fraction(expr))


def _arr(nested):
    return np.vectorize(_ev, otypes=[np.float64])(np.array(nested, dtype=object))


def rand(B, H, Nq, Nk, d, seed, dtype="f16", k_mult=1.0):
    q, k, v = make_inputs(B, H, Nq, Nk, d, dtype=dtype, seed=seed, k_mult=k_mult)
    return q.double().numpy(), k.double().numpy(), v.double().numpy()


# --------------------------------------------------------------------------
# hand-derived closed forms
# --------------------------------------------------------------------------
GOLDEN_FILES = sorted(glob.glob(os.path.join(GOLDEN, "*.json")))


@pytest.mark.parametrize("path", GOLDEN_FILES, ids=[os.path.basename(p) for p in GOLDEN_FILES])
@pytest.mark.parametrize("fn", ["naive", "blocked"])
def test_golden_closed_forms(path, fn):
    fx = json.load(open(path))
    q, k, v = _arr(fx["q"]), _arr(fx["k"]), _arr(fx["v"])
    assert q.shape == (fx["B"], fx["Nq"], fx["H"], fx["d"])
    assert k.shape == (fx["B"], fx["Nk"], fx["H"], fx["d"]) == v.shape
    scale = _ev(fx["scale"])
    for case in fx["cases"]:
        if fn == "naive":
            o, lse = oracle.attn_fwd(q, k, v, causal=case["causal"], scale=scale)
        else:
            o, lse = oracle.attn_fwd_blocked(q, k, v, causal=case["causal"], scale=scale,
                                             block_m=2, block_n=2)
        np.testing.assert_allclose(o, _arr(case["o"]), rtol=0, atol=1e-12)
        exp_lse = _arr(case["lse"])
        assert np.array_equal(np.isneginf(lse), np.isneginf(exp_lse))
        fin = np.isfinite(exp_lse)
        np.testing.assert_allclose(lse[fin], exp_lse[fin], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# invariants and special cases named by the workload description
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal,Nq,Nk", [(False, 7, 11), (True, 9, 9), (True, 5, 12), (True, 12, 5)])
def test_probability_rows_sum_to_one_and_mask(causal, Nq, Nk):
    q, k, v = rand(2, 3, Nq, Nk, 16, seed=11)
    p = oracle.attn_probs(q, k, causal=causal, scale=0.37)
    assert (p >= 0).all()
    i = np.arange(Nq)[:, None]
    j = np.arange(Nk)[None, :]
    allowed = (j <= i + (Nk - Nq)) if causal else np.ones((Nq, Nk), bool)
    assert (p[..., ~allowed] == 0).all()
    sums = p.sum(-1)
    has_key = allowed.any(-1)
    np.testing.assert_allclose(sums[..., has_key], 1.0, rtol=0, atol=1e-14)
    assert (sums[..., ~has_key] == 0).all()
    # the probabilities reproduce O = P V and the ratio of two allowed entries is exp(s_a - s_b)
    o, _ = oracle.attn_fwd(q, k, v, causal=causal, scale=0.37)
    o_pv = np.einsum("bhij,bjhd->bihd", p, v)
    np.testing.assert_allclose(o, o_pv, rtol=0, atol=1e-12)
    ii, jj = np.argwhere(allowed)[0]
    ii2, jj2 = ii, np.argwhere(allowed[ii])[-1][0]
    s1 = 0.37 * q[0, ii, 0] @ k[0, jj, 0]
    s2 = 0.37 * q[0, ii2, 0] @ k[0, jj2, 0]
    assert math.isclose(p[0, 0, ii, jj] / p[0, 0, ii2, jj2], math.exp(s1 - s2), rel_tol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_gives_that_constant(causal):
    q, k, v = rand(2, 2, 33, 33, 8, seed=12)
    c = np.linspace(-3, 3, 8)
    v[:] = c
    o, _ = oracle.attn_fwd(q, k, v, causal=causal, scale=0.5)
    np.testing.assert_allclose(o, np.broadcast_to(c, o.shape), rtol=0, atol=1e-13)


def test_single_key_gives_v0():
    q, k, v = rand(2, 3, 17, 1, 32, seed=13)
    scale = 0.125
    o, lse = oracle.attn_fwd(q, k, v, causal=False, scale=scale)
    np.testing.assert_array_equal(o, np.broadcast_to(v[:, 0:1], o.shape))
    # softmax of one score is 1, so lse is that single score
    s = scale * np.einsum("bihd,bhd->bhi", q, k[:, 0])
    np.testing.assert_allclose(lse, s, rtol=0, atol=1e-13)


def test_causal_first_query_gives_v0():
    q, k, v = rand(2, 2, 40, 40, 16, seed=14)
    o, lse = oracle.attn_fwd(q, k, v, causal=True, scale=0.25)
    np.testing.assert_array_equal(o[:, 0], v[:, 0])
    np.testing.assert_allclose(lse[:, :, 0], 0.25 * np.einsum("bhd,bhd->bh", q[:, 0], k[:, 0]),
                               rtol=0, atol=1e-13)
    # and the last query of a square causal problem sees every key: equals non-causal
    o_nc, lse_nc = oracle.attn_fwd(q, k, v, causal=False, scale=0.25)
    np.testing.assert_allclose(o[:, -1], o_nc[:, -1], rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[:, :, -1], lse_nc[:, :, -1], rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal,Nq,Nk", [(False, 200, 200), (True, 200, 200), (True, 65, 130),
                                          (False, 129, 63), (True, 130, 70)])
@pytest.mark.parametrize("bm,bn", [(128, 64), (64, 128), (7, 5)])
def test_naive_and_blocked_orderings_agree(causal, Nq, Nk, bm, bn):
    q, k, v = rand(1, 2, Nq, Nk, 32, seed=15, k_mult=3.0)
    o1, l1 = oracle.attn_fwd(q, k, v, causal=causal, scale=0.3)
    o2, l2 = oracle.attn_fwd_blocked(q, k, v, causal=causal, scale=0.3, block_m=bm, block_n=bn)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    assert np.array_equal(np.isneginf(l1), np.isneginf(l2))
    f = np.isfinite(l1)
    np.testing.assert_allclose(l1[f], l2[f], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal,Nq,Nk", [(False, 9, 13), (True, 9, 13), (True, 13, 9)])
def test_scale_zero_gives_mean_of_allowed_v(causal, Nq, Nk):
    q, k, v = rand(1, 2, Nq, Nk, 4, seed=16)
    o, lse = oracle.attn_fwd(q, k, v, causal=causal, scale=0.0)
    for i in range(Nq):
        n = Nk if not causal else max(0, min(Nk, i + (Nk - Nq) + 1))
        if n == 0:
            assert (o[:, i] == 0).all() and np.isneginf(lse[:, :, i]).all()
        else:
            np.testing.assert_allclose(o[:, i], v[:, :n].mean(1), rtol=0, atol=1e-13)
            np.testing.assert_allclose(lse[:, :, i], math.log(n), rtol=0, atol=1e-13)


def test_joint_key_value_permutation_invariance():
    q, k, v = rand(2, 2, 21, 37, 16, seed=17)
    perm = np.random.default_rng(0).permutation(37)
    o1, l1 = oracle.attn_fwd(q, k, v, causal=False, scale=0.4)
    o2, l2 = oracle.attn_fwd(q, k[:, perm], v[:, perm], causal=False, scale=0.4)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_row_shift_of_scores(causal):
    """Adding u to every key adds scale*q_i.u to row i: O unchanged, lse shifted."""
    q, k, v = rand(1, 2, 19, 19, 8, seed=18)
    u = np.linspace(-1, 2, 8)
    o1, l1 = oracle.attn_fwd(q, k, v, causal=causal, scale=0.7)
    o2, l2 = oracle.attn_fwd(q, k + u, v, causal=causal, scale=0.7)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    shift = 0.7 * np.einsum("bihd,d->bhi", q, u)
    np.testing.assert_allclose(l2 - l1, shift, rtol=0, atol=1e-12)


def test_linear_in_v():
    q, k, v1 = rand(1, 2, 23, 29, 8, seed=19)
    v2 = rand(1, 2, 23, 29, 8, seed=20)[2]
    o1, _ = oracle.attn_fwd(q, k, v1, causal=True, scale=0.5)
    o2, _ = oracle.attn_fwd(q, k, v2, causal=True, scale=0.5)
    o3, _ = oracle.attn_fwd(q, k, 2.0 * v1 - 3.0 * v2, causal=True, scale=0.5)
    np.testing.assert_allclose(o3, 2.0 * o1 - 3.0 * o2, rtol=0, atol=1e-12)


def test_heads_and_batches_are_independent():
    q, k, v = rand(3, 4, 11, 14, 8, seed=21)
    o, lse = oracle.attn_fwd(q, k, v, causal=True, scale=0.6)
    for b in range(3):
        for h in range(4):
            ob, lb = oracle.attn_fwd(q[b:b + 1, :, h:h + 1], k[b:b + 1, :, h:h + 1],
                                     v[b:b + 1, :, h:h + 1], causal=True, scale=0.6)
            np.testing.assert_array_equal(o[b:b + 1, :, h:h + 1], ob)
            np.testing.assert_array_equal(lse[b:b + 1, h:h + 1], lb)


@pytest.mark.parametrize("causal,Nq,Nk", [(False, 24, 40), (True, 32, 32), (True, 16, 48), (True, 48, 16)])
def test_against_torch_sdpa_fp64(causal, Nq, Nk):
    """Library special case: torch's fp64 CPU SDPA with an explicit bottom-right mask."""
    q, k, v = rand(2, 3, Nq, Nk, 16, seed=22)
    scale = 0.21
    o, lse = oracle.attn_fwd(q, k, v, causal=causal, scale=scale)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    i = torch.arange(Nq)[:, None]
    j = torch.arange(Nk)[None, :]
    mask = (j <= i + (Nk - Nq)) if causal else torch.ones(Nq, Nk, dtype=torch.bool)
    has_key = mask.any(-1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=mask, scale=scale).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(o[:, has_key.numpy()], ref[:, has_key.numpy()], rtol=0, atol=1e-12)
    s = torch.einsum("bhid,bhjd->bhij", tq, tk) * scale
    ref_lse = torch.logsumexp(s.masked_fill(~mask, -math.inf), -1).numpy()
    np.testing.assert_allclose(lse[..., has_key.numpy()], ref_lse[..., has_key.numpy()],
                               rtol=0, atol=1e-12)
    assert np.isneginf(lse[..., ~has_key.numpy()]).all()
    assert (o[:, ~has_key.numpy()] == 0).all()


def test_bottom_right_equals_top_left_when_square():
    q, k, v = rand(1, 2, 30, 30, 8, seed=23)
    o, _ = oracle.attn_fwd(q, k, v, causal=True, scale=0.3)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=0.3)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


def test_large_logits_do_not_overflow():
    """K x 3 with a big scale: the max subtraction keeps every exp finite."""
    q, k, v = rand(1, 1, 16, 64, 64, seed=24, dtype="bf16", k_mult=3.0)
    o, lse = oracle.attn_fwd(q, k, v, causal=False, scale=40.0)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    # with such a scale the softmax is (almost) a one-hot on the largest score
    s = 40.0 * np.einsum("bihd,bjhd->bhij", q, k)
    top = s.argmax(-1)[0, 0]
    gap = np.sort(s[0, 0], -1)[:, -1] - np.sort(s[0, 0], -1)[:, -2]
    sharp = gap > 60
    np.testing.assert_allclose(o[0, sharp, 0], v[0, top[sharp], 0], rtol=0, atol=1e-12)


def test_rejects_bad_shapes():
    q, k, v = rand(1, 1, 4, 4, 4, seed=25)
    with pytest.raises(ValueError):
        oracle.attn_fwd(q, k[:, :, :, :2], v, causal=False, scale=1.0)
