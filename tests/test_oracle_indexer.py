"""Pins of the lightning-indexer oracle (oracle.indexer_score, oracle.topk), no GPU.

Checked against things other than itself: a two-token example worked by hand,
the special case that reduces to a plain matrix product (one head, unit weight,
non-negative inputs), properties the rectified sum must have (odd part linear,
additive over heads, positively homogeneous, invariant under a joint head
permutation), and, for top-k, numpy's stable argsort on rows with ties and
-inf entries.
"""
import numpy as np
import pytest

import oracle

NEG = -np.inf


def rnd(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


def hand_case():
    # token 0 heads: (1, 2), (-1, 0.5); token 1 heads: (1, 2), (1, 0.5)
    q = np.array([[[[1.0, 2.0], [-1.0, 0.5]],
                   [[1.0, 2.0], [1.0, 0.5]]]])
    kp = np.array([[[1.0, 1.0], [2.0, -0.5]]])
    w = np.array([[[0.5, 2.0], [0.25, 3.0]]])
    return q, kp, w


def test_hand_worked_example():
    q, kp, w = hand_case()
    # dot products (token, head, key): t0: h0 (3, 1), h1 (-0.5, -2.25); t1: h0 (3, 1), h1 (1.5, 1.75)
    # t0: key0 = 0.5*3 + 2*0 = 1.5, key1 = 0.5*1 + 2*0 = 0.5
    # t1: key0 = 0.25*3 + 3*1.5 = 5.25, key1 = 0.25*1 + 3*1.75 = 5.5
    expect = np.array([[[1.5, 0.5], [5.25, 5.5]]])
    np.testing.assert_array_equal(oracle.indexer_score(q, kp, w), expect)
    mask = np.array([[[0.0, NEG], [-1.0, 0.0]]])
    np.testing.assert_array_equal(oracle.indexer_score(q, kp, w, mask),
                                  np.array([[[1.5, NEG], [4.25, 5.5]]]))


def test_single_head_nonnegative_is_a_matrix_product():
    rng = np.random.default_rng(7)
    B, T, P, d = 2, 5, 7, 8
    q = rng.uniform(0.0, 1.0, (B, T, 1, d))
    kp = rng.uniform(0.0, 1.0, (B, P, d))
    got = oracle.indexer_score(q, kp, np.ones((B, T, 1)))
    np.testing.assert_allclose(got, np.matmul(q[:, :, 0, :], kp.transpose(0, 2, 1)), rtol=1e-12, atol=1e-15)
    mask = rng.uniform(-2.0, 0.0, (B, T, P))
    got = oracle.indexer_score(q, kp, np.full((B, T, 1), 0.125), mask)
    np.testing.assert_allclose(got, 0.125 * np.matmul(q[:, :, 0, :], kp.transpose(0, 2, 1)) + mask,
                               rtol=1e-12, atol=1e-15)


def test_all_heads_negative_gives_the_mask():
    rng = np.random.default_rng(8)
    B, T, H, P, d = 1, 3, 4, 6, 5
    q = -rng.uniform(0.1, 1.0, (B, T, H, d))
    kp = rng.uniform(0.1, 1.0, (B, P, d))
    mask = rng.uniform(-1.0, 0.0, (B, T, P))
    np.testing.assert_array_equal(oracle.indexer_score(q, kp, rnd(9, B, T, H) ** 2, mask), mask)


def test_odd_part_is_linear():
    # relu(x) - relu(-x) = x, so score(q) - score(-q) = sum_h w_h (q_h . k)
    B, T, H, P, d = 2, 4, 3, 5, 6
    q, kp, w = rnd(10, B, T, H, d), rnd(11, B, P, d), rnd(12, B, T, H)
    diff = oracle.indexer_score(q, kp, w) - oracle.indexer_score(-q, kp, w)
    lin = np.matmul(q.reshape(B, T * H, d), kp.transpose(0, 2, 1)).reshape(B, T, H, P)
    np.testing.assert_allclose(diff, (lin * w[..., None]).sum(axis=2), rtol=1e-12, atol=1e-12)


def test_additive_over_heads():
    B, T, H, P, d = 1, 3, 4, 5, 6
    q, kp, w = rnd(13, B, T, H, d), rnd(14, B, P, d), rnd(15, B, T, H)
    parts = sum(oracle.indexer_score(q[:, :, h:h + 1], kp, w[:, :, h:h + 1]) for h in range(H))
    np.testing.assert_allclose(oracle.indexer_score(q, kp, w), parts, rtol=1e-12, atol=1e-12)


def test_homogeneity_and_head_permutation():
    B, T, H, P, d = 2, 3, 5, 4, 6
    q, kp, w = rnd(16, B, T, H, d), rnd(17, B, P, d), rnd(18, B, T, H)
    base = oracle.indexer_score(q, kp, w)
    np.testing.assert_allclose(oracle.indexer_score(2.5 * q, kp, w), 2.5 * base, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.indexer_score(q, 0.5 * kp, w), 0.5 * base, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.indexer_score(q, kp, -3.0 * w), -3.0 * base, rtol=1e-12, atol=1e-12)
    perm = np.array([3, 0, 4, 1, 2])
    np.testing.assert_allclose(oracle.indexer_score(q[:, :, perm], kp, w[:, :, perm]), base,
                               rtol=1e-12, atol=1e-12)


def test_unweighted_variant():
    # the report's unweighted sum scaled by 1/sqrt(d) is every head weight = 1/sqrt(d)
    B, T, H, P, d = 1, 2, 4, 3, 16
    q, kp = rnd(19, B, T, H, d), rnd(20, B, P, d)
    unit = oracle.indexer_score(q, kp, np.ones((B, T, H)))
    np.testing.assert_allclose(oracle.indexer_score(q, kp, np.full((B, T, H), 0.25)), unit / np.sqrt(d),
                               rtol=1e-12, atol=1e-15)


def test_topk_hand_cases():
    row = np.array([[1.0, 3.0, 3.0, NEG, 2.0]])
    np.testing.assert_array_equal(oracle.topk(row, 4), [[1, 2, 4, 0]])
    np.testing.assert_array_equal(oracle.topk(row, 6), [[1, 2, 4, 0, -1, -1]])
    np.testing.assert_array_equal(oracle.topk(np.full((2, 3), NEG), 2), [[-1, -1], [-1, -1]])
    np.testing.assert_array_equal(oracle.topk(np.array([[np.nan, 0.5, np.nan]]), 2), [[1, -1]])


@pytest.mark.parametrize("k", [1, 5, 17, 40])
def test_topk_matches_stable_argsort(k):
    rng = np.random.default_rng(21)
    R, P = 9, 33
    s = np.round(rng.standard_normal((R, P)) * 2.0) / 2.0  # many ties
    s[rng.uniform(size=(R, P)) < 0.2] = NEG
    got = oracle.topk(s, k)
    for r in range(R):
        order = [int(j) for j in np.argsort(-s[r], kind="stable") if np.isfinite(s[r, j])][:k]
        np.testing.assert_array_equal(got[r], order + [-1] * (k - len(order)))


def test_topk_order_ignores_the_weight_scale():
    # the decode-side indexer drops the softmax scale because only the order is used
    B, T, H, P, d = 1, 4, 4, 64, 16
    q, kp, w = rnd(22, B, T, H, d), rnd(23, B, P, d), np.abs(rnd(24, B, T, H))
    a = oracle.topk(oracle.indexer_score(q, kp, w), 8)
    b = oracle.topk(oracle.indexer_score(q, kp, 0.125 * w), 8)
    np.testing.assert_array_equal(a, b)
