"""GPU parity of the lightning-indexer score (attn_indexer_score, tensor cores) and of
the top-k selection (attn_topk) against the fp64 oracle.

Scores: the GPU accumulates q . kp in fp32 from fp16/bf16 inputs that the oracle reads
exactly, so each score may differ from the oracle by the fp32 rounding of the head
products and of the weighted head sum; the bound used is 2^-14 times the sum of the
magnitudes of the terms (sum_h |w_h| sum_c |q_hc kp_c|), about 16 times the worst-case
fp32 accumulation error of 128 + H terms.  Masked entries must be exactly -inf.

Top-k: an index result, compared bit for bit with the oracle run on the GPU's own fp32
scores (the same precision decides the order on both sides).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from attention_forward_tiled_b200 import get_status, indexer_score, topk
from attention_forward_tiled_b200.inputs import make_indexer_inputs

pytestmark = pytest.mark.gpu


def score_bound(q, kp, w):
    qa, ka, wa = q.double().abs(), kp.double().abs(), w.double().abs()
    mag = torch.einsum("bthc,bpc->bthp", qa, ka)            # sum_c |q_hc kp_c|
    return 2.0 ** -14 * torch.einsum("bth,bthp->btp", wa, mag).numpy() + 1e-30


CASES = [
    # (B, T, H, P, d, dtype, weights, masked)
    (1, 64, 4, 1000, 128, "f16", "random", True),
    (2, 33, 4, 257, 128, "bf16", "constant", True),
    (1, 5, 64, 700, 128, "f16", "random", False),
    (2, 130, 1, 384, 64, "f16", "random", True),
    (1, 40, 16, 129, 64, "bf16", "random", True),
    (1, 3, 128, 300, 128, "f16", "constant", False),
    # every head count's column grouping, with both mask paths (pool length a multiple of 8
    # or not) and a token tail in the last tile
    (1, 70, 2, 520, 128, "f16", "random", True),
    (1, 20, 8, 136, 64, "bf16", "random", True),
    (2, 9, 32, 264, 128, "f16", "random", True),
    (1, 6, 64, 1000, 128, "bf16", "random", True),
    (1, 3, 128, 77, 64, "f16", "random", True),
]


@pytest.mark.parametrize("B,T,H,P,d,dtype,weights,masked", CASES)
def test_indexer_score_matches_oracle(B, T, H, P, d, dtype, weights, masked):
    q, kp, w, mask = make_indexer_inputs(B, T, H, P, d, dtype=dtype, seed=T + P + H,
                                         weights=weights, masked=masked)
    out = indexer_score(q.cuda(), kp.cuda(), w.cuda(), mask.cuda() if mask is not None else None)
    torch.cuda.synchronize()
    assert get_status() == 0
    ref = oracle.indexer_score(q, kp, w, mask)
    got = out.double().cpu().numpy()
    fin = np.isfinite(ref)
    assert np.array_equal(np.isneginf(got), np.isneginf(ref)), "masked entries must be -inf"
    err = np.abs(got[fin] - ref[fin])
    bound = score_bound(q, kp, w)[fin]
    assert (err <= bound).all(), f"score error {float((err - bound).max())} beyond the fp32 bound"
    print(f"indexer B{B} T{T} H{H} P{P} d{d} {dtype}: max_abs={err.max():.2e} max_rel_to_bound="
          f"{float((err / bound).max()):.3f}")
    # the top-k of the GPU's scores, index for index
    k = min(64, P)
    idx = topk(out, k)
    torch.cuda.synchronize()
    assert get_status() == 0
    assert np.array_equal(idx.cpu().numpy(), oracle.topk(got, k))


def _rows_with_ties(R, P, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    s = torch.randint(-20, 20, (R, P), generator=g).float() / 4.0   # many equal values
    s[0, ::7] = float("-inf")
    s[1, ::5] = float("nan")
    s[2, 3:] = float("-inf")                                          # 3 finite entries only
    s[3, :] = float("-inf")                                           # nothing to choose
    s[4, 10] = float("inf")
    s[5, :] = -0.0
    s[5, 1::2] = 0.0                                                  # +0 and -0 tie
    return s


@pytest.mark.parametrize("R,P,k", [(8, 1000, 64), (8, 129, 200), (6, 60000, 2048), (6, 50000, 1),
                                   (7, 4096, 2048), (9, 513, 513)])
def test_topk_matches_oracle(R, P, k):
    s = _rows_with_ties(R, P, seed=R * P + k)
    idx = topk(s.cuda(), k)
    torch.cuda.synchronize()
    assert get_status() == 0
    assert np.array_equal(idx.cpu().numpy(), oracle.topk(s.double().numpy(), k))


def test_topk_distinct_scores_large_rows():
    """Random distinct scores: the chosen set is the k largest, in order (rows read from
    global memory on every pass when they exceed the shared-memory cache)."""
    g = torch.Generator("cpu").manual_seed(11)
    s = torch.randn(4, 70000, generator=g)
    idx = topk(s.cuda(), 300)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), oracle.topk(s.double().numpy(), 300))


def _rows_few_candidates(P, k, seed):
    """Rows whose k-th largest score falls in a radix bin of at most 32 keys after the
    second (or third) 8-bit digit, so the selection sorts those candidates in one warp:
    a background well below, `above` scores that are all chosen, and candidates that
    share the decided top digits (1 + m 2^-15 + j 2^-23 is exact in fp32)."""
    g = torch.Generator("cpu").manual_seed(seed)
    rows = []
    one = 1.0
    for above, cand in [
        (k - 1, [one + j * 2.0 ** -20 for j in range(20)]),                  # one of 20 distinct
        (k - 7, [one + j * 2.0 ** -20 for j in (5, 5, 5, 3, 3, 9, 1, 1, 0, 7, 7, 7, 2)]),
        (k - 32, [one + j * 2.0 ** -21 for j in range(32)]),                  # every candidate
        (k - 10, [one] * 16),                                                 # equal: by position
    ]:
        s = torch.randn(P, generator=g) * 0.1 - 4.0
        vals = torch.cat([2.0 + torch.rand(above, generator=g), torch.tensor(cand)])
        pos = torch.randperm(P, generator=g)[: vals.numel()]
        s[pos] = vals
        rows.append(s)
    # third digit: 100 keys share the top 16 bits; the k-th falls in a bin of 20 of them
    s = torch.randn(P, generator=g) * 0.1 - 4.0
    m_above = [one + m * 2.0 ** -15 for m in range(100 - (k - 11), 100)]   # k - 11 above
    m_below = [one + m * 2.0 ** -15 for m in range(0, 40)]
    cand = [one + 50 * 2.0 ** -15 + j * 2.0 ** -23 for j in (4, 4, 0, 19, 7, 7, 7, 3, 12, 12, 1, 5,
                                                             6, 8, 9, 10, 11, 13, 14, 15)]
    vals = torch.tensor(m_above + m_below + cand)
    pos = torch.randperm(P, generator=g)[: vals.numel()]
    s[pos] = vals
    rows.append(s)
    return torch.stack(rows).float()


@pytest.mark.parametrize("P", [5000, 60000])
def test_topk_few_candidates(P):
    """The selection's short path (<= 32 keys left after two or three digits), with ties
    among the candidates and on either side of the cut, from shared memory (P = 5000) and
    from global memory (P = 60000), against the oracle bit for bit."""
    k = 60
    s = _rows_few_candidates(P, k, seed=P)
    idx = topk(s.cuda(), k)
    torch.cuda.synchronize()
    assert get_status() == 0
    assert np.array_equal(idx.cpu().numpy(), oracle.topk(s.double().numpy(), k))
