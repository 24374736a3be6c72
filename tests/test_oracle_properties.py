"""Property tests of the forward oracles over random small shapes (hypothesis), no GPU.

For random batch, heads, lengths (including Nq > Nk and Nk = 1), head dims,
scales, causal flags, block sizes and split counts:
- the definition order, the blocked online order and the split-KV order agree to 1e-12;
- rows of P sum to 1 over the allowed keys and are 0 elsewhere;
- each output lies in the convex hull of the value rows its query may see;
- max_j s_ij <= lse_i <= max_j s_ij + ln(number of allowed keys);
- a row with no allowed key gives O = 0 and lse = -inf.
The example sequence is fixed (derandomised), so a failure reproduces.
"""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle

SETTINGS = settings(max_examples=60, deadline=None, derandomize=True, database=None,
                    suppress_health_check=[HealthCheck.too_slow])


@st.composite
def problems(draw):
    B = draw(st.integers(1, 2))
    H = draw(st.integers(1, 3))
    Nq = draw(st.integers(1, 40))
    Nk = draw(st.integers(1, 40))
    d = draw(st.sampled_from([1, 2, 3, 8, 16]))
    causal = draw(st.booleans())
    scale = draw(st.sampled_from([0.0, 0.05, 0.3, 1.0, -0.7, 2.5]))
    seed = draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Nq, H, d))
    k = rng.standard_normal((B, Nk, H, d)) * draw(st.sampled_from([0.5, 1.0, 4.0]))
    v = rng.standard_normal((B, Nk, H, d))
    return dict(q=q, k=k, v=v, causal=causal, scale=scale,
                block_m=draw(st.integers(1, 48)), block_n=draw(st.integers(1, 48)),
                splits=draw(st.integers(1, 45)))


def allowed_mask(Nq, Nk, causal):
    i = np.arange(Nq)[:, None]
    j = np.arange(Nk)[None, :]
    return (j <= i + Nk - Nq) if causal else np.ones((Nq, Nk), dtype=bool)


@SETTINGS
@given(problems())
def test_three_orderings_agree(p):
    o, lse = oracle.attn_fwd(p["q"], p["k"], p["v"], causal=p["causal"], scale=p["scale"])
    ob, lseb = oracle.attn_fwd_blocked(p["q"], p["k"], p["v"], causal=p["causal"], scale=p["scale"],
                                       block_m=p["block_m"], block_n=p["block_n"])
    os_, lses = oracle.attn_fwd_splitkv(p["q"], p["k"], p["v"], p["splits"], causal=p["causal"],
                                        scale=p["scale"])
    for other_o, other_lse in ((ob, lseb), (os_, lses)):
        np.testing.assert_allclose(other_o, o, rtol=1e-12, atol=1e-12)
        np.testing.assert_array_equal(np.isneginf(other_lse), np.isneginf(lse))
        fin = np.isfinite(lse)
        np.testing.assert_allclose(other_lse[fin], lse[fin], rtol=1e-12, atol=1e-12)


@SETTINGS
@given(problems())
def test_probabilities_hull_and_lse_bounds(p):
    q, k, v = p["q"], p["k"], p["v"]
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    mask = allowed_mask(Nq, Nk, p["causal"])
    n_allowed = mask.sum(axis=1)
    probs = oracle.attn_probs(q, k, causal=p["causal"], scale=p["scale"])
    o, lse = oracle.attn_fwd(q, k, v, causal=p["causal"], scale=p["scale"])
    scores = p["scale"] * np.einsum("bihd,bjhd->bhij", q, k)
    for b in range(B):
        for h in range(H):
            P = probs[b, h]
            assert np.all(P[~mask] == 0.0) and np.all(P >= 0.0)
            sums = P.sum(axis=1)
            np.testing.assert_allclose(sums[n_allowed > 0], 1.0, rtol=0, atol=1e-12)
            assert np.all(sums[n_allowed == 0] == 0.0)
            for i in range(Nq):
                if n_allowed[i] == 0:
                    assert np.all(o[b, i, h] == 0.0) and lse[b, h, i] == -np.inf
                    continue
                vis = v[b, mask[i], h]
                assert np.all(o[b, i, h] >= vis.min(axis=0) - 1e-12)
                assert np.all(o[b, i, h] <= vis.max(axis=0) + 1e-12)
                smax = scores[b, h, i, mask[i]].max()
                assert smax - 1e-12 <= lse[b, h, i] <= smax + np.log(n_allowed[i]) + 1e-12
