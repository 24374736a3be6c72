"""The GPU parity criteria themselves (tests/parity.py), checked on CPU tensors.

Every GPU parity test decides pass or fail through these helpers, so their
bounds are pinned here with hand-picked values on either side of each bound:
the fp16 max and mean bounds, the bf16 unit in the last place and the bf16
criterion built on it, the lse bound and its -inf pattern, and the convex-hull
property used at full size.
"""
import numpy as np
import pytest
import torch

from tests.parity import (_bf16_ulp, assert_convex_hull, assert_lse_close, assert_o_close,
                          o_errors)


def test_fp16_bounds():
    ref = np.zeros((1, 100, 1, 8))
    ok = torch.zeros(1, 100, 1, 8, dtype=torch.float16)
    ok[0, 0, 0, 0] = 1.9e-3                      # one element just inside the max bound
    assert_o_close(ok, ref, torch.float16)
    bad = ok.clone()
    bad[0, 0, 0, 0] = 2.2e-3                     # just outside (fp16 spacing here ~9.8e-7)
    with pytest.raises(AssertionError):
        assert_o_close(bad, ref, torch.float16)
    mean_bad = torch.full((1, 100, 1, 8), 2.5e-4, dtype=torch.float16)  # every element small, mean too big
    with pytest.raises(AssertionError):
        assert_o_close(mean_bad, ref, torch.float16)
    with pytest.raises(AssertionError):
        assert_o_close(torch.full((1, 1, 1, 8), float("nan"), dtype=torch.float16),
                       np.zeros((1, 1, 1, 8)), torch.float16)


def test_bf16_ulp():
    x = np.array([1.0, 1.5, 1.9921875, 2.0, 3.0, 0.75, 0.5, -4.0, 2.0 ** -126])
    want = np.array([2.0 ** -7, 2.0 ** -7, 2.0 ** -7, 2.0 ** -6, 2.0 ** -6, 2.0 ** -8, 2.0 ** -8,
                     2.0 ** -5, 2.0 ** -133])
    np.testing.assert_array_equal(_bf16_ulp(x), want)


def test_bf16_criterion_is_one_ulp_of_the_rounded_reference():
    n = 1000
    ref = np.full((1, n, 1, 1), 3.0001)          # rounds to 3.0 in bf16; ulp there is 2^-6
    gpu = torch.full((1, n, 1, 1), 3.0, dtype=torch.float64)
    gpu[0, 0] = 3.0 + 2.0 ** -6                  # one element one ulp away: allowed
    r = o_errors(gpu.to(torch.bfloat16), ref, torch.bfloat16)
    assert r["crit_excess"] <= 0 and r["max_abs"] > 2e-3   # the literal bound alone would fail
    assert_o_close(gpu.to(torch.bfloat16), ref, torch.bfloat16)
    gpu[0, 0] = 3.0 + 2.0 ** -5                  # two ulps: rejected
    with pytest.raises(AssertionError):
        assert_o_close(gpu.to(torch.bfloat16), ref, torch.bfloat16)


def test_lse_bound_and_neg_inf_pattern():
    ref = np.array([0.0, 0.5, 100.0, -np.inf])
    ok = torch.tensor([9e-4, 0.5 + 9e-4, 100.0 + 0.09, float("-inf")])
    assert_lse_close(ok, ref)
    for bad in ([1.1e-3, 0.5, 100.0, float("-inf")],      # absolute 1e-3 near zero
                [0.0, 0.5, 100.0 + 0.11, float("-inf")],  # relative 1e-3 at 100
                [0.0, 0.5, 100.0, -1e30]):                # -inf must stay -inf
        with pytest.raises(AssertionError):
            assert_lse_close(torch.tensor(bad), ref)


def test_convex_hull_property():
    v = torch.tensor([[[[0.0]], [[1.0]]]])       # B1, Nk 2, H1, d1: V range [0, 1]
    inside = torch.full((1, 3, 1, 1), 0.5)
    assert_convex_hull(inside, v, causal=False, Nq=3, Nk=2)
    with pytest.raises(AssertionError):
        assert_convex_hull(torch.full((1, 3, 1, 1), 1.1), v, causal=False, Nq=3, Nk=2)
    # causal with Nq > Nk: the first Nq - Nk rows see no key and must be exactly zero
    rows = torch.tensor([[[[0.0]], [[0.3]], [[0.7]]]])
    assert_convex_hull(rows, v, causal=True, Nq=3, Nk=2)
    rows[0, 0, 0, 0] = 0.2
    with pytest.raises(AssertionError):
        assert_convex_hull(rows, v, causal=True, Nq=3, Nk=2)
