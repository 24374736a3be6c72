"""The FMA-pipe exponential of the softmax (exp2_poly.cuh) against its error bound, no GPU.

Part of the softmax exponentials are evaluated without the MUFU unit: Cody-Waite
range reduction 2^x = 2^j * 2^f (j = round(x), f in [-1/2, 1/2]) and a minimax
(Remez) cubic for 2^f whose fp32 coefficients live in the generated header
exp2_poly.cuh.  These tests check that the header is what its generator writes,
and that a bit-level fp32 model of the reduction, the Horner steps (one rounding
per fused multiply-add) and the exponent-field add stays within the header's
stated relative error, far below the half-ulp of the fp16/bf16 P it feeds.
"""
import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "attention_forward_tiled_b200", "csrc")
HEADER = os.path.join(CSRC, "exp2_poly.cuh")


def header_constants():
    text = open(HEADER).read()
    coeffs = [float(m) for _, m in sorted(
        (int(k), v) for k, v in re.findall(r"kExp2PolyC(\d) = ([0-9.eE+-]+)f;", text))]
    bound = float(re.search(r"kExp2PolyMaxRelErr = ([0-9.eE+-]+)f;", text).group(1))
    return [np.float32(c) for c in coeffs], bound


def fma32(a, b, c):
    """fp32 fused multiply-add: the fp32 product is exact in float64, one final rounding."""
    return (a.astype(np.float64) * b.astype(np.float64) + np.float64(c)).astype(np.float32)


def exp2_model(x):
    """The device routine step by step in fp32 (clamp, reduction, Horner, exponent add)."""
    coeffs, _ = header_constants()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)  # 1.5 * 2^23
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = fma32(np.full_like(f, coeffs[3]), f, coeffs[2])
    p = fma32(p, f, coeffs[1])
    p = fma32(p, f, coeffs[0])
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) % (1 << 32)
    return bits.astype(np.uint32).view(np.float32), x


def test_header_is_what_the_generator_writes():
    pytest.importorskip("mpmath")
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    c32, E, errs = fit.fit(3)
    assert fit.header_text(3, c32, E, errs) == open(HEADER).read()


def test_reduced_interval_error():
    coeffs, bound = header_constants()
    f = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    p = fma32(np.full_like(f, coeffs[3]), f, coeffs[2])
    p = fma32(p, f, coeffs[1])
    p = fma32(p, f, coeffs[0])
    err = np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    assert err.max() <= bound * 1.001
    assert err.max() > 0.5 * bound  # the bound is tight, not a loose overestimate


def test_whole_softmax_range():
    # softmax exponents lie in [-inf, 8] (8 = the lazy-rescale threshold); below -125 clamps
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-125.0, 8.0, 1_000_003), rng.uniform(-30.0, 8.0, 200_000),
                        np.arange(-125, 9, dtype=np.float64)]).astype(np.float32)
    y, xc = exp2_model(x)
    err = np.abs(y.astype(np.float64) / np.exp2(xc.astype(np.float64)) - 1.0)
    _, bound = header_constants()
    assert err.max() <= bound * 1.001
    assert np.all(np.isfinite(y)) and np.all(y > 0)
    # far below the relative half-ulp of the fp16 (2^-11) and bf16 (2^-8) P it is rounded to
    assert bound < 2.0 ** -11 / 6


def test_clamp_and_integer_points():
    y, _ = exp2_model(np.array([-1000.0, -126.0, -125.0, 0.0, 1.0, 8.0], dtype=np.float32))
    _, bound = header_constants()
    expect = np.exp2(np.array([-125.0, -125.0, -125.0, 0.0, 1.0, 8.0]))
    assert np.all(np.abs(y / expect - 1.0) <= bound * 1.001)
