"""Tolerances and comparison helpers for GPU-vs-oracle parity.

Bounds (stated for the fused attention forward):
  fp16 O:  max |O_gpu - O_ref| <= 2e-3 and mean |O_gpu - O_ref| <= 2e-4 against the fp64 oracle.
  bf16 O:  the literal bound is out of reach of any bf16 result (an exactly
           computed O rounded once to bf16 already errs by up to 2^-8 |O|), so the
           pass criterion is taken against the oracle rounded once (RN-even) to
           bf16: per element |O_gpu - bf16(O_ref)| <= max(2e-3, one bf16 ulp of
           bf16(O_ref)), and mean |O_gpu - bf16(O_ref)| <= 2e-4.  The literal
           metrics against the unrounded oracle are still computed and reported.
  lse:     the relative bound 1e-3 is read as |lse_gpu - lse_ref| <= 1e-3 * max(|lse_ref|, 1)
           (a relative bound is ill-posed where lse is near 0); -inf must match exactly.
"""
import numpy as np
import torch

O_MAX_ABS = 2e-3
O_MEAN_ABS = 2e-4
LSE_REL = 1e-3


def _bf16_round(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()


def _bf16_ulp(x):
    """Spacing of bf16 at x (x already bf16-representable)."""
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    ulp = np.exp2(e - 7)
    return np.where(a >= 2.0 ** -126, ulp, 2.0 ** -133)


def o_errors(o_gpu, o_ref, dtype):
    """Returns dict of literal and criterion errors; o_gpu torch (any device), o_ref float64 numpy."""
    og = o_gpu.detach().double().cpu().numpy()
    lit = np.abs(og - o_ref)
    res = {"max_abs": float(lit.max()), "mean_abs": float(lit.mean())}
    if dtype == torch.bfloat16:
        rr = _bf16_round(o_ref)
        e = np.abs(og - rr)
        bound = np.maximum(O_MAX_ABS, _bf16_ulp(rr))
        res.update(crit_max_abs=float(e.max()), crit_mean_abs=float(e.mean()),
                   crit_excess=float((e - bound).max()))
    else:
        res.update(crit_max_abs=res["max_abs"], crit_mean_abs=res["mean_abs"],
                   crit_excess=float((lit - O_MAX_ABS).max()))
    return res


def assert_o_close(o_gpu, o_ref, dtype, what=""):
    r = o_errors(o_gpu, o_ref, dtype)
    assert np.isfinite(r["max_abs"]), f"{what}: non-finite output"
    assert r["crit_excess"] <= 0, f"{what}: O max error beyond bound: {r}"
    assert r["crit_mean_abs"] <= O_MEAN_ABS, f"{what}: O mean error beyond bound: {r}"
    return r


def assert_lse_close(lse_gpu, lse_ref, what=""):
    lg = lse_gpu.detach().double().cpu().numpy()
    ninf_ref = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lg), ninf_ref), f"{what}: -inf pattern of lse differs"
    f = ~ninf_ref
    if f.any():
        err = np.abs(lg[f] - lse_ref[f])
        bound = LSE_REL * np.maximum(np.abs(lse_ref[f]), 1.0)
        assert (err <= bound).all(), f"{what}: lse error {float((err - bound).max())} beyond bound"
        return float(err.max())
    return 0.0


def assert_convex_hull(out, v, causal, Nq, Nk):
    """Every O row is a convex combination of allowed V rows: per column, inside [min v, max v].

    A property that holds at any size, checked on the whole output (rows that see
    no key must be exactly zero).  Uses the full per-(b, h) V range, with an
    absolute slack of one 16-bit ulp of the bound.
    """
    vmin = v.float().amin(dim=1, keepdim=True)  # [B, 1, H, d]
    vmax = v.float().amax(dim=1, keepdim=True)
    o = out.float()
    slack = 4e-3 * torch.maximum(vmin.abs(), vmax.abs()).clamp_min(1.0)
    has_key = torch.ones(Nq, dtype=torch.bool, device=out.device)
    if causal and Nq > Nk:
        has_key[: Nq - Nk] = False
    hk = has_key.view(1, Nq, 1, 1)
    assert torch.isfinite(o).all(), "non-finite output"
    assert bool(((o >= vmin - slack) | ~hk).all()), "output below the V range"
    assert bool(((o <= vmax + slack) | ~hk).all()), "output above the V range"
    if (~has_key).any():
        assert bool((o[:, ~has_key] == 0).all()), "rows without keys must be zero"
