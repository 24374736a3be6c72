"""GPU parity of the backward pass (attn_bwd, tensor cores) against the fp64 oracle.

The GPU computes the gradients from its own forward's O and lse, as a training step
does.  Its arithmetic differs from the exact gradients by three roundings: P and dS
are rounded to the input type (relative u: 2^-11 for fp16, 2^-8 for bf16) before
they multiply on the tensor cores; D_i = sum_t dO_it O_it uses the forward's O,
rounded to the input type (relative u per element); everything else accumulates in
fp32.  Per element that gives
  |ddV_kt| <= u sum_q P_qk |dO_qt|
  |ddS_qk| <= E_qk = u |dS_qk| + P_qk u sum_t |dO_qt| |O_qt|
  |ddK_kt| <= scale sum_q E_qk |Q_qt|,   |ddQ_qt| <= scale sum_k E_qk |K_kt|
plus fp32 accumulation, covered by 2^-14 times the same sums of magnitudes.  The
test asserts twice this bound (the first-order terms add up to their bound only when
every rounding has the same sign) and prints the literal max errors.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from attention_forward_tiled_b200 import attn_bwd, attn_fwd, get_status
from attention_forward_tiled_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

U = {"f16": 2.0 ** -11, "bf16": 2.0 ** -8}
# the stored gradient's own rounding below the type's normal range is absolute: half the
# subnormal spacing (fp16: 2^-24; bf16 keeps fp32's exponent range)
SUB = {"f16": 2.0 ** -25, "bf16": 2.0 ** -134}


def bounds(q, k, v, dout, causal, scale, u):
    """Per-element error bounds of dq, dk, dv in [B, N, H, d] layout (fp64 numpy)."""
    P = torch.from_numpy(oracle.attn_probs(q, k, causal=causal, scale=scale))  # [B, H, Nq, Nk]
    o_ref, _ = oracle.attn_fwd(q, k, v, causal=causal, scale=scale)
    qd, kd, vd, gd = (t.double() for t in (q, k, v, dout))
    od = torch.from_numpy(o_ref)
    dP = torch.einsum("bqhd,bkhd->bhqk", gd, vd)
    D = (P * dP).sum(-1, keepdim=True)
    dS = P * (dP - D)
    dOO = torch.einsum("bqhd,bqhd->bhq", gd.abs(), od.abs()).unsqueeze(-1)
    E = u * dS.abs() + P * u * dOO
    g = 2.0 ** -14
    b_dv = torch.einsum("bhqk,bqhd->bkhd", P, gd.abs()) * (u + g)
    b_dk = scale * (torch.einsum("bhqk,bqhd->bkhd", E, qd.abs())
                    + g * torch.einsum("bhqk,bqhd->bkhd", dS.abs(), qd.abs()))
    b_dq = scale * (torch.einsum("bhqk,bkhd->bqhd", E, kd.abs())
                    + g * torch.einsum("bhqk,bkhd->bqhd", dS.abs(), kd.abs()))
    return b_dq.numpy(), b_dk.numpy(), b_dv.numpy()


CASES = [
    # (B, H, Nq, Nk, d, dtype, causal)
    (1, 2, 128, 128, 64, "f16", False),
    (1, 2, 256, 256, 128, "f16", True),
    (2, 3, 200, 300, 128, "bf16", True),    # Nq < Nk: bottom-right diagonal
    (1, 2, 300, 200, 64, "f16", True),      # Nq > Nk: leading query rows see no key
    (1, 1, 64, 1000, 128, "f16", False),
    (1, 2, 129, 65, 64, "bf16", False),     # ragged tiles in both directions
    (2, 2, 384, 384, 128, "bf16", True),
]


@pytest.mark.parametrize("B,H,Nq,Nk,d,dtype,causal", CASES)
def test_backward_matches_oracle(B, H, Nq, Nk, d, dtype, causal):
    q, k, v = make_inputs(B, H, Nq, Nk, d, dtype=dtype, seed=Nq + 7 * Nk + d)
    g = torch.Generator("cpu").manual_seed(Nq * Nk)
    dout = torch.randn(B, Nq, H, d, generator=g).to(q.dtype)
    scale = 1.0 / math.sqrt(d)
    qd, kd, vd, gd = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, lse = attn_fwd(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = attn_bwd(qd, kd, vd, o, lse, gd, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert get_status() == 0
    ref = oracle.attn_bwd(q, k, v, dout, causal=causal, scale=scale)
    bnd = bounds(q, k, v, dout, causal, scale, U[dtype])
    for name, got, r, bd in zip(("dq", "dk", "dv"), (dq, dk, dv), ref, bnd):
        gn = got.double().cpu().numpy()
        err = np.abs(gn - r)
        # the result is stored in the input type: add its own rounding
        lim = 2 * bd + 0.5 * U[dtype] * 2 * np.abs(r) + SUB[dtype] + 1e-12
        assert np.isfinite(gn).all(), name
        assert (err <= lim).all(), f"{name}: error beyond bound by {float((err - lim).max()):.3e}"
        print(f"bwd {B}x{H}x{Nq}x{Nk}x{d} {dtype} causal={causal} {name}: max_abs={err.max():.2e} "
              f"max_ref={np.abs(r).max():.2e} worst_frac_of_bound={float((err / lim).max()):.3f}")
