"""GPU parity of attention with the fused relative-position term (attn_fwd_relpos) against
the fp64 oracle (oracle.attn_fwd_relpos, which takes the distance table written out).

The kernel forms the term q_i . emb[dist(i, j)] on the tensor cores per tile (fp16/bf16
inputs, fp32 accumulation) and adds it to q_i . k_j before the scale, the mask and the
softmax; the output is held to the same criteria as attn_fwd (tests/parity.py): the term
only shifts the scores, and P V runs the same way.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from attention_forward_tiled_b200 import ATTN_ERR_RANGE, attn_fwd_relpos, get_status
from attention_forward_tiled_b200.inputs import RELPOS_WORKLOADS, make_relpos_inputs
from parity import assert_lse_close, assert_o_close

pytestmark = pytest.mark.gpu


def clamped_dist(Nq, Nk, R):
    """The conformer's table: clamp(i - j, -R, R) + R."""
    i = np.arange(Nq).reshape(Nq, 1)
    j = np.arange(Nk).reshape(1, Nk)
    return (np.clip(i - j, -R, R) + R).astype(np.int32)


CASES = [
    # (B, H, Nq, Nk, d, R, causal, dtype)
    (2, 2, 200, 200, 128, 199, False, "f16"),  # block of 200: no distance clamped
    (1, 2, 300, 300, 64, 16, True, "f16"),     # most distances clamped; causal
    (1, 3, 130, 257, 128, 40, True, "bf16"),   # rectangular, bottom-right causal, ragged tiles
    (2, 1, 1, 77, 128, 3, False, "f16"),       # one query row
    (1, 2, 200, 70, 64, 8, True, "bf16"),      # Nq > Nk causal: rows with no key
    (1, 2, 129, 129, 128, 0, False, "f16"),    # R = 0: one embedding row for every pair
    (1, 1, 64, 500, 128, 300, False, "f16"),   # window rows past the table's end
]


@pytest.mark.parametrize("B,H,Nq,Nk,d,R,causal,dtype", CASES)
def test_relpos_matches_oracle(B, H, Nq, Nk, d, R, causal, dtype):
    q, k, v, emb = make_relpos_inputs(B, H, Nq, Nk, d, R, dtype=dtype, seed=Nq + Nk + R)
    scale = 1.0 / math.sqrt(d)
    out, lse = attn_fwd_relpos(q.cuda(), k.cuda(), v.cuda(), emb.cuda(), R, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert get_status() == 0
    ref_o, ref_lse = oracle.attn_fwd_relpos(q, k, v, emb, clamped_dist(Nq, Nk, R), causal=causal,
                                            scale=scale)
    what = f"relpos B{B} H{H} {Nq}x{Nk} d{d} R{R} causal={causal} {dtype}"
    assert_o_close(out, ref_o, q.dtype, what)
    assert_lse_close(lse, ref_lse, what)


@pytest.mark.parametrize("B,H,Nq,Nk,R,causal", [
    (40, 4, 300, 300, 20, True),   # 480 units on 148 persistent CTAs, 1 to 5 key steps each
    (80, 2, 300, 100, 30, True),   # ... and units whose rows see no key, interleaved
])
def test_relpos_persistent_units(B, H, Nq, Nk, R, causal):
    """More units than SMs: every CTA walks several (b, h, tile) units with their barrier
    phases carried across; five batch elements spread over the walk against the oracle."""
    q, k, v, emb = make_relpos_inputs(B, H, Nq, Nk, 128, R, seed=B + Nk)
    scale = 1.0 / math.sqrt(128)
    out, lse = attn_fwd_relpos(q.cuda(), k.cuda(), v.cuda(), emb.cuda(), R, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert get_status() == 0
    dist = clamped_dist(Nq, Nk, R)
    for bb in (0, 1, B // 3, B // 2 + 1, B - 1):
        ref_o, ref_lse = oracle.attn_fwd_relpos(q[bb:bb + 1], k[bb:bb + 1], v[bb:bb + 1], emb, dist,
                                                causal=causal, scale=scale)
        what = f"relpos persistent B{B} {Nq}x{Nk} batch {bb}"
        assert_o_close(out[bb:bb + 1].cpu(), ref_o, q.dtype, what)
        assert_lse_close(lse[bb:bb + 1].cpu(), ref_lse, what)


def test_relpos_term_matters():
    """The same inputs with the term dropped (emb = 0) differ from the result with it, and
    equal plain attention: the kernel really adds the gathered term."""
    from attention_forward_tiled_b200 import attn_fwd
    q, k, v, emb = (t.cuda() for t in make_relpos_inputs(1, 2, 160, 160, 128, 20, seed=3))
    with_term, _ = attn_fwd_relpos(q, k, v, emb, 20)
    without, lse0 = attn_fwd_relpos(q, k, v, torch.zeros_like(emb), 20)
    plain, lse_plain = attn_fwd(q, k, v)
    torch.cuda.synchronize()
    assert get_status() == 0
    assert (with_term.float() - without.float()).abs().max().item() > 1e-2
    # both within 2e-3 of the same exact result
    assert (without.float() - plain.float()).abs().max().item() <= 4e-3
    assert (lse0 - lse_plain).abs().max().item() <= 1e-3


def test_relpos_full_workload_sampled():
    """The benchmark's block-local workload (512 blocks x 8 heads of 200 tokens): every
    element of four blocks spread over the grid (32 block-head pairs) against the oracle."""
    w = RELPOS_WORKLOADS["relpos_block200"]
    q, k, v, emb = make_relpos_inputs(**w)
    out, lse = attn_fwd_relpos(q.cuda(), k.cuda(), v.cuda(), emb.cuda(), w["R"], causal=w["causal"],
                               scale=w["scale"])
    torch.cuda.synchronize()
    assert get_status() == 0
    dist = clamped_dist(w["Nq"], w["Nk"], w["R"])
    blocks = [0, 37, 255, 511]
    for bb in blocks:
        ref_o, ref_lse = oracle.attn_fwd_relpos(q[bb:bb + 1], k[bb:bb + 1], v[bb:bb + 1], emb, dist,
                                                causal=w["causal"], scale=w["scale"])
        what = f"relpos_block200 block {bb}"
        assert_o_close(out[bb:bb + 1].cpu(), ref_o, q.dtype, what)
        assert_lse_close(lse[bb:bb + 1].cpu(), ref_lse, what)


def test_relpos_bf16_values_outside_the_fp16_range():
    """P V runs in fp16 here as in the plain kernel: a bf16 V element with no fp16 value
    records ATTN_ERR_RANGE; the largest bf16 value below fp16's limit (65280) does not.  The
    other head's output and every lse then match the oracle."""
    q, k, v, emb = make_relpos_inputs(1, 2, 200, 200, 128, 30, dtype="bf16", seed=21)
    qd, kd, ed = q.cuda(), k.cuda(), emb.cuda()
    for bad in (1e5, -1e5, float("inf"), 65536.0):
        vb = v.clone()
        vb[0, 150, 1, 77] = bad
        attn_fwd_relpos(qd, kd, vb.cuda(), ed, 30)
        torch.cuda.synchronize()
        assert get_status() == ATTN_ERR_RANGE, bad
    vb = v.clone()
    vb[0, 150, 1, 77] = 65280.0
    out, lse = attn_fwd_relpos(qd, kd, vb.cuda(), ed, 30)
    torch.cuda.synchronize()
    assert get_status() == 0
    ref_o, ref_lse = oracle.attn_fwd_relpos(q, k, vb, emb, clamped_dist(200, 200, 30),
                                            scale=1.0 / math.sqrt(128))
    assert_o_close(out[:, :, :1], ref_o[:, :, :1], q.dtype, "relpos bf16 V at 65280, head 0")
    assert_lse_close(lse, ref_lse, "relpos bf16 V at 65280")
