"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small shapes are compared element by element on every output; the full-size
workloads run exactly as the benchmark launches them and are compared on whole
sampled (batch, head) slices (heads are independent, which the oracle tests
pin) plus properties checked on every output element.
"""
import math

import pytest
import torch

import oracle
from attention_forward_tiled_b200 import ATTN_ERR_RANGE, attn_fwd, get_status
from attention_forward_tiled_b200.inputs import WORKLOADS, make_inputs
from tests.parity import assert_convex_hull, assert_lse_close, assert_o_close

pytestmark = pytest.mark.gpu

DT = {"f16": torch.float16, "bf16": torch.bfloat16}


def run_and_compare(B, H, Nq, Nk, d, dtype, causal, scale, seed, k_mult=1.0, path="auto",
                    splits=0, heads=None):
    q, k, v = make_inputs(B, H, Nq, Nk, d, dtype=dtype, seed=seed, k_mult=k_mult)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    out, lse = attn_fwd(qd, kd, vd, causal=causal, scale=scale, path=path, splits=splits)
    torch.cuda.synchronize()
    assert get_status() == 0
    if heads is None:
        o_ref, lse_ref = oracle.attn_fwd(q, k, v, causal=causal, scale=scale)
        assert_o_close(out, o_ref, DT[dtype], f"{B}x{H}x{Nq}x{Nk}x{d}")
        assert_lse_close(lse, lse_ref, "lse")
    else:
        # the heads of one batch index go to the oracle together (it runs them in parallel)
        out_h, lse_h = out.cpu(), lse.cpu()
        for b in sorted({b for b, _ in heads}):
            hs = torch.tensor(sorted({h for bb, h in heads if bb == b}))
            sel = lambda t: t[b:b + 1].index_select(2, hs)  # noqa: E731
            o_ref, lse_ref = oracle.attn_fwd(sel(q), sel(k), sel(v), causal=causal, scale=scale)
            what = f"batch {b}, heads {hs.tolist()}"
            assert_o_close(sel(out_h), o_ref, DT[dtype], what)
            assert_lse_close(lse_h[b:b + 1].index_select(1, hs), lse_ref, "lse " + what)
    return q, k, v, out, lse


SMALL = [
    # (B, H, Nq, Nk, d, dtype, causal)
    (1, 2, 128, 128, 64, "f16", False),
    (1, 2, 128, 128, 128, "f16", False),
    (2, 3, 256, 256, 128, "f16", True),
    (1, 2, 64, 64, 64, "f16", True),
    (1, 2, 63, 63, 128, "f16", False),
    (1, 2, 65, 65, 64, "f16", True),
    (1, 2, 127, 129, 128, "f16", False),
    (1, 2, 129, 127, 128, "f16", True),
    (1, 1, 200, 200, 128, "f16", True),
    (2, 2, 1000, 1000, 64, "f16", True),
    (1, 2, 1000, 1000, 128, "bf16", False),
    (1, 2, 300, 700, 128, "f16", True),     # Nq < Nk, bottom-right diagonal not on a tile edge
    (1, 2, 700, 300, 64, "f16", True),      # Nq > Nk: leading rows see no key
    (1, 2, 513, 1, 128, "f16", False),      # a single key
    (1, 2, 513, 1, 64, "bf16", True),       # single key, causal: only the last row has it
    (2, 80, 384, 256, 64, "f16", False),    # 320 tile pairs: the last partial wave runs as single
    (2, 80, 320, 200, 128, "bf16", False),  #   tiles (a pair's second tile may lie past Nq)
    (1, 3, 2, 517, 128, "f16", True),       # two query rows
    (3, 1, 384, 384, 64, "bf16", True),     # three Q tiles -> one half-used pair
    (1, 4, 128, 1024, 128, "bf16", True),
    (1, 2, 1, 300, 64, "f16", False),       # one query row on the decode path
    (2, 2, 1, 129, 128, "bf16", True),      # decode path, causal flag is a no-op
    (3, 8, 1, 1000, 64, "bf16", False),     # decode path, bf16 at d = 64
    (2, 3, 1, 4096, 128, "f16", False),     # decode path, a long row split several ways
]


@pytest.mark.parametrize("B,H,Nq,Nk,d,dtype,causal", SMALL)
def test_small_shapes(B, H, Nq, Nk, d, dtype, causal):
    run_and_compare(B, H, Nq, Nk, d, dtype, causal, 1.0 / math.sqrt(d), seed=Nq * 31 + Nk)


@pytest.mark.parametrize("scale", [0.0, -0.09, 0.5])
def test_scale_values(scale):
    run_and_compare(1, 2, 200, 333, 128, "f16", True, scale, seed=77)


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_path_with_one_query_row(d):
    run_and_compare(2, 3, 1, 777, d, "f16", False, 0.1, seed=5, path="prefill")


@pytest.mark.parametrize("splits", [1, 2, 3, 7, 32])
def test_decode_split_counts(splits):
    run_and_compare(2, 4, 1, 4000, 128, "f16", False, 1 / math.sqrt(128), seed=9, path="decode",
                    splits=splits)


def test_large_logits_bf16():
    run_and_compare(1, 4, 384, 512, 64, "bf16", False, 1 / 8, seed=3, k_mult=3.0)


@pytest.mark.parametrize("d,dtype,causal", [(128, "f16", False), (128, "bf16", True),
                                             (64, "f16", True), (64, "bf16", False)])
def test_running_max_jumps(d, dtype, causal):
    """Key norms grow tile by tile, so the row max of scale*log2(e)*s rises by ~9 per key
    tile, past the lazy threshold of 8: every lazy O rescale and the redo of a tile whose
    single-pass exponentials would overflow the running max are exercised (the inputs are
    only reshaped here)."""
    B, H, Nq, Nk = 1, 2, 512, 1024
    q, k, v = make_inputs(B, H, Nq, Nk, d, dtype="f16", seed=21 + d)
    growth = 1.0 + 2.5 * (torch.arange(Nk, dtype=torch.float32) // 128)  # x1 .. x18.5 per key tile
    k = (k.float() * growth.view(1, Nk, 1, 1)).to(DT[dtype])
    # Unit-variance V, as drawn.  The softmax is so peaked here that P rounded to fp16
    # would move O by up to 2^-11 |v| if O were normalised by the sum of the unrounded
    # P; the kernel normalises by the sum of the rounded P, which leaves a second-order
    # error, and the literal fp16 bound applies.
    q, v = q.to(DT[dtype]), v.to(DT[dtype])
    scale = 1 / math.sqrt(d)
    out, lse = attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert get_status() == 0
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, causal=causal, scale=scale)
    r = assert_o_close(out, o_ref, DT[dtype], f"growing keys d={d} {dtype} causal={causal}")
    print(f"growing keys d={d} {dtype} causal={causal}: literal max_abs={r['max_abs']:.3e} "
          f"mean_abs={r['mean_abs']:.3e} (criterion max {r['crit_max_abs']:.3e})")
    assert_lse_close(lse, lse_ref, "lse (growing keys)")


def test_bf16_values_outside_the_fp16_range():
    """The prefill multiplies P by V in fp16, converting bf16 V tiles on chip.  A V element
    with no fp16 value (|v| >= 65536, inf) makes the call record ATTN_ERR_RANGE in the status
    word; the largest bf16 value below that (65280) does not.  Tiny values (about 1e-8, below
    fp16's normal range) keep an absolute error far inside the bound.  The decode path
    computes in fp32 and takes large values as they are."""
    B, H, Nq, Nk, d = 1, 2, 256, 384, 64
    q, k, v = make_inputs(B, H, Nq, Nk, d, dtype="bf16", seed=31)
    qd, kd = q.cuda(), k.cuda()
    for bad in (1e5, -1e5, float("inf"), 65536.0):
        vb = v.clone()
        vb[0, 100, 1, 7] = bad
        attn_fwd(qd, kd, vb.cuda(), scale=0.125)
        assert get_status() == ATTN_ERR_RANGE, bad
    vb = v.clone()
    vb[0, 100, 1, 7] = 65280.0
    attn_fwd(qd, kd, vb.cuda(), scale=0.125)
    assert get_status() == 0
    # tiny values: a quarter of the V columns scaled to ~1e-8
    vt = v.float().clone()
    vt[..., : d // 4] *= 1e-8
    vt = vt.to(torch.bfloat16)
    out, lse = attn_fwd(qd, kd, vt.cuda(), scale=0.125)
    assert get_status() == 0
    o_ref, lse_ref = oracle.attn_fwd(q, k, vt, scale=0.125)
    assert_o_close(out, o_ref, torch.bfloat16, "tiny bf16 V values")
    assert_lse_close(lse, lse_ref, "lse, tiny bf16 V values")
    # one query row (decode path, fp32 arithmetic): 1e5 is no special case there
    vb = v.clone()
    vb[0, 100, 1, 7] = 1e5
    q1 = q[:, :1].contiguous()
    out, lse = attn_fwd(q1.cuda(), kd, vb.cuda(), scale=0.125)
    assert get_status() == 0
    o_ref, lse_ref = oracle.attn_fwd(q1, k, vb, scale=0.125)
    og = out.double().cpu().numpy()
    assert (abs(og - o_ref) <= 2e-3 + 2.0 ** -8 * abs(o_ref)).all(), "decode with a large bf16 V value"
    assert_lse_close(lse, lse_ref, "decode lse, large bf16 V value")


def test_lse_optional_and_deterministic():
    q, k, v = (t.cuda() for t in make_inputs(2, 4, 300, 300, 128, seed=8))
    o1, _ = attn_fwd(q, k, v, causal=True, return_lse=False)
    o2, l2 = attn_fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    assert l2 is not None


def test_side_stream():
    q, k, v = (t.cuda() for t in make_inputs(1, 2, 256, 256, 64, seed=12))
    ref, _ = attn_fwd(q, k, v)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        out, _ = attn_fwd(q, k, v, stream=s)
    s.synchronize()
    assert torch.equal(out, ref)


# ---------------------------------------------------------------------------
# the named workloads, at full size, in the launch configuration the bench uses
# ---------------------------------------------------------------------------
# The prefill hands out work units (b, h, pair of Q tiles) in groups of 16 consecutive
# (b, h) heads, heaviest causal units first, to CTAs that claim them dynamically; the
# last partial wave of a non-causal launch runs as single-tile units.  Every unit of the
# compared heads is checked element by element against the oracle; the rest of the
# output is checked against properties that hold at any size.
HEADS_PER_GROUP = 16


def _group(name, g):
    """(b, h) of scheduling group g of a workload."""
    w = WORKLOADS[name]
    return [divmod(bh, w["H"]) for bh in range(HEADS_PER_GROUP * g, HEADS_PER_GROUP * (g + 1))
            if bh < w["B"] * w["H"]]


def _all_heads(name):
    w = WORKLOADS[name]
    return [(b, h) for b in range(w["B"]) for h in range(w["H"])]


def _workload(name, heads):
    w = WORKLOADS[name]
    q, k, v, out, lse = run_and_compare(w["B"], w["H"], w["Nq"], w["Nk"], w["d"], w["dtype"],
                                        w["causal"], w["scale"], w["seed"], w["k_mult"],
                                        heads=heads)
    assert_convex_hull(out, v.cuda(), w["causal"], w["Nq"], w["Nk"])
    assert torch.isfinite(lse).all()


def test_workload_tiny():
    _workload("tiny", heads=None)


def test_workload_causal4k():
    # the first head, and the whole last group of 16 heads (its units are claimed last)
    _workload("causal4k", heads=[(0, 0)] + _group("causal4k", 7))


def test_workload_bf16_k3():
    # every head: 512 tile pairs on 148 SMs, the last 68 pairs run as 136 single tiles
    _workload("bf16_k3", heads=_all_heads("bf16_k3"))


def test_workload_causal8k():
    # the second (last) group of 16 heads
    _workload("causal8k", heads=_group("causal8k", 1))


def test_workload_causal8000():
    # every head: ragged last tiles in both the query and the key direction
    _workload("causal8000", heads=_all_heads("causal8000"))


def test_workload_decode():
    _workload("decode", heads=None)
