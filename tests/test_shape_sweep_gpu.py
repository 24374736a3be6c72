"""GPU parity over a seeded sweep of attention shapes: attn_fwd (the public entry point,
which picks the prefill or the split-KV decode path) against the fp64 oracle on every
output element.

The shapes are drawn once from a fixed seed (batch 1-3, 1-5 heads, 1-600 query rows,
1-700 keys, head_dim 64 or 128, fp16 or bf16, causal or not, a scale in [0.05, 0.25]
and now and then a negative one), so the cases are the same on every run; they mix
ragged tails of the 128-row query and 128-key tiles, rows without keys (causal with more
query rows than keys), single query rows and single keys.
"""
import random

import pytest
import torch

import oracle
from attention_forward_tiled_b200 import attn_fwd, get_status
from attention_forward_tiled_b200.inputs import make_inputs
from tests.parity import assert_lse_close, assert_o_close

pytestmark = pytest.mark.gpu

DT = {"f16": torch.float16, "bf16": torch.bfloat16}


def _cases(n=48, seed=20261203):
    rnd = random.Random(seed)
    cases = []
    for i in range(n):
        B = rnd.randint(1, 3)
        H = rnd.randint(1, 5)
        Nq = rnd.choice([1, rnd.randint(2, 130), rnd.randint(129, 300), rnd.randint(1, 600)])
        Nk = rnd.choice([1, rnd.randint(2, 130), rnd.randint(129, 400), rnd.randint(1, 700)])
        d = rnd.choice([64, 128])
        dtype = rnd.choice(["f16", "bf16"])
        causal = rnd.random() < 0.5
        scale = rnd.uniform(0.05, 0.25) * (-1.0 if rnd.random() < 0.1 else 1.0)
        cases.append((B, H, Nq, Nk, d, dtype, causal, round(scale, 4), 1000 + i))
    return cases


@pytest.mark.parametrize("B,H,Nq,Nk,d,dtype,causal,scale,seed", _cases())
def test_attn_fwd_shape_sweep(B, H, Nq, Nk, d, dtype, causal, scale, seed):
    q, k, v = make_inputs(B, H, Nq, Nk, d, dtype=dtype, seed=seed)
    out, lse = attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert get_status() == 0
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, causal=causal, scale=scale)
    what = f"B{B} H{H} {Nq}x{Nk} d{d} {dtype} causal={causal} scale={scale}"
    assert_o_close(out, o_ref, DT[dtype], what)
    assert_lse_close(lse, lse_ref, what)
