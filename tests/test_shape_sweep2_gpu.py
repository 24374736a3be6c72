"""GPU parity over seeded shape sweeps of the widened entry points: the backward pass
(attn_bwd), multi-token attention and single-query decode over a paged cache
(attn_fwd_paged, attn_fwd_decode_paged), attention with the relative-position term
(attn_fwd_relpos) and the lightning-indexer score with its top-k, each against the fp64
oracle with the criteria of its own test file.

Every sweep draws its cases once from a fixed seed, so they are the same on every run;
they mix ragged tiles, single rows and keys, empty and short sequences, all page sizes
the paged path takes, both head dims and dtypes, and causal on and off.
"""
import math
import random

import numpy as np
import pytest
import torch

import oracle
from attention_forward_tiled_b200 import attn_bwd, attn_fwd, attn_fwd_paged, attn_fwd_relpos, get_status
from attention_forward_tiled_b200.inputs import make_inputs, make_paged_inputs, make_relpos_inputs
from tests.parity import assert_lse_close, assert_o_close
from tests.test_backward_gpu import SUB, U, bounds

pytestmark = pytest.mark.gpu

DT = {"f16": torch.float16, "bf16": torch.bfloat16}


def clamped_dist(Nq, Nk, R):
    """The conformer's relative-distance table: clamp(i - j, -R, R) + R."""
    i = np.arange(Nq).reshape(Nq, 1)
    j = np.arange(Nk).reshape(1, Nk)
    return (np.clip(i - j, -R, R) + R).astype(np.int32)


def _bwd_cases(n=16, seed=7101):
    rnd = random.Random(seed)
    out = []
    for i in range(n):
        out.append((rnd.randint(1, 2), rnd.randint(1, 3), rnd.choice([1, rnd.randint(2, 140), rnd.randint(129, 400)]),
                    rnd.choice([1, rnd.randint(2, 140), rnd.randint(129, 400)]), rnd.choice([64, 128]),
                    rnd.choice(["f16", "bf16"]), rnd.random() < 0.5, 2000 + i))
    return out


@pytest.mark.parametrize("B,H,Nq,Nk,d,dtype,causal,seed", _bwd_cases())
def test_bwd_shape_sweep(B, H, Nq, Nk, d, dtype, causal, seed):
    q, k, v = make_inputs(B, H, Nq, Nk, d, dtype=dtype, seed=seed)
    g = torch.Generator("cpu").manual_seed(seed)
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
        lim = 2 * bd + 0.5 * U[dtype] * 2 * np.abs(r) + SUB[dtype] + 1e-12  # plus the output's own rounding
        assert np.isfinite(gn).all(), name
        assert (err <= lim).all(), f"{name} B{B} H{H} {Nq}x{Nk} d{d} {dtype} causal={causal}: " \
                                   f"error beyond bound by {float((err - lim).max()):.3e}"


def _paged_cases(n=16, seed=7202):
    rnd = random.Random(seed)
    out = []
    for i in range(n):
        page = rnd.choice([8, 16, 32, 64, 128, 256])
        nreq = rnd.randint(1, 4)
        seq_lens = [rnd.choice([0, 1, rnd.randint(2, 300), rnd.randint(1, 1500)]) for _ in range(nreq)]
        max_blocks = max(1, -(-max(seq_lens) // page) + rnd.randint(0, 2))
        out.append((rnd.randint(1, 4), rnd.choice([64, 128]), rnd.choice(["f16", "bf16"]), page, seq_lens,
                    max_blocks, rnd.randint(1, 16), rnd.random() < 0.5, 3000 + i))
    return out


@pytest.mark.parametrize("H,d,dtype,page,seq_lens,max_blocks,Lq,causal,seed", _paged_cases())
def test_paged_shape_sweep(H, d, dtype, page, seq_lens, max_blocks, Lq, causal, seed):
    B = len(seq_lens)
    q, kc, vc, bt, sl = make_paged_inputs(B, H, d, seq_lens, page, dtype=dtype, Lq=Lq, seed=seed,
                                          max_blocks=max_blocks)
    scale = 1.0 / math.sqrt(d)
    out, lse = attn_fwd_paged(q.cuda(), kc.cuda(), vc.cuda(), bt.cuda(), sl.cuda(), causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert get_status() == 0
    bt_ref = bt.clone()
    bt_ref[bt_ref < 0] = 0  # entries past a sequence are never read; the oracle wants them in range
    o_ref, lse_ref = oracle.attn_fwd_paged(q, kc, vc, bt_ref, sl, causal=causal, scale=scale)
    what = f"Lq={Lq} causal={causal} page={page} d={d} {dtype} seq_lens={seq_lens}"
    assert_o_close(out, o_ref, DT[dtype], what)
    assert_lse_close(lse, lse_ref, "lse " + what)


def _relpos_cases(n=16, seed=7303):
    rnd = random.Random(seed)
    out = []
    for i in range(n):
        Nq = rnd.choice([1, rnd.randint(2, 140), rnd.randint(129, 320)])
        Nk = rnd.choice([1, rnd.randint(2, 140), rnd.randint(129, 320)])
        out.append((rnd.randint(1, 2), rnd.randint(1, 3), Nq, Nk, rnd.choice([64, 128]),
                    rnd.choice([0, rnd.randint(1, 40), rnd.randint(1, 330)]), rnd.random() < 0.5,
                    rnd.choice(["f16", "bf16"]), 4000 + i))
    return out


@pytest.mark.parametrize("B,H,Nq,Nk,d,R,causal,dtype,seed", _relpos_cases())
def test_relpos_shape_sweep(B, H, Nq, Nk, d, R, causal, dtype, seed):
    q, k, v, emb = make_relpos_inputs(B, H, Nq, Nk, d, R, dtype=dtype, seed=seed)
    scale = 1.0 / math.sqrt(d)
    out, lse = attn_fwd_relpos(q.cuda(), k.cuda(), v.cuda(), emb.cuda(), R, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert get_status() == 0
    o_ref, lse_ref = oracle.attn_fwd_relpos(q, k, v, emb, clamped_dist(Nq, Nk, R), causal=causal, scale=scale)
    what = f"relpos B{B} H{H} {Nq}x{Nk} d{d} R{R} causal={causal} {dtype}"
    assert_o_close(out, o_ref, DT[dtype], what)
    assert_lse_close(lse, lse_ref, what)


def _decode_paged_cases(n=12, seed=7404):
    rnd = random.Random(seed)
    out = []
    for i in range(n):
        page = rnd.choice([8, 16, 32, 64, 128, 256])
        nreq = rnd.randint(1, 5)
        seq_lens = [rnd.choice([0, 1, rnd.randint(2, 300), rnd.randint(1, 3000)]) for _ in range(nreq)]
        max_blocks = max(1, -(-max(seq_lens) // page) + rnd.randint(0, 2))
        tiles = -(-max_blocks * page // 128)  # an explicit split count is at most the table's key tiles
        out.append((rnd.randint(1, 4), rnd.choice([64, 128]), rnd.choice(["f16", "bf16"]), page, seq_lens,
                    max_blocks, min(tiles, rnd.choice([0, 0, 1, rnd.randint(2, 6)])), 5000 + i))
    return out


@pytest.mark.parametrize("H,d,dtype,page,seq_lens,max_blocks,splits,seed", _decode_paged_cases())
def test_decode_paged_shape_sweep(H, d, dtype, page, seq_lens, max_blocks, splits, seed):
    from attention_forward_tiled_b200 import attn_fwd_decode_paged
    B = len(seq_lens)
    q, kc, vc, bt, sl = make_paged_inputs(B, H, d, seq_lens, page, dtype=dtype, seed=seed, max_blocks=max_blocks)
    scale = 1.0 / math.sqrt(d)
    out, lse = attn_fwd_decode_paged(q.cuda(), kc.cuda(), vc.cuda(), bt.cuda(), sl.cuda(), scale=scale,
                                     splits=splits)
    torch.cuda.synchronize()
    assert get_status() == 0
    bt_ref = bt.clone()
    bt_ref[bt_ref < 0] = 0  # entries past a sequence are never read; the oracle wants them in range
    o_ref, lse_ref = oracle.attn_fwd_paged(q, kc, vc, bt_ref, sl, causal=False, scale=scale)
    what = f"decode page={page} d={d} {dtype} seq_lens={seq_lens} splits={splits}"
    assert_o_close(out, o_ref, DT[dtype], what)
    assert_lse_close(lse.unsqueeze(-1), lse_ref, "lse " + what)  # [B, H] against [B, H, 1]


def _indexer_cases(n=12, seed=7505):
    rnd = random.Random(seed)
    out = []
    for i in range(n):
        H = rnd.choice([1, 2, 4, 8, 16, 32, 64, 128])
        out.append((rnd.randint(1, 2), rnd.choice([1, rnd.randint(2, 70), rnd.randint(60, 200)]), H,
                    rnd.choice([1, rnd.randint(2, 300), rnd.randint(257, 1100)]), rnd.choice([64, 128]),
                    rnd.choice(["f16", "bf16"]), rnd.choice(["random", "constant"]), rnd.random() < 0.7,
                    6000 + i))
    return out


@pytest.mark.parametrize("B,T,H,P,d,dtype,weights,masked,seed", _indexer_cases())
def test_indexer_shape_sweep(B, T, H, P, d, dtype, weights, masked, seed):
    """Scores within the fp32-accumulation bound of the indexer's own test (2^-14 times the
    sum of the magnitudes of the terms), masked entries exactly -inf, and the top-k of the
    GPU's scores equal to the oracle's top-k of the same scores, index for index."""
    from attention_forward_tiled_b200 import indexer_score, topk
    from attention_forward_tiled_b200.inputs import make_indexer_inputs
    q, kp, w, mask = make_indexer_inputs(B, T, H, P, d, dtype=dtype, seed=seed, weights=weights, masked=masked)
    out = indexer_score(q.cuda(), kp.cuda(), w.cuda(), mask.cuda() if mask is not None else None)
    torch.cuda.synchronize()
    assert get_status() == 0
    ref = oracle.indexer_score(q, kp, w, mask)
    got = out.double().cpu().numpy()
    fin = np.isfinite(ref)
    assert np.array_equal(np.isneginf(got), np.isneginf(ref)), "masked entries must be -inf"
    qa, ka, wa = q.double().abs(), kp.double().abs(), w.double().abs()
    bound = 2.0 ** -14 * torch.einsum("bth,bthp->btp", wa, torch.einsum("bthc,bpc->bthp", qa, ka)).numpy() + 1e-30
    err = np.abs(got[fin] - ref[fin])
    assert (err <= bound[fin]).all(), f"score error {float((err - bound[fin]).max())} beyond the fp32 bound"
    k = min(P, [1, 7, 64, 300][seed % 4])
    idx = topk(out, k)
    torch.cuda.synchronize()
    assert get_status() == 0
    assert np.array_equal(idx.cpu().numpy(), oracle.topk(got.reshape(-1, P), k).reshape(idx.shape))
