"""GPU parity of the multi-token paged attention (attn_fwd_paged, tensor cores) against
the fp64 oracle's own paged walk (oracle.attn_fwd_paged).

Request b's Lq query tokens are the last Lq positions of its seq_lens[b] keys (the
bottom-right rule); the cases cover ragged and empty sequences, sequences shorter
than Lq under the causal flag (leading tokens see no key: O = 0, lse = -inf), page
sizes 8 to 256, head dims 64 and 128, fp16 and bf16, 1 to 16 tokens and explicit
split counts.
"""
import math

import pytest
import torch

import oracle
from attention_forward_tiled_b200 import attn_fwd_decode_paged, attn_fwd_paged, get_status
from attention_forward_tiled_b200.inputs import make_paged_inputs
from tests.parity import assert_lse_close, assert_o_close

pytestmark = pytest.mark.gpu

DT = {"f16": torch.float16, "bf16": torch.bfloat16}

CASES = [
    # (H, d, dtype, page_size, seq_lens, max_blocks, Lq, causal, splits)
    (4, 128, "f16", 16, [1, 17, 300, 1000], 64, 4, True, 0),
    (4, 128, "f16", 16, [1, 17, 300, 1000], 64, 4, False, 0),
    (2, 64, "bf16", 128, [0, 128, 129, 700], 6, 8, True, 0),
    (2, 64, "f16", 128, [5, 3, 1000], 8, 8, True, 0),        # L < Lq: leading tokens see nothing
    (3, 128, "bf16", 16, [4096, 2049, 33], 256, 2, True, 0),
    (2, 128, "f16", 256, [4096, 1, 2049], 16, 16, False, 0),
    (2, 128, "f16", 8, [5, 200, 129], 64, 3, True, 3),       # 512-key table: 4 tiles, 3 splits
    (2, 64, "bf16", 32, [1000, 999], 32, 1, False, 1),
    (1, 128, "f16", 64, [130], 4, 16, True, 2),
]


@pytest.mark.parametrize("H,d,dtype,page,seq_lens,max_blocks,Lq,causal,splits", CASES)
def test_paged_multi_token_matches_oracle(H, d, dtype, page, seq_lens, max_blocks, Lq, causal, splits):
    B = len(seq_lens)
    q, kc, vc, bt, sl = make_paged_inputs(B, H, d, seq_lens, page, dtype=dtype, Lq=Lq,
                                          seed=page + d + B + Lq, max_blocks=max_blocks)
    scale = 1.0 / math.sqrt(d)
    out, lse = attn_fwd_paged(q.cuda(), kc.cuda(), vc.cuda(), bt.cuda(), sl.cuda(), causal=causal,
                              scale=scale, splits=splits)
    torch.cuda.synchronize()
    assert get_status() == 0
    bt_ref = bt.clone()
    bt_ref[bt_ref < 0] = 0  # entries past a sequence are never read; the oracle wants them in range
    o_ref, lse_ref = oracle.attn_fwd_paged(q, kc, vc, bt_ref, sl, causal=causal, scale=scale)
    what = f"Lq={Lq} causal={causal} page={page} d={d} {dtype} seq_lens={seq_lens}"
    r = assert_o_close(out, o_ref, DT[dtype], what)
    print(f"{what}: max_abs={r['max_abs']:.2e} mean_abs={r['mean_abs']:.2e}")
    assert_lse_close(lse, lse_ref, "lse " + what)


def test_one_token_equals_single_query_decode():
    """Lq = 1 without the causal flag is the single-query paged decode: same result up to
    the rounding of P (fp32 on the CUDA-core path, the input type on the tensor cores)."""
    H, d, page, seq_lens = 4, 128, 16, [37, 4000, 512]
    q, kc, vc, bt, sl = (t.cuda() for t in make_paged_inputs(3, H, d, seq_lens, page, seed=91))
    out1, lse1 = attn_fwd_decode_paged(q, kc, vc, bt, sl)
    out2, lse2 = attn_fwd_paged(q, kc, vc, bt, sl, causal=False)
    torch.cuda.synchronize()
    assert get_status() == 0
    assert_o_close(out2, out1.double().cpu().numpy(), torch.float16, "Lq=1 vs single-query decode")
    assert_lse_close(lse2[:, :, 0], lse1.double().cpu().numpy(), "Lq=1 lse vs single-query decode")


def test_tokens_past_sixteen_are_rejected():
    from attention_forward_tiled_b200 import AttnError
    q, kc, vc, bt, sl = (t.cuda() for t in make_paged_inputs(1, 2, 64, [100], 16, Lq=17, seed=3))
    with pytest.raises(AttnError):
        attn_fwd_paged(q, kc, vc, bt, sl)


def test_paged_multi_token_bf16_range_status():
    """bf16 V tiles are converted to fp16 on chip for the P V product: a V element of a
    request's sequence with no fp16 value records ATTN_ERR_RANGE; the largest bf16 value
    below fp16's limit (65280) does not, and neither does a huge value in a cache row that
    no request reads."""
    from attention_forward_tiled_b200 import ATTN_ERR_RANGE
    H, d, page, seq_lens, Lq = 2, 128, 16, [40, 70], 4
    q, kc, vc, bt, sl = make_paged_inputs(len(seq_lens), H, d, seq_lens, page, dtype="bf16", Lq=Lq, seed=77,
                                          max_blocks=8)
    used = int(bt[1, 2])            # a page of request 1 (keys 32..47, inside its 70 keys)
    spare = kc.shape[0] - 1         # the spare pages at the end of the cache are never listed
    assert spare not in set(bt[bt >= 0].tolist())
    args = lambda v: (q.cuda(), kc.cuda(), v.cuda(), bt.cuda(), sl.cuda())  # noqa: E731
    for bad in (1e5, float("inf")):
        v = vc.clone()
        v[used, 3, 1, 5] = bad
        attn_fwd_paged(*args(v), causal=True)
        torch.cuda.synchronize()
        assert get_status() == ATTN_ERR_RANGE, bad
    v = vc.clone()
    v[used, 3, 1, 5] = 65280.0
    v[spare, 0, 0, 0] = 1e5
    attn_fwd_paged(*args(v), causal=True)
    torch.cuda.synchronize()
    assert get_status() == 0
