"""GPU parity of the paged-cache decode (attn_fwd_decode_paged) against the oracle.

Each request's keys and values are gathered from its pages on the host (plain
indexing) and handed to the fp64 oracle as a dense [1, L, H, d] row; requests
with no key must come back as O = 0, lse = -inf.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from attention_forward_tiled_b200 import attn_fwd_decode_paged, get_status
from attention_forward_tiled_b200.inputs import make_paged_inputs
from tests.parity import assert_lse_close, assert_o_close

pytestmark = pytest.mark.gpu

DT = {"f16": torch.float16, "bf16": torch.bfloat16}


def gather(cache, table_row, L):
    page = cache.shape[1]
    n = (L + page - 1) // page
    rows = torch.cat([cache[int(p)] for p in table_row[:n]], dim=0) if n else cache[:0, 0]
    return rows[:L].unsqueeze(0)  # [1, L, H, d]


CASES = [
    # (H, d, dtype, page_size, seq_lens, max_blocks, splits)
    (4, 128, "f16", 16, [1, 17, 300, 1000], 64, 0),
    (2, 64, "bf16", 64, [0, 128, 129, 700], 12, 0),
    (4, 128, "f16", 256, [4096, 1, 2049], 16, 0),
    (3, 128, "bf16", 8, [5, 200, 129], 64, 3),   # 512-key table: 4 tiles, 3 splits
    (2, 64, "f16", 128, [1000, 999], 8, 1),
]


@pytest.mark.parametrize("H,d,dtype,page,seq_lens,max_blocks,splits", CASES)
def test_paged_decode_matches_oracle(H, d, dtype, page, seq_lens, max_blocks, splits):
    B = len(seq_lens)
    q, kc, vc, bt, sl = make_paged_inputs(B, H, d, seq_lens, page, dtype=dtype,
                                          seed=page + d + B, max_blocks=max_blocks)
    scale = 1.0 / math.sqrt(d)
    out, lse = attn_fwd_decode_paged(q.cuda(), kc.cuda(), vc.cuda(), bt.cuda(), sl.cuda(),
                                     scale=scale, splits=splits)
    torch.cuda.synchronize()
    assert get_status() == 0
    for b, L in enumerate(seq_lens):
        if L == 0:
            assert torch.all(out[b] == 0)
            assert torch.all(torch.isneginf(lse[b]))
            continue
        kb, vb = gather(kc, bt[b], L), gather(vc, bt[b], L)
        o_ref, lse_ref = oracle.attn_fwd(q[b:b + 1], kb, vb, causal=False, scale=scale)
        assert_o_close(out[b:b + 1], o_ref, DT[dtype], f"request {b} (L={L}, page {page})")
        assert_lse_close(lse[b:b + 1].unsqueeze(-1), np.asarray(lse_ref), f"lse request {b}")


def test_paged_equals_dense_layout_decode():
    """A cache whose pages are laid out in order is a dense cache: same result as attn_fwd."""
    from attention_forward_tiled_b200 import attn_fwd
    from attention_forward_tiled_b200.inputs import make_inputs
    B, H, Nk, d, page = 2, 4, 1024, 128, 16
    q, k, v = (t.cuda() for t in make_inputs(B, H, 1, Nk, d, seed=55))
    kc = k.reshape(B * Nk // page, page, H, d)
    vc = v.reshape(B * Nk // page, page, H, d)
    bt = torch.arange(B * Nk // page, dtype=torch.int32, device="cuda").reshape(B, Nk // page)
    sl = torch.full((B,), Nk, dtype=torch.int32, device="cuda")
    out_p, lse_p = attn_fwd_decode_paged(q, kc, vc, bt, sl, splits=4)
    out_d, lse_d = attn_fwd(q, k, v, path="decode", splits=4)
    torch.cuda.synchronize()
    assert torch.equal(out_p, out_d)
    assert torch.equal(lse_p, lse_d[:, :, 0])
