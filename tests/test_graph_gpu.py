"""CUDA-graph capture of the library's calls (the boundary's asynchrony contract).

Every entry point only enqueues work on the caller's stream and takes its workspace
(split-KV partials, the backward's D and dQ accumulator) from the stream-ordered
allocator, so a call can be captured into a CUDA graph and replayed; the replay must
reproduce the eager result bit for bit (the backward's dQ within rounding: its
accumulation order over key tiles is not fixed).
"""
import math

import pytest
import torch

from attention_forward_tiled_b200 import attn_fwd, get_status
from attention_forward_tiled_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,Nq,Nk,d,dtype,causal", [
    (2, 4, 700, 700, 128, "f16", True),   # prefill, d = 128
    (1, 4, 300, 900, 64, "bf16", False),  # prefill, d = 64
    (4, 8, 1, 3000, 128, "f16", False),   # decode (split over keys, workspace allocated in the call)
])
def test_graph_replay_matches_eager(B, H, Nq, Nk, d, dtype, causal):
    q, k, v = (t.cuda() for t in make_inputs(B, H, Nq, Nk, d, dtype=dtype, seed=77 + d))
    scale = 1.0 / math.sqrt(d)
    ref, ref_lse = attn_fwd(q, k, v, causal=causal, scale=scale)
    out = torch.empty_like(ref)
    lse = torch.empty_like(ref_lse)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up on the capture stream
        attn_fwd(q, k, v, causal=causal, scale=scale, out=out, lse=lse)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    out.zero_()
    lse.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        attn_fwd(q, k, v, causal=causal, scale=scale, out=out, lse=lse)
    for _ in range(3):
        out.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert get_status() == 0
    assert torch.equal(out, ref)
    assert torch.equal(lse, ref_lse)
    del g


def _replay_equals_eager(run, outs):
    """Capture run() (after one eager call on the capture stream) and check that replays
    reproduce the eager outputs bit for bit."""
    ref = [o.clone() for o in run()]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    for o in outs:
        o.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    for _ in range(3):
        for o in outs:
            o.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert get_status() == 0
    for o, r in zip(outs, ref):
        assert torch.equal(o, r)
    del g


def test_graph_replay_paged_multi_token():
    from attention_forward_tiled_b200 import attn_fwd_paged
    from attention_forward_tiled_b200.inputs import make_paged_inputs
    q, kc, vc, bt, sl = (t.cuda() for t in make_paged_inputs(3, 4, 128, [700, 33, 2000], 16, Lq=4, seed=5))
    out = torch.empty_like(q)
    lse = torch.empty((3, 4, 4), dtype=torch.float32, device="cuda")
    _replay_equals_eager(lambda: attn_fwd_paged(q, kc, vc, bt, sl, causal=True, out=out, lse=lse), [out, lse])


def test_graph_replay_indexer_and_topk():
    from attention_forward_tiled_b200 import indexer_score, topk
    from attention_forward_tiled_b200.inputs import make_indexer_inputs
    q, kp, w, mask = (t.cuda() for t in make_indexer_inputs(1, 64, 4, 1000, 128, seed=6))
    score = torch.empty((1, 64, 1000), dtype=torch.float32, device="cuda")
    idx = torch.empty((1, 64, 32), dtype=torch.int32, device="cuda")

    def run():
        indexer_score(q, kp, w, mask, out=score)
        topk(score, 32, out=idx)
        return score, idx

    _replay_equals_eager(run, [score, idx])


def test_graph_replay_relpos():
    from attention_forward_tiled_b200 import attn_fwd_relpos
    from attention_forward_tiled_b200.inputs import make_relpos_inputs
    q, k, v, emb = (t.cuda() for t in make_relpos_inputs(2, 2, 200, 200, 128, 50, seed=12))
    out = torch.empty_like(q)
    lse = torch.empty((2, 2, 200), dtype=torch.float32, device="cuda")
    _replay_equals_eager(lambda: attn_fwd_relpos(q, k, v, emb, 50, causal=True, out=out, lse=lse), [out, lse])


def test_graph_replay_backward():
    from attention_forward_tiled_b200 import attn_bwd
    q, k, v = (t.cuda() for t in make_inputs(1, 2, 200, 300, 128, dtype="f16", seed=8))
    dout = torch.randn_like(q, dtype=torch.float32).to(q.dtype)
    o, lse = attn_fwd(q, k, v, causal=True)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    # the dQ accumulation order over key tiles is not fixed (atomic adds), so dq is compared
    # within a small bound; dk and dv are written once and must match exactly
    def run():
        return attn_bwd(q, k, v, o, lse, dout, causal=True, dq=dq, dk=dk, dv=dv)

    ref = [t.clone() for t in run()]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    for t in (dq, dk, dv):
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert get_status() == 0
    assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])
    assert (dq.float() - ref[0].float()).abs().max().item() <= 1e-3 * max(1.0, ref[0].float().abs().max().item())
    del g
