"""CUDA-graph capture of the forward (the boundary's asynchrony contract).

attn_fwd only enqueues work on the caller's stream and takes its split-KV workspace
from the stream-ordered allocator, so a call can be captured into a CUDA graph and
replayed; the replay must reproduce the eager result bit for bit.
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
