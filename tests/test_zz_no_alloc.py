"""attn_fwd_decode_noalloc: the decode entry point that allocates no device memory.

It exists for callers that cannot allocate while they run -- a plug-in inside a
framework that owns all device memory and only hands over input and output
buffers, a serving loop that bans allocation after start-up, a process at its
memory limit.  Its split partials live in a fixed 4 MiB array compiled into the
library.  These tests call it through the C ABI and compare its output with the
allocating entry point attn_fwd_decode on two calls in a row (different shapes,
so the second call runs over the first call's leftovers in the shared array),
using the parity tolerances of the rest of the suite.
"""
import ctypes
import math

import pytest
import torch

import attention_forward_tiled_b200 as attn
from attention_forward_tiled_b200.inputs import make_inputs
from tests.parity import assert_lse_close, assert_o_close

pytestmark = pytest.mark.gpu

SCRATCH_FLOATS = 1 << 20


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr() if t is not None else 0)


def _call(fn, q, k, v, out, lse, splits, stream):
    B, Nk, H, d = k.shape
    dt = attn.ATTN_BF16 if q.dtype == torch.bfloat16 else attn.ATTN_F16
    return fn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Nk, d,
              1.0 / math.sqrt(d), dt, splits, ctypes.c_void_p(stream.cuda_stream))


CASES = [
    # (B, H, Nk, d, dtype, splits): the 16 x 32 x 4096 decode workload, then a bf16 one
    (16, 32, 4096, 128, "f16", 0),
    (3, 8, 1000, 64, "bf16", 5),
]


def test_noalloc_matches_allocating_entry_point_two_calls():
    lib = attn.load_library()
    stream = torch.cuda.current_stream()
    for B, H, Nk, d, dtype, splits in CASES:
        q, k, v = (t.cuda() for t in make_inputs(B, H, 1, Nk, d, dtype=dtype, seed=Nk + d))
        out_ref = torch.empty_like(q)
        lse_ref = torch.empty((B, H, 1), dtype=torch.float32, device="cuda")
        assert _call(lib.attn_fwd_decode, q, k, v, out_ref, lse_ref, splits, stream) == attn.ATTN_OK
        out = torch.full_like(q, float("nan"))
        lse = torch.full((B, H, 1), float("nan"), dtype=torch.float32, device="cuda")
        assert _call(lib.attn_fwd_decode_noalloc, q, k, v, out, lse, splits, stream) == attn.ATTN_OK
        torch.cuda.synchronize()
        assert attn.get_status() == attn.ATTN_OK
        assert_o_close(out, out_ref.double().cpu().numpy(), q.dtype, f"no-alloc {B}x{H}x{Nk}x{d}")
        assert_lse_close(lse, lse_ref.double().cpu().numpy(), "no-alloc lse")


def test_noalloc_rejects_sizes_beyond_its_array():
    lib = attn.load_library()
    stream = torch.cuda.current_stream()
    B, H, Nk, d = 64, 64, 4096, 128
    splits = 32  # 64 * 64 * 32 * 130 floats > 2^20
    assert B * H * splits * (d + 2) > SCRATCH_FLOATS
    q = torch.zeros((B, 1, H, d), dtype=torch.float16, device="cuda")
    k = torch.zeros((B, Nk, H, d), dtype=torch.float16, device="cuda")
    out = torch.zeros_like(q)
    rc = _call(lib.attn_fwd_decode_noalloc, q, k, k, out, None, splits, stream)
    assert rc == attn.ATTN_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert attn.get_status() == attn.ATTN_OK
