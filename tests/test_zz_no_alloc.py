"""attn_fwd_decode_noalloc: the decode entry point that allocates no device memory.

It exists for callers that cannot allocate while they run -- a plug-in inside a
framework that owns all device memory and only hands over input and output
buffers, a serving loop that bans allocation after start-up, a process at its
memory limit.  Its split partials live in a fixed 4 MiB array compiled into the
library.  These tests call it through the C ABI and compare its output with the
allocating entry point attn_fwd_decode and with the fp64 oracle on two calls in a
row (different shapes, so the second call runs over the first call's leftovers in
the shared array), using the parity tolerances of the rest of the suite; they
check the size limit at its edge, the automatic split choice under that limit,
and, through the device's default memory pool, that a call allocates nothing.

This file is collected last, so a run that stops at the first failure has run
every other test before it.
"""
import ctypes
import math

import pytest
import torch

import attention_forward_tiled_b200 as attn
import oracle
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


def _run_pair(lib, q, k, v, splits, stream):
    """(out, lse) of attn_fwd_decode and of attn_fwd_decode_noalloc on the same inputs."""
    B, _, H, _ = q.shape
    out_ref = torch.empty_like(q)
    lse_ref = torch.empty((B, H, 1), dtype=torch.float32, device=q.device)
    assert _call(lib.attn_fwd_decode, q, k, v, out_ref, lse_ref, splits, stream) == attn.ATTN_OK
    out = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, 1), float("nan"), dtype=torch.float32, device=q.device)
    assert _call(lib.attn_fwd_decode_noalloc, q, k, v, out, lse, splits, stream) == attn.ATTN_OK
    torch.cuda.synchronize()
    assert attn.get_status() == attn.ATTN_OK
    return out_ref, lse_ref, out, lse


CASES = [
    # (B, H, Nk, d, dtype, splits): the 16 x 32 x 4096 decode workload, then a bf16 one
    (16, 32, 4096, 128, "f16", 0),
    (3, 8, 1000, 64, "bf16", 5),
]


def test_noalloc_matches_allocating_entry_point_and_oracle_two_calls():
    lib = attn.load_library()
    stream = torch.cuda.current_stream()
    for B, H, Nk, d, dtype, splits in CASES:
        qc, kc, vc = make_inputs(B, H, 1, Nk, d, dtype=dtype, seed=Nk + d)
        q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
        out_ref, lse_ref, out, lse = _run_pair(lib, q, k, v, splits, stream)
        what = f"no-alloc {B}x{H}x{Nk}x{d} {dtype}"
        assert_o_close(out, out_ref.double().cpu().numpy(), q.dtype, what + " vs attn_fwd_decode")
        assert_lse_close(lse, lse_ref.double().cpu().numpy(), what + " lse vs attn_fwd_decode")
        o_or, lse_or = oracle.attn_fwd(qc, kc, vc, causal=False, scale=1.0 / math.sqrt(d))
        assert_o_close(out, o_or, q.dtype, what + " vs oracle")
        assert_lse_close(lse, lse_or, what + " lse vs oracle")


def test_noalloc_automatic_splits_fit_the_array():
    """48 rows of 65536 keys: the unconstrained choice would take 512 splits (1.6 M
    floats of partials); the automatic choice of the no-alloc call stays within 2^20."""
    lib = attn.load_library()
    stream = torch.cuda.current_stream()
    B, H, Nk, d = 1, 48, 65536, 64
    qc, kc, vc = make_inputs(B, H, 1, Nk, d, dtype="f16", seed=4848)
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    out = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, 1), float("nan"), dtype=torch.float32, device="cuda")
    assert _call(lib.attn_fwd_decode_noalloc, q, k, v, out, lse, 0, stream) == attn.ATTN_OK
    torch.cuda.synchronize()
    assert attn.get_status() == attn.ATTN_OK
    o_or, lse_or = oracle.attn_fwd(qc, kc, vc, causal=False, scale=1.0 / math.sqrt(d))
    assert_o_close(out, o_or, q.dtype, "no-alloc, automatic splits under the limit")
    assert_lse_close(lse, lse_or, "no-alloc lse, automatic splits under the limit")


def test_noalloc_size_limit_at_its_edge():
    """B*H*splits*(d+2) floats: 8065 rows x 130 fits 2^20, 8066 rows do not."""
    lib = attn.load_library()
    stream = torch.cuda.current_stream()
    B, H, Nk, d = 5, 1613, 128, 128
    assert B * H * (d + 2) <= SCRATCH_FLOATS < (B * H + 1) * (d + 2)
    q, k, v = (t.cuda() for t in make_inputs(B, H, 1, Nk, d, dtype="f16", seed=8065))
    out_ref, lse_ref, out, lse = _run_pair(lib, q, k, v, 1, stream)
    assert_o_close(out, out_ref.double().cpu().numpy(), q.dtype, "no-alloc at the limit")
    assert_lse_close(lse, lse_ref.double().cpu().numpy(), "no-alloc lse at the limit")
    del q, k, v, out_ref, lse_ref, out, lse
    B, H = 74, 109  # 8066 rows
    assert B * H * (d + 2) > SCRATCH_FLOATS
    q = torch.zeros((B, 1, H, d), dtype=torch.float16, device="cuda")
    k = torch.zeros((B, Nk, H, d), dtype=torch.float16, device="cuda")
    out = torch.zeros_like(q)
    assert _call(lib.attn_fwd_decode_noalloc, q, k, k, out, None, 1, stream) == attn.ATTN_ERR_INVALID_ARG
    assert _call(lib.attn_fwd_decode_noalloc, q, k, k, out, None, 0, stream) == attn.ATTN_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert attn.get_status() == attn.ATTN_OK


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


def test_noalloc_allocates_nothing():
    """The device's default memory pool (where the allocating decode takes its partials)
    sees no allocation during a no-alloc call; the allocating call, as a control, does."""
    rt = pytest.importorskip("cuda.bindings.runtime")
    drv = pytest.importorskip("cuda.bindings.driver")
    lib = attn.load_library()
    stream = torch.cuda.current_stream()
    err, pool = rt.cudaDeviceGetDefaultMemPool(torch.cuda.current_device())
    assert err == rt.cudaError_t.cudaSuccess
    high = rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemHigh
    cur = rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemCurrent

    def attr(a):
        e, val = rt.cudaMemPoolGetAttribute(pool, a)
        assert e == rt.cudaError_t.cudaSuccess
        return int(val)

    def reset_high():
        (e,) = rt.cudaMemPoolSetAttribute(pool, high, drv.cuuint64_t(0))
        assert e == rt.cudaError_t.cudaSuccess

    B, H, Nk, d = 4, 8, 2048, 128
    q, k, v = (t.cuda() for t in make_inputs(B, H, 1, Nk, d, dtype="f16", seed=77))
    out = torch.empty_like(q)
    lse = torch.empty((B, H, 1), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    reset_high()
    base = attr(cur)
    assert attr(high) == base
    assert _call(lib.attn_fwd_decode_noalloc, q, k, v, out, lse, 4, stream) == attn.ATTN_OK
    torch.cuda.synchronize()
    assert attr(high) == base, "the no-alloc call took memory from the default pool"
    assert _call(lib.attn_fwd_decode, q, k, v, out, lse, 4, stream) == attn.ATTN_OK
    torch.cuda.synchronize()
    assert attr(high) >= base + B * H * 4 * (d + 2) * 4, "control: the probe saw no allocation"
    assert attn.get_status() == attn.ATTN_OK
