"""Failure detection on the GPU without faulting it.

The prefill producer is told (test hook) to skip its first Q-tile copy, so the
matrix-multiply issuer's bounded mbarrier wait for that tile runs out after a
short limit.  The kernel must record ATTN_ERR_TIMEOUT in the device status
word, every role must leave its loops (no trap, no hang), and the context must
stay usable: the next normal call returns correct results and a clean status.
"""
import math

import pytest
import torch

import oracle
import attention_forward_tiled_b200 as attn
from attention_forward_tiled_b200.inputs import make_inputs
from tests.parity import assert_lse_close, assert_o_close

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_context_survives():
    q, k, v = make_inputs(1, 2, 256, 384, 128, seed=31)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    assert attn.get_status() == attn.ATTN_OK
    attn.debug_set(inject=1, wait_timeout_ns=20_000_000)  # 20 ms limit per wait
    try:
        attn.attn_fwd(qd, kd, vd, causal=True)
        status = attn.get_status()
    finally:
        attn.debug_set(0, 0)
    assert status == attn.ATTN_ERR_TIMEOUT
    assert attn.get_status() == attn.ATTN_OK  # reading the word cleared it

    out, lse = attn.attn_fwd(qd, kd, vd, causal=True)
    assert attn.get_status() == attn.ATTN_OK
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, causal=True, scale=1 / math.sqrt(128))
    assert_o_close(out, o_ref, torch.float16, "after recovery")
    assert_lse_close(lse, lse_ref, "after recovery")


def test_error_strings_from_the_device_path():
    assert "TIMEOUT" in attn.error_string(attn.ATTN_ERR_TIMEOUT)
