"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws random numbers and names workloads; it contains none of
the attention arithmetic, so the oracle and the CUDA path can both be fed from
it without sharing any computation.

Recipe (stands in for the LLaMA-7B seq-4096 attention shapes of the
FlashAttention/ops-transformer article, section "如何使用": [batch, seq,
heads, head_dim] fp16 tensors drawn with randn):
  g = torch.Generator('cpu').manual_seed(seed)
  q = randn(B, Nq, H, d), k = randn(B, Nk, H, d) * k_mult, v = randn(B, Nk, H, d)
  (fp32 draws, in that order), then each is cast to the workload's dtype.
"""
import math

import torch

DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}

# The five workloads plus the ragged-tail variant of the long causal one.
WORKLOADS = {
    "tiny": dict(B=1, H=2, Nq=128, Nk=128, d=64, causal=False, dtype="f16",
                 scale=1.0 / math.sqrt(64), seed=1, k_mult=1.0),
    "causal4k": dict(B=4, H=32, Nq=4096, Nk=4096, d=128, causal=True, dtype="f16",
                     scale=1.0 / math.sqrt(128), seed=2, k_mult=1.0),
    "bf16_k3": dict(B=8, H=16, Nq=1024, Nk=1024, d=64, causal=False, dtype="bf16",
                    scale=1.0 / math.sqrt(64), seed=3, k_mult=3.0),
    "causal8k": dict(B=1, H=32, Nq=8192, Nk=8192, d=128, causal=True, dtype="f16",
                     scale=1.0 / math.sqrt(128), seed=4, k_mult=1.0),
    "causal8000": dict(B=1, H=32, Nq=8000, Nk=8000, d=128, causal=True, dtype="f16",
                       scale=1.0 / math.sqrt(128), seed=40, k_mult=1.0),
    "decode": dict(B=16, H=32, Nq=1, Nk=4096, d=128, causal=False, dtype="f16",
                   scale=1.0 / math.sqrt(128), seed=5, k_mult=1.0),
}


def make_inputs(B, H, Nq, Nk, d, dtype="f16", seed=0, k_mult=1.0, **_):
    """Return CPU tensors (q, k, v) in [B, N, H, d] layout and the given dtype."""
    g = torch.Generator("cpu").manual_seed(int(seed))
    q = torch.randn(B, Nq, H, d, generator=g, dtype=torch.float32)
    k = torch.randn(B, Nk, H, d, generator=g, dtype=torch.float32)
    v = torch.randn(B, Nk, H, d, generator=g, dtype=torch.float32)
    if k_mult != 1.0:
        k = k * k_mult
    dt = DTYPES[dtype]
    return q.to(dt), k.to(dt), v.to(dt)


def workload_inputs(name):
    """(q, k, v) CPU tensors for a named workload."""
    return make_inputs(**WORKLOADS[name])


def flops(B, H, Nq, Nk, d, causal, **_):
    """Nominal forward FLOPs: 4*B*H*Nq*Nk*d, halved when causal (the metric's formula)."""
    f = 4.0 * B * H * Nq * Nk * d
    return f / 2.0 if causal else f


def kv_bytes(B, H, Nk, d, dtype="f16", **_):
    """Bytes of K plus V (the decode metric's numerator)."""
    return 2 * B * Nk * H * d * torch.tensor([], dtype=DTYPES[dtype]).element_size()
