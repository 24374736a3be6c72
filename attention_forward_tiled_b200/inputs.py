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

# The decode workload over a paged cache: the same 16 requests x 4096 keys, stored in
# randomly placed 16-key pages (a common serving page size).  The speculative-decoding
# variant scores 8 query tokens per request together (causal within the request).
PAGED_WORKLOADS = {
    "decode_paged16": dict(B=16, H=32, d=128, seq_lens=[4096] * 16, page_size=16, dtype="f16",
                           scale=1.0 / math.sqrt(128), seed=6, Lq=1, causal=False),
    "spec8_paged16": dict(B=16, H=32, d=128, seq_lens=[4096] * 16, page_size=16, dtype="f16",
                          scale=1.0 / math.sqrt(128), seed=7, Lq=8, causal=True),
}


# The lightning-indexer workload: 4096 query tokens of 4 indexer heads (the head count the
# llama.cpp report's CUDA kernel supports) against 4096 pooled keys, d 128, the unweighted
# form (w = 1/sqrt(d)) with the bottom-right f16 pool mask; top-k keeps 512 per token.
INDEXER_WORKLOADS = {
    "indexer_h4": dict(B=1, T=4096, H=4, P=4096, d=128, dtype="f16", seed=8, weights="constant",
                       masked=True, k=512),
}


# Block-local attention with the relative-position term (the Granite-Speech conformer of the
# vLLM "PR #42933" page): the sequence is cut into blocks of 200 tokens (B counts batch x
# blocks), 8 heads of d 128, every distance within a block distinct (R = 199 -> 399
# embedding rows).  The page gives no sizes; these are a plain reading of a block-local
# speech encoder.
RELPOS_WORKLOADS = {
    "relpos_block200": dict(B=512, H=8, Nq=200, Nk=200, d=128, R=199, causal=False, dtype="f16",
                            scale=1.0 / math.sqrt(128), seed=9),
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


def make_paged_inputs(B, H, d, seq_lens, page_size, dtype="f16", seed=0, max_blocks=None,
                      spare_pages=3, Lq=1):
    """Seeded paged decode inputs (CPU tensors): q [B, Lq, H, d]; k_cache, v_cache
    [num_blocks, page_size, H, d]; block_table [B, max_blocks] int32 (-1 past each
    sequence); seq_lens [B] int32.  The pages of all requests (plus `spare_pages`
    unused ones) are a random permutation of the cache, so no request's pages are
    contiguous.  Draw order: q, the page permutation, k_cache, v_cache."""
    g = torch.Generator("cpu").manual_seed(int(seed))
    npages = [(int(L) + page_size - 1) // page_size for L in seq_lens]
    max_blocks = max(max(npages), 1) if max_blocks is None else int(max_blocks)
    num_blocks = sum(npages) + spare_pages
    q = torch.randn(B, Lq, H, d, generator=g, dtype=torch.float32)
    perm = torch.randperm(num_blocks, generator=g)
    k_cache = torch.randn(num_blocks, page_size, H, d, generator=g, dtype=torch.float32)
    v_cache = torch.randn(num_blocks, page_size, H, d, generator=g, dtype=torch.float32)
    block_table = torch.full((B, max_blocks), -1, dtype=torch.int32)
    nxt = 0
    for b, n in enumerate(npages):
        block_table[b, :n] = perm[nxt:nxt + n].to(torch.int32)
        nxt += n
    dt = DTYPES[dtype]
    return (q.to(dt), k_cache.to(dt), v_cache.to(dt), block_table,
            torch.tensor([int(L) for L in seq_lens], dtype=torch.int32))


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


def make_indexer_inputs(B, T, H, P, d, dtype="f16", seed=0, weights="random", masked=True):
    """Seeded lightning-indexer inputs (CPU tensors): q [B, T, H, d], kp [B, P, d] in the
    dtype; w [B, T, H] float32 (randn, or 1/sqrt(d) everywhere for the unweighted form);
    mask [B, T, P] float16 with 0 where pool entry p is visible to token t (p <= t + P - T,
    the bottom-right rule) and -inf elsewhere, or None.  Draw order: q, kp, w."""
    g = torch.Generator("cpu").manual_seed(int(seed))
    q = torch.randn(B, T, H, d, generator=g, dtype=torch.float32)
    kp = torch.randn(B, P, d, generator=g, dtype=torch.float32)
    if weights == "random":
        w = torch.randn(B, T, H, generator=g, dtype=torch.float32)
    else:
        w = torch.full((B, T, H), 1.0 / math.sqrt(d), dtype=torch.float32)
    mask = None
    if masked:
        t = torch.arange(T).view(T, 1)
        p = torch.arange(P).view(1, P)
        mask = torch.where(p <= t + (P - T), 0.0, float("-inf")).to(torch.float16)
        mask = mask.expand(B, T, P).contiguous()
    dt = DTYPES[dtype]
    return q.to(dt), kp.to(dt), w, mask


def make_relpos_inputs(B, H, Nq, Nk, d, R, dtype="f16", seed=0, **_):
    """q, k, v as make_inputs and the relative-position table emb [2R + 1, d] (randn), CPU
    tensors in the dtype.  Draw order: q, k, v, emb."""
    g = torch.Generator("cpu").manual_seed(int(seed))
    q = torch.randn(B, Nq, H, d, generator=g, dtype=torch.float32)
    k = torch.randn(B, Nk, H, d, generator=g, dtype=torch.float32)
    v = torch.randn(B, Nk, H, d, generator=g, dtype=torch.float32)
    emb = torch.randn(2 * R + 1, d, generator=g, dtype=torch.float32)
    dt = DTYPES[dtype]
    return q.to(dt), k.to(dt), v.to(dt), emb.to(dt)
