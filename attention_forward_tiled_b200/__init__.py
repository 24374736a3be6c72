"""B200 (sm_100a) fused attention forward behind a C ABI (libattn.so).

    from attention_forward_tiled_b200 import attn_fwd
    out, lse = attn_fwd(q, k, v, causal=True)      # q, k, v: [B, N, H, d] fp16/bf16 CUDA tensors

The library is loaded on first use; a missing build raises instead of falling
back to anything else.  ``inputs`` holds the seeded synthetic workloads.
"""
from ._binding import (ATTN_BF16, ATTN_ERR_CUDA, ATTN_ERR_INVALID_ARG, ATTN_ERR_RANGE, ATTN_ERR_TIMEOUT,
                       ATTN_ERR_UNSUPPORTED, ATTN_F16, ATTN_OK, LIB_PATH, SIGNATURES, AttnError,
                       HostRunner, attn_bwd, attn_fwd, attn_fwd_decode_paged, attn_fwd_paged, attn_fwd_relpos, debug_set, error_string,
                       get_status, indexer_score, load_library, topk, version)

__all__ = [
    "attn_fwd", "attn_bwd", "attn_fwd_decode_paged", "attn_fwd_paged", "attn_fwd_relpos", "indexer_score", "topk", "get_status", "error_string", "version", "debug_set", "load_library",
    "HostRunner", "AttnError", "LIB_PATH", "SIGNATURES", "ATTN_OK", "ATTN_ERR_INVALID_ARG",
    "ATTN_ERR_UNSUPPORTED", "ATTN_ERR_CUDA", "ATTN_ERR_TIMEOUT", "ATTN_ERR_RANGE", "ATTN_F16", "ATTN_BF16",
]
