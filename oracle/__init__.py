"""fp64 CPU oracle for the fused attention forward -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline / reference leg may import this package.  The CUDA library and its
Python binding never import it, and it imports nothing from them.

The arithmetic lives in ``attn_oracle.c`` (plain C, double precision, OpenMP
over (batch, head)); this module only marshals numpy arrays through ctypes.
Every input must already be the exact values the GPU path sees (fp16/bf16
rounded, then widened to float64).

Functions
---------
attn_fwd(q, k, v, causal, scale)            -> (o, lse)   definition order
attn_fwd_blocked(q, k, v, causal, scale, block_m=128, block_n=64) -> (o, lse)
attn_fwd_splitkv(q, k, v, splits, causal, scale) -> (o, lse)   split-KV + combine order
attn_probs(q, k, causal, scale)             -> p [B, H, Nq, Nk]
attn_fwd_relpos(q, k, v, emb, dist, causal, scale) -> (o, lse)   relative-position term
attn_bwd(q, k, v, dout, causal, scale)      -> (dq, dk, dv)
attn_fwd_paged(q, k_cache, v_cache, block_table, seq_lens, causal, scale) -> (o, lse)
indexer_score(q, kp, w, mask)               -> score [B, T, P]   lightning indexer
topk(score, k)                              -> idx [..., k]
num_threads() / set_num_threads(n)

Layouts: q, o [B, Nq, H, d]; k, v [B, Nk, H, d]; lse [B, H, Nq].
"""
import ctypes

import numpy as np

from . import build as _build

_lib = None
_lib_path = None


def load(path=None):
    """Load (building first if stale) the oracle library; returns the CDLL."""
    global _lib, _lib_path
    path = path or _build.LIB
    if _lib is not None and _lib_path == path:
        return _lib
    if path == _build.LIB and _build.needs_build():
        _build.build()
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    i, d = ctypes.c_int, ctypes.c_double
    lib.oracle_attn_fwd_f64.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, i, i, d]
    lib.oracle_attn_fwd_f64.restype = i
    lib.oracle_attn_fwd_blocked_f64.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, i, i, d, i, i]
    lib.oracle_attn_fwd_blocked_f64.restype = i
    lib.oracle_attn_probs_f64.argtypes = [dp, dp, dp, i, i, i, i, i, i, d]
    lib.oracle_attn_bwd_f64.restype = i
    lib.oracle_attn_bwd_f64.argtypes = [dp, dp, dp, dp, dp, dp, dp, i, i, i, i, i, i, d]
    ip = ctypes.POINTER(ctypes.c_int)
    lib.oracle_attn_fwd_relpos_f64.restype = i
    lib.oracle_attn_fwd_relpos_f64.argtypes = [dp, dp, dp, dp, ip, dp, dp, i, i, i, i, i, i, i, d]
    lib.oracle_attn_probs_f64.restype = i
    lib.oracle_attn_fwd_splitkv_f64.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, i, i, d, i]
    lib.oracle_attn_fwd_splitkv_f64.restype = i
    lib.oracle_attn_fwd_paged_f64.argtypes = [dp, dp, dp, ip, ip, dp, dp, i, i, i, i, i, i, i, i, d]
    lib.oracle_attn_fwd_paged_f64.restype = i
    lib.oracle_indexer_score_f64.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, i]
    lib.oracle_indexer_score_f64.restype = i
    lib.oracle_topk_f64.argtypes = [dp, i, i, i, ip]
    lib.oracle_topk_f64.restype = i
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = i
    lib.oracle_set_num_threads.argtypes = [i]
    lib.oracle_set_num_threads.restype = None
    if path == _build.LIB:
        _lib, _lib_path = lib, path
    return lib


def _f64(x):
    """Contiguous float64 numpy view/copy of a numpy array or CPU torch tensor."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _shapes(q, k, v=None):
    if q.ndim != 4 or k.ndim != 4:
        raise ValueError("q and k must be [B, N, H, d]")
    B, Nq, H, d = q.shape
    if k.shape[0] != B or k.shape[2] != H or k.shape[3] != d:
        raise ValueError("k must be [B, Nk, H, d] with q's B, H, d")
    if v is not None and v.shape != k.shape:
        raise ValueError("v must have k's shape")
    return B, H, Nq, k.shape[1], d


def attn_fwd(q, k, v, causal=False, scale=None, lib=None):
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Nq, Nk, d = _shapes(q, k, v)
    scale = float(1.0 / np.sqrt(d)) if scale is None else float(scale)
    o = np.zeros((B, Nq, H, d), dtype=np.float64)
    lse = np.zeros((B, H, Nq), dtype=np.float64)
    rc = (lib or load()).oracle_attn_fwd_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                             B, H, Nq, Nk, d, int(bool(causal)), scale)
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd_f64 failed ({rc})")
    return o, lse


def attn_fwd_blocked(q, k, v, causal=False, scale=None, block_m=128, block_n=64, lib=None):
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Nq, Nk, d = _shapes(q, k, v)
    scale = float(1.0 / np.sqrt(d)) if scale is None else float(scale)
    o = np.zeros((B, Nq, H, d), dtype=np.float64)
    lse = np.zeros((B, H, Nq), dtype=np.float64)
    rc = (lib or load()).oracle_attn_fwd_blocked_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                                     B, H, Nq, Nk, d, int(bool(causal)), scale,
                                                     int(block_m), int(block_n))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd_blocked_f64 failed ({rc})")
    return o, lse


def attn_fwd_splitkv(q, k, v, splits, causal=False, scale=None, lib=None):
    """The decode path's ordering: keys cut into `splits` ranges, per-range (m, l, o)
    states, then the combine step.  Same result as attn_fwd up to rounding."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Nq, Nk, d = _shapes(q, k, v)
    scale = float(1.0 / np.sqrt(d)) if scale is None else float(scale)
    o = np.zeros((B, Nq, H, d), dtype=np.float64)
    lse = np.zeros((B, H, Nq), dtype=np.float64)
    rc = (lib or load()).oracle_attn_fwd_splitkv_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                                     B, H, Nq, Nk, d, int(bool(causal)), scale,
                                                     int(splits))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd_splitkv_f64 failed ({rc})")
    return o, lse


def attn_probs(q, k, causal=False, scale=None, lib=None):
    q, k = _f64(q), _f64(k)
    B, H, Nq, Nk, d = _shapes(q, k)
    scale = float(1.0 / np.sqrt(d)) if scale is None else float(scale)
    p = np.zeros((B, H, Nq, Nk), dtype=np.float64)
    rc = (lib or load()).oracle_attn_probs_f64(_ptr(q), _ptr(k), _ptr(p),
                                               B, H, Nq, Nk, d, int(bool(causal)), scale)
    if rc != 0:
        raise RuntimeError(f"oracle_attn_probs_f64 failed ({rc})")
    return p


def attn_fwd_relpos(q, k, v, emb, dist, causal=False, scale=None, lib=None):
    """Attention whose scores carry the relative-position term scale * q_i . emb[dist[i, j]]
    (emb [n_emb, d], dist int [Nq, Nk], shared by every batch and head)."""
    q, k, v, emb = _f64(q), _f64(k), _f64(v), _f64(emb)
    B, H, Nq, Nk, d = _shapes(q, k, v)
    if hasattr(dist, "detach"):
        dist = dist.detach().cpu().numpy()
    dist = np.ascontiguousarray(dist, dtype=np.int32)
    if dist.shape != (Nq, Nk) or emb.ndim != 2 or emb.shape[1] != d:
        raise ValueError("dist must be [Nq, Nk] and emb [n_emb, d]")
    scale = float(1.0 / np.sqrt(d)) if scale is None else float(scale)
    o = np.zeros((B, Nq, H, d), dtype=np.float64)
    lse = np.zeros((B, H, Nq), dtype=np.float64)
    rc = (lib or load()).oracle_attn_fwd_relpos_f64(
        _ptr(q), _ptr(k), _ptr(v), _ptr(emb), dist.ctypes.data_as(ctypes.POINTER(ctypes.c_int)),
        _ptr(o), _ptr(lse), B, H, Nq, Nk, d, emb.shape[0], int(bool(causal)), scale)
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd_relpos_f64 failed ({rc})")
    return o, lse


def attn_bwd(q, k, v, dout, causal=False, scale=None, lib=None):
    """Gradients (dq, dk, dv) of attn_fwd's O for an upstream gradient dout [B, Nq, H, d]."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, Nq, Nk, d = _shapes(q, k, v)
    if dout.shape != q.shape:
        raise ValueError("dout must have q's shape")
    scale = float(1.0 / np.sqrt(d)) if scale is None else float(scale)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    rc = (lib or load()).oracle_attn_bwd_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq),
                                             _ptr(dk), _ptr(dv), B, H, Nq, Nk, d,
                                             int(bool(causal)), scale)
    if rc != 0:
        raise RuntimeError(f"oracle_attn_bwd_f64 failed ({rc})")
    return dq, dk, dv


def _i32(x):
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(x, dtype=np.int32)


def attn_fwd_paged(q, k_cache, v_cache, block_table, seq_lens, causal=False, scale=None, lib=None):
    """Attention of q [B, Lq, H, d] over a paged cache (k_cache, v_cache [num_blocks, page_size,
    H, d], block_table int [B, max_blocks], seq_lens int [B]); the Lq queries of a request are
    the last Lq positions of its sequence.  Returns (o [B, Lq, H, d], lse [B, H, Lq])."""
    q, k_cache, v_cache = _f64(q), _f64(k_cache), _f64(v_cache)
    block_table, seq_lens = _i32(block_table), _i32(seq_lens)
    if q.ndim != 4 or k_cache.ndim != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("q must be [B, Lq, H, d] and k_cache, v_cache [num_blocks, page_size, H, d]")
    B, Lq, H, d = q.shape
    num_blocks, page_size = k_cache.shape[:2]
    if k_cache.shape[2:] != (H, d) or block_table.ndim != 2 or block_table.shape[0] != B \
            or seq_lens.shape != (B,):
        raise ValueError("k_cache [num_blocks, page_size, H, d], block_table [B, max_blocks], seq_lens [B]")
    scale = float(1.0 / np.sqrt(d)) if scale is None else float(scale)
    o = np.zeros((B, Lq, H, d), dtype=np.float64)
    lse = np.zeros((B, H, Lq), dtype=np.float64)
    ip = ctypes.POINTER(ctypes.c_int)
    rc = (lib or load()).oracle_attn_fwd_paged_f64(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), block_table.ctypes.data_as(ip),
        seq_lens.ctypes.data_as(ip), _ptr(o), _ptr(lse), B, Lq, H, d, num_blocks, page_size,
        block_table.shape[1], int(bool(causal)), scale)
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd_paged_f64 failed ({rc})")
    return o, lse


def indexer_score(q, kp, w, mask=None, lib=None):
    """Lightning-indexer score [B, T, P] = sum_h w[b,t,h] * relu(q[b,t,h] . kp[b,p]) + mask
    (q [B, T, H, d], kp [B, P, d], w [B, T, H], mask [B, T, P] or None)."""
    q, kp, w = _f64(q), _f64(kp), _f64(w)
    if q.ndim != 4 or kp.ndim != 3 or w.ndim != 3:
        raise ValueError("q must be [B, T, H, d], kp [B, P, d] and w [B, T, H]")
    B, T, H, d = q.shape
    P = kp.shape[1]
    if kp.shape != (B, P, d) or w.shape != (B, T, H):
        raise ValueError("kp must be [B, P, d] and w [B, T, H] with q's B, T, H, d")
    mptr = None
    if mask is not None:
        mask = _f64(mask)
        if mask.shape != (B, T, P):
            raise ValueError("mask must be [B, T, P]")
        mptr = _ptr(mask)
    score = np.zeros((B, T, P), dtype=np.float64)
    rc = (lib or load()).oracle_indexer_score_f64(_ptr(q), _ptr(kp), _ptr(w), mptr, _ptr(score),
                                                  B, T, H, P, d)
    if rc != 0:
        raise RuntimeError(f"oracle_indexer_score_f64 failed ({rc})")
    return score


def topk(score, k, lib=None):
    """Positions of the k largest finite entries of each row of score [..., P], largest
    first, ties lowest position first; -1 where a row has fewer than k finite entries."""
    score = _f64(score)
    lead, P = score.shape[:-1], score.shape[-1]
    R = int(np.prod(lead)) if lead else 1
    idx = np.zeros((R, int(k)), dtype=np.int32)
    rc = (lib or load()).oracle_topk_f64(_ptr(score), R, P, int(k),
                                         idx.ctypes.data_as(ctypes.POINTER(ctypes.c_int)))
    if rc != 0:
        raise RuntimeError(f"oracle_topk_f64 failed ({rc})")
    return idx.reshape(*lead, int(k))


def num_threads():
    return load().oracle_num_threads()


def set_num_threads(n):
    load().oracle_set_num_threads(int(n))


__all__ = ["attn_fwd", "attn_fwd_blocked", "attn_fwd_splitkv", "attn_probs", "attn_fwd_relpos",
           "attn_bwd", "attn_fwd_paged", "indexer_score", "topk", "num_threads", "set_num_threads", "load"]
