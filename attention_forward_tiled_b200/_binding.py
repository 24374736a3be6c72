"""ctypes binding of libattn.so: argument marshalling only.

Every step of the attention forward runs in the CUDA kernels behind the C ABI
(include/attn.h).  PyTorch is used for device memory and streams; there is no
CPU or PyTorch fallback: if the library is missing or the call fails, an
exception is raised.
"""
import ctypes
import math
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libattn.so")

ATTN_F16, ATTN_BF16 = 0, 1
ATTN_OK = 0
ATTN_ERR_INVALID_ARG = -1
ATTN_ERR_UNSUPPORTED = -2
ATTN_ERR_CUDA = -3
ATTN_ERR_TIMEOUT = -4
ATTN_ERR_RANGE = -5

# every entry point declared in include/attn.h: name -> (restype, argtypes)
_vp, _i, _f, _u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_ulonglong
SIGNATURES = {
    "attn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp]),
    "attn_fwd_prefill": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp]),
    "attn_fwd_decode": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _i, _vp]),
    "attn_fwd_decode_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _i, _vp]),
    "attn_fwd_decode_paged": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i,
                                   _i, _vp]),
    "attn_fwd_paged": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f,
                            _i, _i, _vp]),
    "attn_fwd_relpos": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f, _i, _vp]),
    "attn_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp]),
    "attn_indexer_score": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "attn_topk": (_i, [_vp, _i, _i, _i, _vp, _vp]),
    "attn_get_status": (_i, [_vp]),
    "attn_error_string": (ctypes.c_char_p, [_i]),
    "attn_version": (_i, []),
    "attn_debug_set": (_i, [_i, _u64]),
}

_lib = None


class AttnError(RuntimeError):
    def __init__(self, code, where=""):
        self.code = code
        msg = error_string(code) if _lib is not None else f"attn status {code}"
        super().__init__(f"{where}: {msg}" if where else msg)


def load_library(path=LIB_PATH):
    """Load libattn.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built: run `python -m attention_forward_tiled_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def error_string(code):
    return load_library().attn_error_string(int(code)).decode()


def version():
    return load_library().attn_version()


def debug_set(inject=0, wait_timeout_ns=0):
    return load_library().attn_debug_set(int(inject), int(wait_timeout_ns))


def _dtype_code(t):
    import torch
    if t == torch.float16:
        return ATTN_F16
    if t == torch.bfloat16:
        return ATTN_BF16
    raise TypeError(f"unsupported dtype {t}; expected float16 or bfloat16")


def _check(q, k, v):
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor")
        if t.dim() != 4:
            raise ValueError(f"{name} must be [batch, seq, heads, head_dim]")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    if not (q.device == k.device == v.device):
        raise ValueError("q, k, v must be on one device")
    B, Nq, H, d = q.shape
    if k.shape[0] != B or k.shape[2] != H or k.shape[3] != d or v.shape != k.shape:
        raise ValueError("k and v must be [B, Nk, H, d] with q's B, H, d")
    return B, H, Nq, k.shape[1], d


def _check_buffer(name, t, shape, dtype, device):
    """A caller-supplied result buffer must be exactly what the library writes: it fills
    the whole of it, so a smaller or strided tensor, or one on another device, would be
    written out of bounds."""
    import torch
    if not isinstance(t, torch.Tensor) or t.device != device:
        raise ValueError(f"{name} must be a tensor on {device}")
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)}")


def _stream_ptr(stream, device):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def attn_fwd(q, k, v, causal=False, scale=None, out=None, lse=None, return_lse=True,
             stream=None, path="auto", splits=0):
    """Fused attention forward on CUDA tensors laid out [B, N, H, d].

    Returns (out, lse): out [B, Nq, H, d] in q's dtype, lse [B, H, Nq] float32
    (None when return_lse is False and no lse buffer is given).
    path: "auto" (decode kernels when Nq == 1), "prefill" or "decode".
    """
    import torch
    lib = load_library()
    B, H, Nq, Nk, d = _check(q, k, v)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _check_buffer("out", out, q.shape, q.dtype, q.device)
    if lse is not None:
        _check_buffer("lse", lse, (B, H, Nq), torch.float32, q.device)
    dt = _dtype_code(q.dtype)
    lse_ptr = ctypes.c_void_p(lse.data_ptr() if lse is not None else 0)
    with torch.cuda.device(q.device):
        s = _stream_ptr(stream, q.device)
        ptrs = (ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()), lse_ptr)
        if path == "auto":
            rc = lib.attn_fwd(*ptrs, B, H, Nq, Nk, d, int(bool(causal)), scale, dt, s)
        elif path == "prefill":
            rc = lib.attn_fwd_prefill(*ptrs, B, H, Nq, Nk, d, int(bool(causal)), scale, dt, s)
        elif path == "decode":
            rc = lib.attn_fwd_decode(*ptrs, B, H, Nk, d, scale, dt, int(splits), s)
        else:
            raise ValueError(f"unknown path {path!r}")
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd")
    return out, lse


def attn_fwd_relpos(q, k, v, emb, R, causal=False, scale=None, out=None, lse=None, return_lse=True,
                    stream=None):
    """Attention whose scores carry the relative-position term scale * q_i . emb[dist(i, j)],
    dist(i, j) = clamp(i - j, -R, R) + R (emb [n_emb, d] in q's dtype, n_emb >= 2R + 1).

    q, k, v [B, N, H, d] as attn_fwd (B may be batch x blocks of a block-local model).
    Returns (out, lse) as attn_fwd."""
    import torch
    lib = load_library()
    B, H, Nq, Nk, d = _check(q, k, v)
    if emb.dim() != 2 or emb.shape[1] != d or emb.dtype != q.dtype or emb.device != q.device:
        raise ValueError("emb must be [n_emb, d] in q's dtype on q's device")
    if not emb.is_contiguous():
        raise ValueError("emb must be contiguous")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _check_buffer("out", out, q.shape, q.dtype, q.device)
    if lse is not None:
        _check_buffer("lse", lse, (B, H, Nq), torch.float32, q.device)
    with torch.cuda.device(q.device):
        rc = lib.attn_fwd_relpos(
            ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
            ctypes.c_void_p(emb.data_ptr()), ctypes.c_void_p(out.data_ptr()),
            ctypes.c_void_p(lse.data_ptr() if lse is not None else 0), B, H, Nq, Nk, d, emb.shape[0],
            int(R), int(bool(causal)), scale, _dtype_code(q.dtype), _stream_ptr(stream, q.device))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_relpos")
    return out, lse


def attn_fwd_decode_paged(q, k_cache, v_cache, block_table, seq_lens, scale=None, out=None,
                          lse=None, return_lse=True, stream=None, splits=0):
    """Single-query attention over a paged key/value cache.

    q [B, 1, H, d]; k_cache, v_cache [num_blocks, page_size, H, d] (q's dtype);
    block_table [B, max_blocks] and seq_lens [B], int32 CUDA tensors.  Request b
    attends to its first seq_lens[b] keys, stored page by page in the pages its
    block-table row lists.  Returns (out [B, 1, H, d], lse [B, H] float32 or None).
    """
    import torch
    lib = load_library()
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                    ("block_table", block_table), ("seq_lens", seq_lens)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous CUDA tensor")
        if t.device != q.device:
            raise ValueError(f"{name} must be on q's device {q.device}")
    if q.dim() != 4 or q.shape[1] != 1:
        raise ValueError("q must be [batch, 1, heads, head_dim]")
    B, _, H, d = q.shape
    if not (q.dtype == k_cache.dtype == v_cache.dtype):
        raise TypeError("q, k_cache, v_cache must share one dtype")
    if k_cache.shape != v_cache.shape or k_cache.dim() != 4 or k_cache.shape[2:] != (H, d):
        raise ValueError("k_cache and v_cache must be [num_blocks, page_size, heads, head_dim]")
    if block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be an int32 [batch, max_blocks] tensor")
    if seq_lens.dtype != torch.int32 or seq_lens.shape != (B,):
        raise ValueError("seq_lens must be an int32 [batch] tensor")
    num_blocks, page_size = k_cache.shape[0], k_cache.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    _check_buffer("out", out, q.shape, q.dtype, q.device)
    if lse is not None:
        _check_buffer("lse", lse, (B, H), torch.float32, q.device)
    with torch.cuda.device(q.device):
        rc = lib.attn_fwd_decode_paged(
            ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k_cache.data_ptr()),
            ctypes.c_void_p(v_cache.data_ptr()), ctypes.c_void_p(block_table.data_ptr()),
            ctypes.c_void_p(seq_lens.data_ptr()), ctypes.c_void_p(out.data_ptr()),
            ctypes.c_void_p(lse.data_ptr() if lse is not None else 0), B, H, d, num_blocks,
            page_size, block_table.shape[1], scale, _dtype_code(q.dtype), int(splits),
            _stream_ptr(stream, q.device))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_decode_paged")
    return out, lse


def attn_fwd_paged(q, k_cache, v_cache, block_table, seq_lens, causal=False, scale=None, out=None,
                   lse=None, return_lse=True, stream=None, splits=0):
    """Lq <= 16 query tokens per request over a paged key/value cache (tensor cores).

    q [B, Lq, H, d]; k_cache, v_cache [num_blocks, page_size, H, d] (q's dtype);
    block_table [B, max_blocks] and seq_lens [B], int32 CUDA tensors.  Request b's
    tokens are the last Lq positions of its seq_lens[b] keys; with causal, token i
    sees keys up to its own position.  Returns (out [B, Lq, H, d], lse [B, H, Lq]
    float32 or None).
    """
    import torch
    lib = load_library()
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                    ("block_table", block_table), ("seq_lens", seq_lens)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous CUDA tensor")
        if t.device != q.device:
            raise ValueError(f"{name} must be on q's device {q.device}")
    if q.dim() != 4:
        raise ValueError("q must be [batch, tokens, heads, head_dim]")
    B, Lq, H, d = q.shape
    if not (q.dtype == k_cache.dtype == v_cache.dtype):
        raise TypeError("q, k_cache, v_cache must share one dtype")
    if k_cache.shape != v_cache.shape or k_cache.dim() != 4 or k_cache.shape[2:] != (H, d):
        raise ValueError("k_cache and v_cache must be [num_blocks, page_size, heads, head_dim]")
    if block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be an int32 [batch, max_blocks] tensor")
    if seq_lens.dtype != torch.int32 or seq_lens.shape != (B,):
        raise ValueError("seq_lens must be an int32 [batch] tensor")
    num_blocks, page_size = k_cache.shape[0], k_cache.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
    _check_buffer("out", out, q.shape, q.dtype, q.device)
    if lse is not None:
        _check_buffer("lse", lse, (B, H, Lq), torch.float32, q.device)
    with torch.cuda.device(q.device):
        rc = lib.attn_fwd_paged(
            ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k_cache.data_ptr()),
            ctypes.c_void_p(v_cache.data_ptr()), ctypes.c_void_p(block_table.data_ptr()),
            ctypes.c_void_p(seq_lens.data_ptr()), ctypes.c_void_p(out.data_ptr()),
            ctypes.c_void_p(lse.data_ptr() if lse is not None else 0), B, H, Lq, d, num_blocks,
            page_size, block_table.shape[1], int(bool(causal)), scale, _dtype_code(q.dtype),
            int(splits), _stream_ptr(stream, q.device))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_paged")
    return out, lse


def attn_bwd(q, k, v, o, lse, dout, causal=False, scale=None, stream=None, dq=None, dk=None, dv=None):
    """Gradients (dq, dk, dv) of attn_fwd for the upstream gradient dout, from the
    forward's inputs, its output o and its lse (all CUDA tensors, [B, N, H, d] layout)."""
    import torch
    lib = load_library()
    B, H, Nq, Nk, d = _check(q, k, v)
    for name, t in (("o", o), ("dout", dout)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous CUDA tensor")
    _check_buffer("o", o, q.shape, q.dtype, q.device)
    _check_buffer("dout", dout, q.shape, q.dtype, q.device)
    _check_buffer("lse", lse, (B, H, Nq), torch.float32, q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_buffer("dq", dq, q.shape, q.dtype, q.device)
    _check_buffer("dk", dk, k.shape, k.dtype, q.device)
    _check_buffer("dv", dv, v.shape, v.dtype, q.device)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    with torch.cuda.device(q.device):
        rc = lib.attn_bwd(ptr(q), ptr(k), ptr(v), ptr(o), ptr(dout), ptr(lse), ptr(dq), ptr(dk), ptr(dv),
                          B, H, Nq, Nk, d, int(bool(causal)), scale, _dtype_code(q.dtype),
                          _stream_ptr(stream, q.device))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_bwd")
    return dq, dk, dv


def indexer_score(q, kp, w, mask=None, out=None, stream=None):
    """Lightning-indexer score: q [B, T, H, d], kp [B, P, d] (fp16/bf16), w [B, T, H]
    float32, mask [B, T, P] float16 (0 / -inf) or None.  Returns score [B, T, P] float32."""
    import torch
    lib = load_library()
    for name, t in (("q", q), ("kp", kp), ("w", w)) + ((("mask", mask),) if mask is not None else ()):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous CUDA tensor")
        if t.device != q.device:
            raise ValueError(f"{name} must be on q's device {q.device}")
    if q.dim() != 4 or kp.dim() != 3:
        raise ValueError("q must be [B, T, H, d] and kp [B, P, d]")
    B, T, H, d = q.shape
    P = kp.shape[1]
    if kp.shape[0] != B or kp.shape[2] != d or kp.dtype != q.dtype:
        raise ValueError("kp must be [B, P, d] in q's dtype")
    if w.dtype != torch.float32 or tuple(w.shape) != (B, T, H):
        raise ValueError("w must be a float32 [B, T, H] tensor")
    if mask is not None and (mask.dtype != torch.float16 or tuple(mask.shape) != (B, T, P)):
        raise ValueError("mask must be a float16 [B, T, P] tensor")
    if out is None:
        out = torch.empty((B, T, P), dtype=torch.float32, device=q.device)
    _check_buffer("out", out, (B, T, P), torch.float32, q.device)
    with torch.cuda.device(q.device):
        rc = lib.attn_indexer_score(
            ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kp.data_ptr()), ctypes.c_void_p(w.data_ptr()),
            ctypes.c_void_p(mask.data_ptr() if mask is not None else 0), ctypes.c_void_p(out.data_ptr()),
            B, T, H, P, d, _dtype_code(q.dtype), _stream_ptr(stream, q.device))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_indexer_score")
    return out


def topk(score, k, out=None, stream=None):
    """Positions [..., k] int32 of the k largest finite scores of each row of score [..., P]
    (float32 CUDA tensor), largest first, ties to the lower position, -1 padding."""
    import torch
    lib = load_library()
    if not isinstance(score, torch.Tensor) or not score.is_cuda or not score.is_contiguous() \
            or score.dtype != torch.float32:
        raise TypeError("score must be a contiguous float32 CUDA tensor")
    P = score.shape[-1]
    R = score.numel() // P
    shape = tuple(score.shape[:-1]) + (int(k),)
    if out is None:
        out = torch.empty(shape, dtype=torch.int32, device=score.device)
    _check_buffer("out", out, shape, torch.int32, score.device)
    with torch.cuda.device(score.device):
        rc = lib.attn_topk(ctypes.c_void_p(score.data_ptr()), R, P, int(k), ctypes.c_void_p(out.data_ptr()),
                           _stream_ptr(stream, score.device))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_topk")
    return out


def get_status(stream=None, device=None):
    """Synchronise the stream and return (then clear) the device status word."""
    import torch
    lib = load_library()
    device = device if device is not None else torch.cuda.current_device()
    with torch.cuda.device(device):
        return lib.attn_get_status(_stream_ptr(stream, device))


class HostRunner:
    """End-to-end call from host buffers: H2D copies, the kernel, D2H copy of O (and lse).

    Device buffers are allocated once at construction; each call copies the host
    tensors (pinned for asynchronous copies) to them on the runner's stream,
    runs attn_fwd and copies the results back into pinned host tensors.
    """

    def __init__(self, B, H, Nq, Nk, d, dtype, device="cuda", causal=False, scale=None,
                 with_lse=True):
        import torch
        self.device = torch.device(device)
        self.causal, self.scale = causal, scale
        self.q = torch.empty((B, Nq, H, d), dtype=dtype, device=self.device)
        self.k = torch.empty((B, Nk, H, d), dtype=dtype, device=self.device)
        self.v = torch.empty_like(self.k)
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty((B, H, Nq), dtype=torch.float32, device=self.device) if with_lse else None
        self.out_host = torch.empty(self.out.shape, dtype=dtype, pin_memory=True)
        self.lse_host = (torch.empty(self.lse.shape, dtype=torch.float32, pin_memory=True)
                         if with_lse else None)

    @property
    def h2d_bytes(self):
        return sum(t.numel() * t.element_size() for t in (self.q, self.k, self.v))

    @property
    def d2h_bytes(self):
        n = self.out.numel() * self.out.element_size()
        return n + (self.lse.numel() * 4 if self.lse is not None else 0)

    def __call__(self, q_host, k_host, v_host, stream=None):
        import torch
        stream = stream or torch.cuda.current_stream(self.device)
        with torch.cuda.stream(stream):
            self.q.copy_(q_host, non_blocking=True)
            self.k.copy_(k_host, non_blocking=True)
            self.v.copy_(v_host, non_blocking=True)
            attn_fwd(self.q, self.k, self.v, causal=self.causal, scale=self.scale, out=self.out,
                     lse=self.lse, stream=stream)
            self.out_host.copy_(self.out, non_blocking=True)
            if self.lse is not None:
                self.lse_host.copy_(self.lse, non_blocking=True)
        return self.out_host, self.lse_host
