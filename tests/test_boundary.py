"""C-ABI boundary checks that need no GPU.

The library must load, export every entry point include/attn.h declares, and
reject bad arguments on the host with the documented code before any CUDA call
(the pointers below are never dereferenced: validation fails first).
"""
import ctypes
import math
import os
import re

import pytest

import attention_forward_tiled_b200 as attn
from attention_forward_tiled_b200 import build as abuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module")
def lib():
    abuild.build()
    return attn.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:ATTN_API\s+)?(?:const\s+)?\w+\s*\*?\s*(attn_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("attn_fwd", "attn_get_status", "attn_error_string"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in attn.h but not exported"
    assert set(declared_functions()) == set(attn.SIGNATURES), "binding and header disagree"


def test_only_the_c_abi_is_exported():
    """-fvisibility=hidden: nothing but the attn_* entry points leaks out of the library."""
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", attn.LIB_PATH], capture_output=True,
                         text=True).stdout
    syms = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert syms and all(s.startswith("attn_") for s in syms), sorted(syms)[:20]


def test_version_and_error_strings(lib):
    assert lib.attn_version() == 10000
    for code in (0, -1, -2, -3, -4, -5):
        assert len(lib.attn_error_string(code)) > 10
    assert b"unknown" in lib.attn_error_string(-99)


# fake, 256-byte aligned, non-overlapping device addresses (never dereferenced)
Q, K, V, O, L = (ctypes.c_void_p(0x100000000 * (i + 1)) for i in range(5))
NULL = ctypes.c_void_p(0)


def call(lib, q=Q, k=K, v=V, o=O, lse=L, B=1, H=2, Nq=128, Nk=128, d=64, causal=0,
         scale=0.125, dtype=0):
    return lib.attn_fwd(q, k, v, o, lse, B, H, Nq, Nk, d, causal, scale, dtype, NULL)


@pytest.mark.parametrize("kw,code", [
    (dict(q=NULL), attn.ATTN_ERR_INVALID_ARG),
    (dict(k=NULL), attn.ATTN_ERR_INVALID_ARG),
    (dict(v=NULL), attn.ATTN_ERR_INVALID_ARG),
    (dict(o=NULL), attn.ATTN_ERR_INVALID_ARG),
    (dict(B=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(H=-1), attn.ATTN_ERR_INVALID_ARG),
    (dict(Nq=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(Nk=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(d=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(causal=2), attn.ATTN_ERR_INVALID_ARG),
    (dict(scale=math.nan), attn.ATTN_ERR_INVALID_ARG),
    (dict(scale=math.inf), attn.ATTN_ERR_INVALID_ARG),
    (dict(d=96), attn.ATTN_ERR_UNSUPPORTED),
    (dict(d=256), attn.ATTN_ERR_UNSUPPORTED),
    (dict(dtype=2), attn.ATTN_ERR_UNSUPPORTED),
    (dict(q=ctypes.c_void_p(0x100000008)), attn.ATTN_ERR_INVALID_ARG),   # 8-byte aligned only
    (dict(o=ctypes.c_void_p(0x500000004)), attn.ATTN_ERR_INVALID_ARG),
    (dict(lse=ctypes.c_void_p(0x500000002)), attn.ATTN_ERR_INVALID_ARG),
    (dict(o=ctypes.c_void_p(0x100000000 + 4096)), attn.ATTN_ERR_INVALID_ARG),  # out overlaps q
    (dict(o=ctypes.c_void_p(0x200000000)), attn.ATTN_ERR_INVALID_ARG),         # out aliases k
    (dict(lse=ctypes.c_void_p(0x400000000 + 64)), attn.ATTN_ERR_INVALID_ARG),  # lse inside out
    (dict(Nk=1 << 30, H=64, d=128), attn.ATTN_ERR_INVALID_ARG),                # batch stride >= 2^40
])
def test_invalid_arguments_rejected_on_host(lib, kw, code):
    assert call(lib, **kw) == code


def test_decode_entry_validation(lib):
    assert lib.attn_fwd_decode(Q, K, V, O, L, 1, 2, 128, 64, 0.1, 0, -1, NULL) == attn.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_decode(NULL, K, V, O, L, 1, 2, 128, 64, 0.1, 0, 0, NULL) == attn.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_decode(Q, K, V, O, L, 1, 2, 128, 80, 0.1, 0, 0, NULL) == attn.ATTN_ERR_UNSUPPORTED


BT, SL = ctypes.c_void_p(0x700000000), ctypes.c_void_p(0x800000000)  # block table, seq lens


def paged(lib, q=Q, kc=K, vc=V, bt=BT, sl=SL, o=O, lse=L, B=2, H=4, d=128, num_blocks=64,
          page_size=16, max_blocks=32, scale=0.1, dtype=0, splits=0):
    return lib.attn_fwd_decode_paged(q, kc, vc, bt, sl, o, lse, B, H, d, num_blocks, page_size,
                                     max_blocks, scale, dtype, splits, NULL)


@pytest.mark.parametrize("kw,code", [
    (dict(bt=NULL), attn.ATTN_ERR_INVALID_ARG),
    (dict(sl=NULL), attn.ATTN_ERR_INVALID_ARG),
    (dict(kc=NULL), attn.ATTN_ERR_INVALID_ARG),
    (dict(num_blocks=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(max_blocks=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(splits=-1), attn.ATTN_ERR_INVALID_ARG),
    (dict(page_size=24), attn.ATTN_ERR_UNSUPPORTED),    # 128 is no multiple of 24
    (dict(page_size=4), attn.ATTN_ERR_UNSUPPORTED),     # below 8 rows
    (dict(page_size=192), attn.ATTN_ERR_UNSUPPORTED),   # above 128: multiples of 128 only
    (dict(d=80), attn.ATTN_ERR_UNSUPPORTED),
    (dict(max_blocks=1 << 28, page_size=16), attn.ATTN_ERR_INVALID_ARG),  # table length >= 2^31 keys
    (dict(bt=ctypes.c_void_p(0x700000002)), attn.ATTN_ERR_INVALID_ARG),   # misaligned table
    (dict(o=ctypes.c_void_p(0x200000000 + 4096)), attn.ATTN_ERR_INVALID_ARG),  # out inside k_cache
])
def test_paged_decode_entry_validation(lib, kw, code):
    assert paged(lib, **kw) == code


def test_prefill_entry_validation(lib):
    assert lib.attn_fwd_prefill(Q, K, V, NULL, L, 1, 2, 64, 64, 64, 0, 0.1, 0, NULL) == attn.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_prefill(Q, K, V, O, L, 1, 2, 64, 64, 32, 0, 0.1, 1, NULL) == attn.ATTN_ERR_UNSUPPORTED


EMB = ctypes.c_void_p(0x900000000)


def relpos(lib, q=Q, k=K, v=V, emb=EMB, o=O, lse=L, B=2, H=4, Nq=200, Nk=200, d=128, n_emb=401,
           R=200, causal=0, scale=0.1, dtype=0):
    return lib.attn_fwd_relpos(q, k, v, emb, o, lse, B, H, Nq, Nk, d, n_emb, R, causal, scale, dtype, NULL)


@pytest.mark.parametrize("kw,code", [
    (dict(emb=NULL), attn.ATTN_ERR_INVALID_ARG),
    (dict(R=-1), attn.ATTN_ERR_INVALID_ARG),
    (dict(n_emb=400), attn.ATTN_ERR_INVALID_ARG),                          # fewer than 2R + 1 rows
    (dict(emb=ctypes.c_void_p(0x900000008)), attn.ATTN_ERR_INVALID_ARG),   # 8-byte aligned only
    (dict(emb=ctypes.c_void_p(0x400000000 + 1024)), attn.ATTN_ERR_INVALID_ARG),  # out overlaps emb
    (dict(o=NULL), attn.ATTN_ERR_INVALID_ARG),
    (dict(causal=3), attn.ATTN_ERR_INVALID_ARG),
    (dict(d=32), attn.ATTN_ERR_UNSUPPORTED),
    (dict(dtype=5), attn.ATTN_ERR_UNSUPPORTED),
])
def test_relpos_entry_validation(lib, kw, code):
    assert relpos(lib, **kw) == code


def test_python_binding_rejects_cpu_tensors():
    import torch
    q = torch.zeros(1, 8, 1, 64, dtype=torch.float16)
    with pytest.raises(TypeError):
        attn.attn_fwd(q, q, q)


def test_package_import_is_lazy_and_loud_without_library(tmp_path):
    """A missing library raises instead of silently falling back."""
    from attention_forward_tiled_b200 import _binding
    saved = _binding._lib
    _binding._lib = None
    try:
        with pytest.raises(RuntimeError):
            _binding.load_library(str(tmp_path / "missing.so"))
    finally:
        _binding._lib = saved


def test_result_buffers_are_checked_before_the_call():
    """A caller's out/lse buffer must match exactly: the library writes all of it."""
    import torch
    from attention_forward_tiled_b200._binding import _check_buffer
    cpu = torch.device("cpu")
    ok = torch.empty(2, 3, 4, dtype=torch.float16)
    _check_buffer("out", ok, (2, 3, 4), torch.float16, cpu)
    bad = [
        torch.empty(2, 3, 3, dtype=torch.float16),                 # too small
        torch.empty(2, 3, 4, dtype=torch.float32),                 # wrong dtype
        torch.empty(2, 4, 3, dtype=torch.float16).transpose(1, 2),  # strided
        torch.empty(2, 3, 4, dtype=torch.float16, device="meta"),  # another device
        ok.numpy(),                                                # not a tensor
    ]
    for t in bad:
        with pytest.raises(ValueError):
            _check_buffer("out", t, (2, 3, 4), torch.float16, cpu)


def test_paged_binding_rejects_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 2, 64, dtype=torch.float16)
    kc = torch.zeros(4, 16, 2, 64, dtype=torch.float16)
    bt = torch.zeros(1, 4, dtype=torch.int32)
    sl = torch.ones(1, dtype=torch.int32)
    with pytest.raises(TypeError):
        attn.attn_fwd_decode_paged(q, kc, kc, bt, sl)
