"""Per-kernel resources as ptxas reports them, no GPU.

The library's translation unit is compiled once more for sm_100a with the
build's own flags plus -Xptxas -v, and ptxas's per-entry report is checked:
- every kernel fits its launch (registers x threads within the 64 K register
  file for the one CTA per SM the persistent kernels run);
- the decode and combine kernels spill nothing;
- the prefill kernels' spill traffic stays at or below what it is today (a
  regression guard: growth there lands in the softmax's inner loop).
"""
import os
import re
import shutil
import subprocess

import pytest

from attention_forward_tiled_b200 import build as abuild

THREADS = {"attn_prefill_kernel": 384, "attn_decode_partial_kernel": 160,
           "attn_decode_combine_kernel": 128, "attn_mq_partial_kernel": 192,
           "attn_mq_combine_kernel": 128, "attn_indexer_score_kernel": 352,
           "attn_topk_kernel": 512, "attn_bwd_kernel": 320, "attn_bwd_pre_kernel": 128,
           "attn_bwd_dq_kernel": 256, "attn_relpos_kernel": 320}
# bytes of spill stores / loads per prefill instantiation (head_dim, bf16) at this version
# (d = 64: the softmax warps' scores stay in registers; what is left is outside the step loop)
PREFILL_SPILL_CEILING = {(64, False): (8, 44), (64, True): (8, 48),
                         (128, False): (8, 8), (128, True): (8, 8)}
# d = 64 re-balances registers between warpgroups (setmaxnreg) from exactly this count at launch
PREFILL_LAUNCH_REGS = 168


@pytest.fixture(scope="module")
def ptxas_report(tmp_path_factory):
    if shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"):
        pytest.skip("nvcc not available")
    out = tmp_path_factory.mktemp("ptxas") / "attn_api.o"
    flags = [f for f in abuild.NVCC_FLAGS if f not in ("--shared", "-cudart", "static")]
    cmd = [abuild.nvcc_path(), *flags, "-Xptxas", "-v", "-I", abuild.INCLUDE, "-I", abuild.CSRC,
           "-c", *abuild.SOURCES, "-o", str(out)]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stderr[-3000:]
    entries = {}
    current = None
    for line in res.stderr.splitlines():
        m = re.search(r"Compiling entry function '(\w+)'", line)
        if m:
            current = m.group(1)
            entries[current] = {}
            continue
        if current is None:
            continue
        m = re.search(r"(\d+) bytes stack frame, (\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and "spill_stores" not in entries[current]:
            entries[current].update(stack=int(m.group(1)), spill_stores=int(m.group(2)),
                                    spill_loads=int(m.group(3)))
        m = re.search(r"Used (\d+) registers", line)
        if m:
            entries[current]["registers"] = int(m.group(1))
    return entries


def kernel_kind(mangled):
    for name in THREADS:
        if name in mangled:
            return name
    return None


def template_args(mangled):
    m = re.search(r"ILi(\d+)ELb([01])E", mangled)
    return int(m.group(1)), m.group(2) == "1"



def test_every_kernel_is_reported(ptxas_report):
    kinds = [kernel_kind(k) for k in ptxas_report]
    assert kinds.count("attn_prefill_kernel") == 4      # d 64/128 x fp16/bf16
    assert kinds.count("attn_decode_partial_kernel") == 8  # x dense/paged
    assert kinds.count("attn_decode_combine_kernel") == 4
    assert kinds.count("attn_mq_partial_kernel") == 4
    assert kinds.count("attn_mq_combine_kernel") == 4
    assert kinds.count("attn_indexer_score_kernel") == 4
    assert kinds.count("attn_topk_kernel") == 2
    assert kinds.count("attn_bwd_kernel") == 4
    assert kinds.count("attn_bwd_pre_kernel") == 4
    assert kinds.count("attn_bwd_dq_kernel") == 2
    assert kinds.count("attn_relpos_kernel") == 4
    assert all(kinds)


def test_registers_fit_the_launch(ptxas_report):
    for name, info in ptxas_report.items():
        threads = THREADS[kernel_kind(name)]
        assert info["registers"] * threads <= 65536, (name, info)


def test_non_prefill_kernels_do_not_spill(ptxas_report):
    for name, info in ptxas_report.items():
        if kernel_kind(name) != "attn_prefill_kernel":
            assert info["spill_stores"] == 0 and info["spill_loads"] == 0, (name, info)


def test_prefill_launch_registers_match_the_split(ptxas_report):
    """The d = 64 kernel's warpgroups trade registers (2 x 208 + 88 = 3 x 168 per sub-
    partition); that only adds up if ptxas gives the kernel exactly 168 at launch."""
    for name, info in ptxas_report.items():
        if kernel_kind(name) == "attn_prefill_kernel" and template_args(name)[0] == 64:
            assert info["registers"] == PREFILL_LAUNCH_REGS, (name, info)


def test_prefill_spills_do_not_grow(ptxas_report):
    for name, info in ptxas_report.items():
        if kernel_kind(name) == "attn_prefill_kernel":
            stores, loads = PREFILL_SPILL_CEILING[template_args(name)]
            assert info["spill_stores"] <= stores and info["spill_loads"] <= loads, (name, info)
