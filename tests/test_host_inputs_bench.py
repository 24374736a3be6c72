"""Host logic of the seeded inputs and of the benchmark's bookkeeping, no GPU.

- make_inputs: same seed, same tensors; K x k_mult; the dtype asked for.
- make_paged_inputs: every request's pages are distinct cache pages no other
  request uses, its table row is -1 past its pages, and the spare pages are
  never referenced.
- kernel_source_sha: code edits change it, comment and whitespace edits do not,
  so a committed ncu traffic figure stays tied to the kernel it measured.
- committed_traffic: a figure is used only when its source hash matches.
"""
import os
import shutil

import numpy as np
import torch

import bench
from attention_forward_tiled_b200.inputs import make_inputs, make_paged_inputs


def test_make_inputs_is_seeded_and_scaled():
    a = make_inputs(2, 3, 17, 19, 64, dtype="f16", seed=11)
    b = make_inputs(2, 3, 17, 19, 64, dtype="f16", seed=11)
    c = make_inputs(2, 3, 17, 19, 64, dtype="f16", seed=12)
    for x, y in zip(a, b):
        assert torch.equal(x, y) and x.dtype == torch.float16
    assert not torch.equal(a[0], c[0])
    assert [tuple(t.shape) for t in a] == [(2, 17, 3, 64), (2, 19, 3, 64), (2, 19, 3, 64)]
    q3, k3, v3 = make_inputs(2, 3, 17, 19, 64, dtype="bf16", seed=11, k_mult=3.0)
    q1, k1, v1 = make_inputs(2, 3, 17, 19, 64, dtype="bf16", seed=11)
    assert torch.equal(q3, q1) and torch.equal(v3, v1) and k3.dtype == torch.bfloat16
    np.testing.assert_allclose(k3.double().numpy(), 3.0 * k1.double().numpy(), rtol=2.0 ** -7, atol=0)


def test_paged_inputs_layout():
    lens = [37, 300, 0, 16, 1]
    page = 16
    q, kc, vc, bt, sl = make_paged_inputs(5, 2, 64, lens, page, seed=3, max_blocks=24, spare_pages=3)
    npages = [-(-L // page) for L in lens]
    assert kc.shape == vc.shape == (sum(npages) + 3, page, 2, 64)
    assert bt.shape == (5, 24) and bt.dtype == torch.int32 and sl.tolist() == lens
    used = []
    for b, n in enumerate(npages):
        row = bt[b].tolist()
        assert all(0 <= e < kc.shape[0] for e in row[:n]) and all(e == -1 for e in row[n:])
        used += row[:n]
    assert len(used) == len(set(used)) == sum(npages)          # no page shared or repeated
    assert len(set(range(kc.shape[0])) - set(used)) == 3       # the spare pages stay unused
    again = make_paged_inputs(5, 2, 64, lens, page, seed=3, max_blocks=24, spare_pages=3)
    assert all(torch.equal(x, y) for x, y in zip((q, kc, vc, bt, sl), again))


def _copy_csrc(tmp_path):
    root = tmp_path / "root"
    shutil.copytree(os.path.join(bench.ROOT, "attention_forward_tiled_b200", "csrc"),
                    root / "attention_forward_tiled_b200" / "csrc")
    return root


def test_source_hash_ignores_comments_only(tmp_path, monkeypatch):
    base = {k: bench.kernel_source_sha(k) for k in ("prefill", "decode")}
    root = _copy_csrc(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert {k: bench.kernel_source_sha(k) for k in base} == base
    path = root / "attention_forward_tiled_b200" / "csrc" / "decode_sm100.cuh"
    text = path.read_text()
    path.write_text("// a new comment line\n/* and a block\n   comment */\n" + text.replace("\n", "\n\n", 3))
    assert {k: bench.kernel_source_sha(k) for k in base} == base
    path.write_text(text + "\nstatic_assert(true, \"code\");\n")
    assert bench.kernel_source_sha("decode") != base["decode"]
    assert bench.kernel_source_sha("prefill") == base["prefill"]   # a decode-only file


def test_committed_traffic_needs_a_matching_hash(tmp_path, monkeypatch):
    root = _copy_csrc(tmp_path)
    (root / "profiles").mkdir()
    sha = bench.kernel_source_sha("prefill")
    (root / "profiles" / "x.md").write_text(
        f"bench-traffic: workload=causal4k bytes_per_launch=123 source_sha={sha}\n"
        "bench-traffic: workload=bf16_k3 bytes_per_launch=456 source_sha=0000000000000000\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.committed_traffic("causal4k") == 123.0
    assert bench.committed_traffic("bf16_k3") is None
    assert bench.committed_traffic("decode") is None


def test_clock_sampler_against_a_fake_nvml(monkeypatch):
    """The bench's clock record (median SM clock under load and every clock-event reason
    seen), read from a fake NVML: the sampler only reads, it sets nothing."""
    import sys
    import types
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=0, nvmlClocksEventReasonSwPowerCap=0x4, nvmlClocksEventReasonHwSlowdown=0x8,
        nvmlClocksEventReasonSwThermalSlowdown=0x20, nvmlClocksEventReasonGpuIdle=0x1)
    clocks = iter([1965, 1800, 1965, 1950, 1965])
    reasons = iter([0x0, 0x4, 0x4, 0x0, 0x4 | 0x8])
    calls = []
    fake.nvmlInit = lambda: calls.append("init")
    fake.nvmlDeviceGetHandleByIndex = lambda i: ("handle", i)
    fake.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965
    fake.nvmlDeviceGetClockInfo = lambda h, kind: next(clocks)
    fake.nvmlDeviceGetCurrentClocksEventReasons = lambda h: next(reasons)
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    s = bench.ClockSampler(0)
    for _ in range(5):
        s.sample_once()
    summ = s.summary()
    assert summ["sm_mhz"] == 1965 and summ["sm_max_mhz"] == 1965 and summ["samples"] == 5
    assert summ["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert calls == ["init"]


def test_clock_sampler_without_nvml(monkeypatch):
    import sys
    monkeypatch.setitem(sys.modules, "pynvml", None)   # import fails
    s = bench.ClockSampler(0)
    s.start()
    s.stop()
    summ = s.summary()
    assert summ["sm_mhz"] is None and summ["samples"] == 0 and "error" in summ


def test_traffic_figures_follow_their_kernel():
    """Each benchmark workload's traffic figure is tied to the sources of the kernel it ran."""
    import bench
    assert bench.kernel_kind("causal4k") == "prefill" and bench.kernel_kind("bf16_k3") == "prefill"
    assert bench.kernel_kind("decode") == "decode" and bench.kernel_kind("decode_paged16") == "decode"
    assert bench.kernel_kind("spec8_paged16") == "mq"
    assert bench.kernel_kind("indexer_h4") == "indexer" and bench.kernel_kind("bwd_causal4k") == "bwd"
    assert bench.kernel_kind("relpos_block200") == "relpos"
    shas = {k: bench.kernel_source_sha(k) for k in bench.KERNEL_SOURCES}
    assert len(set(shas.values())) == len(shas)
