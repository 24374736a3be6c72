#!/usr/bin/env python
"""Benchmark of the fused attention forward on B200.  Rank 0 prints ONE JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload causal4k] [--no-extra]

A step is one call of the whole forward (the tiled prefill kernel for the
prefill workloads; the split-KV partial and combine kernels for decode) over
one batch of seeded synthetic inputs already resident in HBM.  Timing: W
untimed warm-up steps, then exactly K steps bracketed by a barrier and a device
synchronise, CUDA events on the launching stream, max over ranks; the stream spins
on the device while the host enqueues the K steps, so they run back to back (the
spin is outside the timed intervals).  Every rank runs an independent replica of
the workload (the forward of one (b, h) never talks to another, so there is no
data-path collective): scaling is weak.  `--gpus N` means N ranks: started as one
process, the script relaunches itself under torchrun with N ranks; started by a
launcher with a different number of ranks, it exits with status 2.  `extra`
carries the decode, causal8k, causal8000 and bf16_k3 workloads, the decode over a
16-key-page cache, the 8-token (speculative) decode over the same cache on the
tensor cores, the lightning-indexer score and top-k, and the backward pass on the
causal4k shapes, each with its roofline.

--impl reference times the fp64 CPU oracle (the only other implementation of
the method available here) on bounded samples of the same workload.
"""
import argparse
import hashlib
import re
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attn fwd TFLOP/s & % of B200 fp16 tensor peak; decode K+V GB/s vs HBM peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


# Device sources each kind of kernel is built from (the host launchers in attn_api.cu are
# left out, so adding an unrelated entry point does not orphan a committed traffic figure).
KERNEL_SOURCES = {
    "prefill": ("prefill_sm100.cuh", "sm100_ptx.cuh", "exp2_poly.cuh"),
    "decode": ("decode_sm100.cuh", "sm100_ptx.cuh"),
    "mq": ("decode_mq_sm100.cuh", "sm100_ptx.cuh"),
    "indexer": ("indexer_sm100.cuh", "sm100_ptx.cuh"),
    "bwd": ("backward_sm100.cuh", "sm100_ptx.cuh"),
    "relpos": ("relpos_sm100.cuh", "sm100_ptx.cuh"),
}


def kernel_kind(workload):
    """Which kernel's sources a workload's traffic figure belongs to."""
    for prefix, kind in (("decode", "decode"), ("spec", "mq"), ("indexer", "indexer"), ("bwd", "bwd"),
                         ("relpos", "relpos")):
        if workload.startswith(prefix):
            return kind
    return "prefill"


def kernel_source_sha(kind="prefill"):
    """Hash of the code (comments and blank space removed) of the sources one kind of
    kernel is built from: ties a committed ncu traffic figure to the kernel it measured,
    so editing a comment, or the other kernel, does not orphan it."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "attention_forward_tiled_b200", "csrc")
    for name in KERNEL_SOURCES[kind]:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        text = " ".join(text.split())
        h.update(name.encode() + b"\0" + text.encode())
    return h.hexdigest()[:16]


def committed_traffic(workload):
    """DRAM bytes per launch from the committed ncu summary, if it matches the current kernel."""
    sha = kernel_source_sha(kernel_kind(workload))
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    for name in sorted(os.listdir(pdir)):
        if not name.endswith((".md", ".txt")):
            continue
        with open(os.path.join(pdir, name)) as f:
            for line in f:
                if line.startswith("bench-traffic:"):
                    kv = dict(tok.split("=", 1) for tok in line.split()[1:] if "=" in tok)
                    if kv.get("workload") == workload and kv.get("source_sha") == sha:
                        return float(kv["bytes_per_launch"])
    return None


class ClockSampler(threading.Thread):
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    NAMES = {
        "nvmlClocksEventReasonGpuIdle": "gpu_idle",
        "nvmlClocksEventReasonApplicationsClocksSetting": "applications_clocks_setting",
        "nvmlClocksEventReasonSwPowerCap": "sw_power_cap",
        "nvmlClocksEventReasonHwSlowdown": "hw_slowdown",
        "nvmlClocksEventReasonSyncBoost": "sync_boost",
        "nvmlClocksEventReasonSwThermalSlowdown": "sw_thermal_slowdown",
        "nvmlClocksEventReasonHwThermalSlowdown": "hw_thermal_slowdown",
        "nvmlClocksEventReasonHwPowerBrakeSlowdown": "hw_power_brake_slowdown",
    }

    def __init__(self, device_index, period_s=0.0005):
        super().__init__(daemon=True)
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.error = None
        self._halt = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - NVML missing
            self.nvml = None
            self.error = str(e)

    def sample_once(self):
        n = self.nvml
        self.samples.append(n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM))
        bits = n.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
        for attr, name in self.NAMES.items():
            if bits & getattr(n, attr, 0):
                self.reasons.add(name)

    def run(self):
        if self.nvml is None:
            return
        while not self._halt.is_set():
            try:
                self.sample_once()
            except Exception as e:  # pragma: no cover
                self.error = str(e)
                return
            time.sleep(self.period)

    def stop(self):
        self._halt.set()
        self.join(timeout=5)
        if self.nvml is not None and not self.samples:
            try:
                self.sample_once()
            except Exception:
                pass

    def summary(self):
        d = {"sm_mhz": statistics.median(self.samples) if self.samples else None,
             "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
             "samples": len(self.samples), "source": "nvml"}
        if self.error:
            d["error"] = self.error
        return d


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def launch_plan(gpus, world):
    """What `--gpus N` means for a process that sees WORLD_SIZE `world`:
    "run" (already N ranks), "spawn" (a single process asked for N > 1 ranks: it
    relaunches itself under torchrun with N ranks) or "refuse" (a launcher started a
    different number of ranks than --gpus says)."""
    if gpus < 1:
        return "refuse"
    if world == gpus:
        return "run"
    if world == 1 and "RANK" not in os.environ:
        return "spawn"
    return "refuse"


def spawn_ranks(gpus, argv):
    """Relaunch this script as `gpus` ranks (one per GPU) under torchrun on 127.0.0.1;
    returns torchrun's exit code."""
    import socket
    import subprocess
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node", str(gpus), "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def max_over_ranks(x, world, device="cuda"):
    """Max of a host float over all ranks (the timing rule: the slowest rank counts)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def workload_config(name, w):
    q_bytes = w["B"] * w["Nq"] * w["H"] * w["d"] * 2
    kv_bytes = 2 * w["B"] * w["Nk"] * w["H"] * w["d"] * 2
    total = 2 * q_bytes + kv_bytes
    l2 = ("inputs larger than L2 (%.0f MB of Q, K, V, O per step vs 126 MB L2): no flush"
          % (total / 1e6)) if total > L2_BYTES else "L2 flushed between steps (256 MB memset)"
    return {"workload": name, "B": w["B"], "H": w["H"], "Nq": w["Nq"], "Nk": w["Nk"], "d": w["d"],
            "causal": w["causal"], "dtype": w["dtype"], "scale": w["scale"], "seed": w["seed"],
            "k_mult": w["k_mult"], "layout": "[B,N,H,d]", "l2": l2, "parallelism": "replicas"}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def time_gpu_steps(step, K, stream, flush=None):
    """Per-step device times (ms) from CUDA events on `stream`; an L2 flush, when
    given, runs between steps outside the timed intervals.

    The stream first runs a device-side spin long enough for the host to enqueue all K
    steps, so the timed steps run back to back on the GPU instead of waiting for a host
    thread (Python launch overhead, the clock sampler's share of the interpreter) between
    short launches; the spin itself is outside every timed interval."""
    import torch
    spin_cycles = max(10_000_000, K * 1_000_000)  # >= 5 ms at 2 GHz, 0.5 ms of host time per step
    if flush is None:  # back-to-back steps: one event between consecutive steps
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
        with torch.cuda.stream(stream):
            torch.cuda._sleep(spin_cycles)
            evs[0].record(stream)
            for i in range(K):
                step()
                evs[i + 1].record(stream)
        stream.synchronize()
        return [evs[i].elapsed_time(evs[i + 1]) for i in range(K)]
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    with torch.cuda.stream(stream):
        torch.cuda._sleep(spin_cycles)
        for i in range(K):
            flush()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
    stream.synchronize()
    return [starts[i].elapsed_time(ends[i]) for i in range(K)]


def measure_workload(name, K, W, world, device, peaks, want_e2e=True):
    import torch

    import attention_forward_tiled_b200 as attn
    from attention_forward_tiled_b200.inputs import WORKLOADS, flops, kv_bytes, make_inputs

    w = WORKLOADS[name]
    q, k, v = make_inputs(**w)
    qd, kd, vd = q.to(device), k.to(device), v.to(device)
    out = torch.empty_like(qd)
    lse = torch.empty((w["B"], w["H"], w["Nq"]), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    total_bytes = 2 * qd.numel() * 2 + 2 * kd.numel() * 2
    flush_buf = None
    if total_bytes <= L2_BYTES:
        flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)

    def step():
        attn.attn_fwd(qd, kd, vd, causal=w["causal"], scale=w["scale"], out=out, lse=lse,
                      stream=stream)

    flush = (lambda: flush_buf.zero_()) if flush_buf is not None else None
    for _ in range(W):
        step()
    torch.cuda.synchronize(device)
    if attn.get_status(device=device) != 0:
        raise RuntimeError("device status error during warm-up")

    sampler = ClockSampler(device.index if device.index is not None else 0)
    barrier(world)
    torch.cuda.synchronize(device)
    sampler.start()
    t_steps = time_gpu_steps(step, K, stream, flush)
    sampler.stop()
    torch.cuda.synchronize(device)
    barrier(world)
    if attn.get_status(device=device) != 0:
        raise RuntimeError("device status error during the timed region")
    elapsed_ms = max_over_ranks(sum(t_steps), world)

    is_decode = w["Nq"] == 1
    res = {"elapsed_ms": elapsed_ms, "ms_per_step": elapsed_ms / K, "clocks": sampler.summary()}
    if is_decode:
        nbytes = kv_bytes(**w)
        res["value"] = world * K * nbytes / (elapsed_ms * 1e-3) / 1e9
        res["unit"] = "GB/s"
        # each step: partial kernel (dominant) + combine kernel; the step time bounds the partial
        per_launch = statistics.mean(t_steps)
        achieved = nbytes / (per_launch * 1e-3) / 1e9
        res["roofline"] = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                           "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                           "traffic": committed_traffic(name),
                           "algorithmic_bytes_per_launch": nbytes,
                           "note": "launch time includes the combine kernel"}
        res["gpu_launches"] = 2 * K
    else:
        f = flops(**w)
        res["value"] = world * K * f / (elapsed_ms * 1e-3) / 1e12
        res["unit"] = "TFLOP/s"
        per_launch = statistics.mean(t_steps)
        achieved = f / (per_launch * 1e-3) / 1e12
        res["roofline"] = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                           "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                           "traffic": committed_traffic(name),
                           "algorithmic_flops_per_launch": f,
                           "peak_note": "%s burst bf16 dense GEMM peak (fp16:bf16 nominal ratio 1:1); "
                                        "sustained %.1f" % (peaks["source"], peaks["bf16_tflops_sustained"])}
        res["gpu_launches"] = K
    res["min_ms"] = min(t_steps)
    res["median_ms"] = statistics.median(t_steps)

    if want_e2e:
        runner = attn.HostRunner(w["B"], w["H"], w["Nq"], w["Nk"], w["d"], q.dtype, device=device,
                                 causal=w["causal"], scale=w["scale"])
        qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
        runner(qh, kh, vh)
        torch.cuda.synchronize(device)
        barrier(world)
        t_e2e = time_gpu_steps(lambda: runner(qh, kh, vh, stream=stream), K, stream)
        barrier(world)
        e_ms = max_over_ranks(sum(t_e2e), world)
        unit_work = kv_bytes(**w) / 1e9 if is_decode else flops(**w) / 1e12
        res["e2e"] = {"value": world * K * unit_work / (e_ms * 1e-3), "unit": res["unit"],
                      "h2d_bytes_per_step": runner.h2d_bytes, "d2h_bytes_per_step": runner.d2h_bytes,
                      "ms_per_step": e_ms / K}
        # the result of the last e2e step must match the device-resident run
        if not torch.equal(runner.out_host, out.cpu()):
            raise RuntimeError("end-to-end result differs from the device-resident result")
    del qd, kd, vd, out, lse, flush_buf
    torch.cuda.empty_cache()
    return res


def cpu_baseline_sample(name, budget_s=20.0):
    """Time the oracle, as it stands, on a bounded sample of the workload (rank 0, host cores)."""
    import oracle
    from attention_forward_tiled_b200.inputs import WORKLOADS, make_inputs

    w = WORKLOADS[name]
    q, k, v = make_inputs(**w)
    threads = oracle.num_threads()
    heads = min(w["H"], max(1, threads))

    def run(rows):
        qs = q[0:1, w["Nq"] - rows:, :heads]
        ks, vs = k[0:1, :, :heads], v[0:1, :, :heads]
        t0 = time.perf_counter()
        oracle.attn_fwd(qs, ks, vs, causal=w["causal"], scale=w["scale"])
        return time.perf_counter() - t0

    def work(rows):  # exact allowed (query, key) pairs x 4 d (bottom-right causal slice)
        nq, nk = w["Nq"], w["Nk"]
        if not w["causal"]:
            pairs = rows * nk
        else:
            pairs = sum(max(0, min(nk, i + nk - nq + 1)) for i in range(nq - rows, nq))
        return 4.0 * w["d"] * pairs * heads

    rows = min(w["Nq"], 32)
    t = run(rows)
    if rows < w["Nq"]:
        rows = int(min(w["Nq"], max(rows, rows * budget_s / max(t, 1e-3))))
        t = run(rows)
    is_decode = w["Nq"] == 1
    if is_decode:
        value = 2 * heads * w["Nk"] * w["d"] * 2 / t / 1e9
        unit = "GB/s"
    else:
        value = work(rows) / t / 1e12
        unit = "TFLOP/s"
    return {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
            "sample": "batch 0, heads 0..%d, last %d query rows x all %d keys (%s), %.1f s"
                      % (heads - 1, rows, w["Nk"], "causal, bottom-right" if w["causal"] else "non-causal", t)}


def measure_paged(name, K, W, world, device, peaks):
    """The paged-cache decode (attn_fwd_decode_paged): K+V bytes per second, as decode."""
    import torch

    import attention_forward_tiled_b200 as attn
    from attention_forward_tiled_b200.inputs import PAGED_WORKLOADS, make_paged_inputs

    w = PAGED_WORKLOADS[name]
    B, H, d, Lq = w["B"], w["H"], w["d"], w["Lq"]
    q, kc, vc, bt, sl = (t.to(device) for t in make_paged_inputs(
        B, H, d, w["seq_lens"], w["page_size"], dtype=w["dtype"], seed=w["seed"], Lq=Lq))
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream(device)
    if Lq == 1 and not w["causal"]:  # one token: the CUDA-core split-KV decode
        lse = torch.empty((B, H), dtype=torch.float32, device=device)

        def step():
            attn.attn_fwd_decode_paged(q, kc, vc, bt, sl, scale=w["scale"], out=out, lse=lse,
                                       stream=stream)
    else:  # several tokens per request: the tensor-core kernel
        lse = torch.empty((B, H, Lq), dtype=torch.float32, device=device)

        def step():
            attn.attn_fwd_paged(q, kc, vc, bt, sl, causal=w["causal"], scale=w["scale"], out=out,
                                lse=lse, stream=stream)

    for _ in range(W):
        step()
    torch.cuda.synchronize(device)
    if attn.get_status(device=device) != 0:
        raise RuntimeError("device status error during warm-up")
    sampler = ClockSampler(device.index if device.index is not None else 0)
    barrier(world)
    torch.cuda.synchronize(device)
    sampler.start()
    t_steps = time_gpu_steps(step, K, stream, None)  # 1.07 GB of K+V per step > L2
    sampler.stop()
    torch.cuda.synchronize(device)
    barrier(world)
    if attn.get_status(device=device) != 0:
        raise RuntimeError("device status error during the timed region")
    elapsed_ms = max_over_ranks(sum(t_steps), world)
    nbytes = 2 * sum(w["seq_lens"]) * H * d * q.element_size()
    achieved = nbytes / (statistics.mean(t_steps) * 1e-3) / 1e9
    del q, kc, vc, bt, sl, out, lse
    torch.cuda.empty_cache()
    return {"value": world * K * nbytes / (elapsed_ms * 1e-3) / 1e9, "unit": "GB/s",
            "ms_per_step": elapsed_ms / K,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": committed_traffic(name),
                         "algorithmic_bytes_per_launch": nbytes,
                         "note": "launch time includes the combine kernel"},
            "clocks": sampler.summary(),
            "config": {"workload": name, "B": B, "H": H, "d": d, "seq_lens": "4096 each",
                       "query_tokens": Lq, "causal": w["causal"],
                       "page_size": w["page_size"], "pages": "randomly placed", "dtype": w["dtype"],
                       "l2": "K+V of 1074 MB per step vs 126 MB L2: no flush"}}


def measure_indexer(name, K, W, world, device, peaks):
    """Lightning-indexer score and top-k: bytes each kernel must move per call, per second."""
    import torch

    import attention_forward_tiled_b200 as attn
    from attention_forward_tiled_b200.inputs import INDEXER_WORKLOADS, make_indexer_inputs

    w = INDEXER_WORKLOADS[name]
    B, T, H, P, d, k = w["B"], w["T"], w["H"], w["P"], w["d"], w["k"]
    q, kp, wt, mask = (t.to(device) if t is not None else None for t in make_indexer_inputs(
        B, T, H, P, d, dtype=w["dtype"], seed=w["seed"], weights=w["weights"], masked=w["masked"]))
    score = torch.empty((B, T, P), dtype=torch.float32, device=device)
    idx = torch.empty((B, T, k), dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)
    res = {}
    for kind in ("score", "topk"):
        if kind == "score":
            def step():
                attn.indexer_score(q, kp, wt, mask, out=score, stream=stream)
            nbytes = (q.numel() + kp.numel()) * q.element_size() + wt.numel() * 4 + score.numel() * 4 + \
                (mask.numel() * 2 if mask is not None else 0)
        else:
            def step():
                attn.topk(score, k, out=idx, stream=stream)
            nbytes = score.numel() * 4 + idx.numel() * 4
        for _ in range(W):
            step()
        torch.cuda.synchronize(device)
        if attn.get_status(device=device) != 0:
            raise RuntimeError("device status error during warm-up")
        sampler = ClockSampler(device.index if device.index is not None else 0)
        barrier(world)
        torch.cuda.synchronize(device)
        sampler.start()
        t_steps = time_gpu_steps(step, K, stream, None)
        sampler.stop()
        torch.cuda.synchronize(device)
        barrier(world)
        elapsed_ms = max_over_ranks(sum(t_steps), world)
        achieved = nbytes / (statistics.mean(t_steps) * 1e-3) / 1e9
        res[kind] = {"value": world * K * nbytes / (elapsed_ms * 1e-3) / 1e9, "unit": "GB/s",
                     "ms_per_step": elapsed_ms / K,
                     "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                                  "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": committed_traffic("%s.%s" % (name, kind)),
                                  "algorithmic_bytes_per_launch": nbytes},
                     "clocks": sampler.summary(),
                     "config": {"workload": name, "kernel": kind, "B": B, "T": T, "H": H, "P": P, "d": d,
                                "k": k, "dtype": w["dtype"], "weights": w["weights"], "masked": w["masked"],
                                "l2": "%.0f MB moved per call" % (nbytes / 1e6)}}
    del q, kp, wt, mask, score, idx
    torch.cuda.empty_cache()
    return res


BWD_WORKLOADS = {"bwd_causal4k": "causal4k"}  # backward of a forward workload, same shapes


def measure_bwd(name, K, W, world, device, peaks):
    """Backward pass (attn_bwd) on a forward workload's shapes: TFLOP/s counted as 2.5 times
    the forward's (five products of the forward's size instead of two), halved when causal."""
    import torch

    import attention_forward_tiled_b200 as attn
    from attention_forward_tiled_b200.inputs import WORKLOADS, flops, make_inputs

    w = WORKLOADS[BWD_WORKLOADS[name]]
    q, k, v = (t.to(device) for t in make_inputs(**w))
    g = torch.Generator("cpu").manual_seed(w["seed"] + 1000)
    dout = torch.randn(q.shape, generator=g).to(q.dtype).to(device)
    o, lse = attn.attn_fwd(q, k, v, causal=w["causal"], scale=w["scale"])
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    stream = torch.cuda.current_stream(device)

    def step():
        attn.attn_bwd(q, k, v, o, lse, dout, causal=w["causal"], scale=w["scale"], stream=stream,
                      dq=dq, dk=dk, dv=dv)

    for _ in range(W):
        step()
    torch.cuda.synchronize(device)
    if attn.get_status(device=device) != 0:
        raise RuntimeError("device status error during warm-up")
    sampler = ClockSampler(device.index if device.index is not None else 0)
    barrier(world)
    torch.cuda.synchronize(device)
    sampler.start()
    t_steps = time_gpu_steps(step, K, stream, None)
    sampler.stop()
    torch.cuda.synchronize(device)
    barrier(world)
    if attn.get_status(device=device) != 0:
        raise RuntimeError("device status error during the timed region")
    elapsed_ms = max_over_ranks(sum(t_steps), world)
    f = 2.5 * flops(**w)
    achieved = f / (statistics.mean(t_steps) * 1e-3) / 1e12
    del q, k, v, dout, o, lse, dq, dk, dv
    torch.cuda.empty_cache()
    cfg = workload_config(BWD_WORKLOADS[name], w)
    cfg["workload"] = name
    return {"value": world * K * f / (elapsed_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": elapsed_ms / K,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                         "traffic": committed_traffic(name), "algorithmic_flops_per_launch": f,
                         "note": "the step is the D pre-pass, the gradient kernel and the dQ cast"},
            "clocks": sampler.summary(), "config": cfg}


def measure_relpos(name, K, W, world, device, peaks):
    """Attention with the relative-position term (attn_fwd_relpos): TFLOP/s counted from the
    three products the definition takes per score (q.k, q.emb[dist] and p.v, 2d FLOP each),
    6 B H Nq Nk d, on the block-local workload; the kernel's window product does more."""
    import torch

    import attention_forward_tiled_b200 as attn
    from attention_forward_tiled_b200.inputs import RELPOS_WORKLOADS, make_relpos_inputs

    w = RELPOS_WORKLOADS[name]
    q, k, v, emb = (t.to(device) for t in make_relpos_inputs(**w))
    out = torch.empty_like(q)
    lse = torch.empty((w["B"], w["H"], w["Nq"]), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        attn.attn_fwd_relpos(q, k, v, emb, w["R"], causal=w["causal"], scale=w["scale"], out=out, lse=lse,
                             stream=stream)

    for _ in range(W):
        step()
    torch.cuda.synchronize(device)
    if attn.get_status(device=device) != 0:
        raise RuntimeError("device status error during warm-up")
    sampler = ClockSampler(device.index if device.index is not None else 0)
    barrier(world)
    torch.cuda.synchronize(device)
    sampler.start()
    t_steps = time_gpu_steps(step, K, stream, None)
    sampler.stop()
    torch.cuda.synchronize(device)
    barrier(world)
    if attn.get_status(device=device) != 0:
        raise RuntimeError("device status error during the timed region")
    elapsed_ms = max_over_ranks(sum(t_steps), world)
    f = 6.0 * w["B"] * w["H"] * w["Nq"] * w["Nk"] * w["d"]
    if w["causal"]:
        f *= 0.5
    nbytes = (2 * q.numel() + k.numel() + v.numel() + emb.numel()) * q.element_size() + lse.numel() * 4
    # 6 d FLOP per score against 16 d bytes per key row of a 200-token block: ~150 FLOP per byte,
    # below the tensor/HBM ridge (~240), so the roofline is the bandwidth one
    achieved = nbytes / (statistics.mean(t_steps) * 1e-3) / 1e9
    del q, k, v, emb, out, lse
    torch.cuda.empty_cache()
    return {"value": world * K * f / (elapsed_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": elapsed_ms / K,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "traffic": committed_traffic(name), "algorithmic_bytes_per_launch": nbytes,
                         "algorithmic_flops_per_launch": f},
            "clocks": sampler.summary(),
            "config": {"workload": name, "B": w["B"], "H": w["H"], "Nq": w["Nq"], "Nk": w["Nk"], "d": w["d"],
                       "R": w["R"], "causal": w["causal"], "dtype": w["dtype"],
                       "l2": "%.0f MB moved per call" % (nbytes / 1e6)}}


def print_single(args, world, rank, r, dtype):
    """One JSON line for a workload timed on its own (profiling and single-kernel runs)."""
    line = {"metric": METRIC, "value": r["value"], "unit": r["unit"], "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": r["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic (seeded randn)",
            "config": r["config"], "roofline": r["roofline"], "e2e": None, "clocks": r["clocks"],
            "impl": "ours"}
    if "extra" in r:
        line["extra"] = r["extra"]
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def keep_pool_memory(device_index):
    """The library takes its per-call workspaces from the device's default stream-ordered
    pool, which by default returns its memory to the driver at every synchronisation, so the
    first call after one would grow the pool again inside a timed region; keep what it holds."""
    try:
        from cuda.bindings import driver as drv
        from cuda.bindings import runtime as rt
    except ImportError:  # pragma: no cover - cuda-python missing
        return False
    err, pool = rt.cudaDeviceGetDefaultMemPool(device_index)
    if err != rt.cudaError_t.cudaSuccess:
        return False
    (err,) = rt.cudaMemPoolSetAttribute(pool, rt.cudaMemPoolAttr.cudaMemPoolAttrReleaseThreshold,
                                        drv.cuuint64_t(1 << 40))
    return err == rt.cudaError_t.cudaSuccess


def run_ours(args):
    import torch

    world, rank, local = dist_setup(args)
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    device = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(device)
    keep_pool_memory(device.index)
    peaks = load_peaks()
    K, W = args.steps, max(3, args.warmup)

    from attention_forward_tiled_b200.inputs import (INDEXER_WORKLOADS, PAGED_WORKLOADS, RELPOS_WORKLOADS,
                                                     WORKLOADS)
    if args.workload in RELPOS_WORKLOADS:
        r = measure_relpos(args.workload, K, W, world, device, peaks)
        return print_single(args, world, rank, r, RELPOS_WORKLOADS[args.workload]["dtype"])
    if args.workload in INDEXER_WORKLOADS:
        r = measure_indexer(args.workload, K, W, world, device, peaks)
        r["score"]["extra"] = {"topk": r["topk"]}
        return print_single(args, world, rank, r["score"], INDEXER_WORKLOADS[args.workload]["dtype"])
    if args.workload in BWD_WORKLOADS:
        r = measure_bwd(args.workload, K, W, world, device, peaks)
        return print_single(args, world, rank, r, WORKLOADS[BWD_WORKLOADS[args.workload]]["dtype"])
    if args.workload in PAGED_WORKLOADS:
        # the paged decode on its own (profiling runs): its line has no end-to-end figure
        r = measure_paged(args.workload, K, W, world, device, peaks)
        line = {"metric": METRIC, "value": r["value"], "unit": r["unit"], "n_gpus": world, "steps": K,
                "warmup": W, "ms_per_step": r["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": PAGED_WORKLOADS[args.workload]["dtype"],
                "data": "synthetic (seeded randn, pages placed at random)", "config": r["config"],
                "roofline": r["roofline"], "e2e": None, "gpu_launches": 2 * K, "clocks": r["clocks"],
                "impl": "ours"}
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps(line), flush=True)
        return
    main = measure_workload(args.workload, K, W, world, device, peaks, want_e2e=True)
    extra = {}
    if not args.no_extra:
        for name in ("decode", "causal8k", "causal8000", "bf16_k3"):
            if name == args.workload:
                continue
            r = measure_workload(name, K, W, world, device, peaks, want_e2e=False)
            extra[name] = {"value": r["value"], "unit": r["unit"], "ms_per_step": r["ms_per_step"],
                           "roofline": r["roofline"], "clocks": r["clocks"],
                           "config": workload_config(name, WORKLOADS[name])}
        extra["decode_paged16"] = measure_paged("decode_paged16", K, W, world, device, peaks)
        extra["spec8_paged16"] = measure_paged("spec8_paged16", K, W, world, device, peaks)
        r = measure_indexer("indexer_h4", K, W, world, device, peaks)
        extra["indexer_h4_score"] = r["score"]
        extra["indexer_h4_topk"] = r["topk"]
        extra["bwd_causal4k"] = measure_bwd("bwd_causal4k", K, W, world, device, peaks)
        extra["relpos_block200"] = measure_relpos("relpos_block200", K, W, world, device, peaks)
    line = {
        "metric": METRIC,
        "value": main["value"],
        "unit": main["unit"],
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": main["ms_per_step"],
        "ms_per_step_median": main["median_ms"],  # this rank's steps
        "ms_per_step_min": main["min_ms"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": WORKLOADS[args.workload]["dtype"],
        "data": "synthetic (seeded randn, the article's [batch, seq, heads, head_dim] shapes)",
        "config": workload_config(args.workload, WORKLOADS[args.workload]),
        "roofline": main["roofline"],
        "e2e": main["e2e"],
        "gpu_launches": main["gpu_launches"],
        "clocks": main["clocks"],
        "impl": "ours",
    }
    if extra:
        line["extra"] = extra
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_sample(args.workload)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# reference arm: the fp64 oracle on bounded samples of the same workload
# ---------------------------------------------------------------------------
def run_reference(args):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return
    import oracle
    from attention_forward_tiled_b200.inputs import WORKLOADS, make_inputs

    w = WORKLOADS[args.workload]
    K, W = args.steps, max(3, args.warmup)
    q, k, v = make_inputs(**w)
    threads = oracle.num_threads()
    heads = min(w["H"], max(1, threads))
    budget = max(0.2, 150.0 / (K + W))  # seconds per step, whole run within a few minutes

    def run(rows):
        qs = q[0:1, w["Nq"] - rows:, :heads]
        t0 = time.perf_counter()
        oracle.attn_fwd(qs, k[0:1, :, :heads], v[0:1, :, :heads], causal=w["causal"], scale=w["scale"])
        return time.perf_counter() - t0

    rows = min(w["Nq"], 8)
    t = run(rows)
    rows = int(min(w["Nq"], max(1, rows * budget / max(t, 1e-4))))
    for _ in range(W):
        run(rows)
    times = [run(rows) for _ in range(K)]
    nq, nk = w["Nq"], w["Nk"]
    if w["Nq"] == 1:
        unit = "GB/s"
        per_step = 2 * heads * nk * w["d"] * 2 / 1e9
    else:
        unit = "TFLOP/s"
        pairs = (rows * nk if not w["causal"] else
                 sum(max(0, min(nk, i + nk - nq + 1)) for i in range(nq - rows, nq)))
        per_step = 4.0 * w["d"] * pairs * heads / 1e12
    total = sum(times)
    value = K * per_step / total
    sample = ("per step: batch 0, heads 0..%d, last %d query rows x all %d keys"
              % (heads - 1, rows, nk))
    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": 1e3 * total / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded randn)",
        "config": workload_config(args.workload, w), "impl": "reference",
        "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="causal4k")
    ap.add_argument("--no-extra", action="store_true", help="skip the decode/causal8k/bf16 lines")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    plan = launch_plan(args.gpus, world)
    if plan == "spawn":
        sys.exit(spawn_ranks(args.gpus, sys.argv[1:]))
    if plan == "refuse":
        sys.stderr.write("bench.py: --gpus %d but the launcher started %d rank(s)\n" % (args.gpus, world))
        sys.exit(2)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
