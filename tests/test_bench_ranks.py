"""Multi-rank logic of the benchmark on CPU (gloo, world size 2).

The forward has no data-path collective (every (b, h) row is independent), so the
only cross-rank steps are the barrier around the timed region and the max over
ranks of the elapsed time; the reference arm runs on rank 0 only.
"""
import os
import socket

import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        elapsed = 10.0 + 5.0 * rank  # each rank's own timed region (ms)
        m = bench.max_over_ranks(elapsed, world, device="cpu")
        w, r, lr = bench.dist_setup(None)
        q.put((rank, m, w, r, lr))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_barrier_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert [g[1] for g in got] == [15.0, 15.0]          # both ranks see the slowest rank's time
    assert [(g[2], g[3], g[4]) for g in got] == [(2, 0, 0), (2, 1, 1)]


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")

    class A:
        workload, steps, warmup = "tiny", 1, 3

    bench.run_reference(A())        # rank 1: returns at once, prints nothing
    assert capsys.readouterr().out == ""


def test_reference_arm_json_line():
    """The reference arm (the oracle on the host cores) prints one JSON line with the keys
    the benchmark contract asks for; the tiny workload keeps it to seconds."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    res = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                          "--steps", "2", "--warmup", "1"], cwd=root, env=env, capture_output=True,
                         text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "TFLOP/s"
    assert line["n_gpus"] == 1 and line["steps"] == 2 and line["warmup"] >= 3
    assert line["config"]["workload"] == "tiny" and line["higher_is_better"] is True
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_under_torchrun_two_ranks():
    """Launched as the multi-GPU runs are (torchrun, two ranks), the reference arm prints
    exactly one line, from rank 0, and every rank exits 0."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--workload", "tiny", "--gpus", "2", "--steps", "2",
           "--warmup", "3"]
    res = subprocess.run(cmd, cwd=root, env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0


def test_launch_plan(monkeypatch):
    """--gpus N means N ranks: run as is, relaunch a single process as N ranks, or refuse."""
    import bench
    monkeypatch.delenv("RANK", raising=False)
    assert bench.launch_plan(1, 1) == "run"
    assert bench.launch_plan(4, 1) == "spawn"
    assert bench.launch_plan(0, 1) == "refuse"
    monkeypatch.setenv("RANK", "0")
    assert bench.launch_plan(2, 2) == "run"
    assert bench.launch_plan(3, 2) == "refuse"
    assert bench.launch_plan(2, 1) == "refuse"  # a launcher started one rank


def test_gpus_two_without_a_launcher_runs_two_ranks():
    """`bench.py --gpus 2` started as one process relaunches itself as two ranks (gloo-free
    reference arm on CPU): one JSON line, from rank 0, with n_gpus 2."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    res = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                          "--gpus", "2", "--steps", "1", "--warmup", "3"], cwd=root, env=env,
                         capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    assert json.loads(lines[0])["n_gpus"] == 2


def test_gpus_mismatch_with_the_launcher_is_refused():
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="2", RANK="0", LOCAL_RANK="0")
    res = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                          "--gpus", "3", "--steps", "1"], cwd=root, env=env, capture_output=True,
                         text=True, timeout=120)
    assert res.returncode == 2
    assert "--gpus 3" in res.stderr and not res.stdout.strip()
