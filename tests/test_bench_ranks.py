"""The benchmark's multi-rank logic on CPU (gloo, world size 2): the device time of a run
is the maximum over ranks, and under torchrun the reference arm prints one line, from
rank 0, while the other rank exits cleanly without work."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.max_over_ranks(3.0 * (rank + 1) + 0.25, world, "cpu")
        again = bench.max_over_ranks(-float(rank), world, "cpu")
        out.put((rank, got, again))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res == [(0, 6.25, 0.0), (1, 6.25, 0.0)]


def test_max_over_ranks_single_rank_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1.5, 1, "cpu") == 1.5


def test_reference_arm_under_torchrun_prints_one_line():
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--cpu-blocks", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_gpus_flag_spawns_ranks_without_torchrun():
    """`bench.py --gpus 2` outside torchrun re-launches itself on two ranks; rank 0 alone
    prints the (reference-arm) line, whose unit string is the one the device arm prints."""
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "0", "--cpu-blocks", "2", "--workload", "32k-exact"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    sys.path.insert(0, ROOT)
    import bench
    assert d["n_gpus"] == 2 and d["impl"] == "reference"
    assert d["unit"] == bench.unit_of(bench.WORKLOADS["32k-exact"]) == d["e2e"]["unit"]


def test_spawn_command_keeps_arguments():
    sys.path.insert(0, ROOT)
    import bench
    cmd = bench.spawn_ranks_command(["--gpus", "4", "--steps", "7"], 4, 29555)
    i = cmd.index("--nproc-per-node")
    assert cmd[i + 1] == "4" and "127.0.0.1" in cmd and cmd[-3:] == ["--gpus", "4", "--steps", "7"][-3:]
    assert cmd[cmd.index("--master-port") + 1] == "29555"
