"""Host-side logic of the multi-process (replica) bench on CPU: two gloo
ranks agree on the slowest rank's time, the whole-job rate counts every
rank's work, and the reference arm under torchrun prints one line from
rank 0 while the other rank exits cleanly."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m = bench.max_over_ranks(times[rank], world, "cpu")
        rate = bench.aggregate_rate(world, 1.0e12, 10, m)
        out.put((rank, m, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_rate_gloo():
    world, port = 2, _free_port()
    times = [3.5, 7.25]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, rate in res:
        assert m == 7.25                                  # slowest rank, on every rank
        assert rate == pytest.approx(2 * 1.0e12 * 10 / 7.25e-3)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(4.0, 1, "cpu") == 4.0
    assert bench.aggregate_rate(1, 2.0, 3, 1000.0) == pytest.approx(6.0)


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600,
                       env=dict(os.environ, OMP_NUM_THREADS="4"))
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
