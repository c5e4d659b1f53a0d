"""The benchmark's multi-process path on the CPU (gloo, world size 2): the
step time every rank reports is the maximum over ranks, the job value counts
every rank's batch, and under torchrun the reference arm prints one line from
rank 0 while the other ranks exit cleanly."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        step_ms = [3.5, 1.25][rank]
        got = bench.max_over_ranks(step_ms, world, "cpu")
        out.put((rank, got, bench.job_value(world, 4, got)))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert [r[1] for r in res] == [3.5, 3.5]                 # both ranks see the slowest replica
    assert res[0][2] == pytest.approx(2 * 4 / 3.5e-3)       # weak scaling: 2 ranks x 4 sequences


def test_single_process_helpers_need_no_process_group():
    bench.barrier(1)
    assert bench.max_over_ranks(2.0, 1, "cpu") == 2.0
    assert bench.job_value(1, 1, 1.0) == pytest.approx(1000.0)


def test_reference_arm_under_torchrun_prints_once():
    """--impl reference times the oracle on the host cores; under torchrun with
    two ranks only rank 0 runs and prints, the other rank exits 0."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "tiny", "--gpus", "2", "--steps", "2", "--warmup", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["higher_is_better"] is True
