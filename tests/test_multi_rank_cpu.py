"""Host logic of the N > 1 benchmark path on CPU ranks (gloo, world size 2).

Each GPU runs an independent replica of the workload, so the only multi-rank
logic is around the timing: every rank passes the same barriers, the job time
is the maximum over ranks, the whole-job rate counts every rank's tokens, and
only rank 0 prints.  None of this needs a GPU.
"""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w, r, local = bench.dist_env()
        ranks = bench.Ranks(dist, "cpu")
        ranks.barrier()
        # each rank's own "device time"; the job time is the slowest rank's
        own_ms = 10.0 + 5.0 * rank
        job_ms = ranks.max(own_ms)
        ranks.barrier()
        rate = bench.aggregate_rate(w, 32, 4, job_ms)
        q.put((r, w, local, own_ms, job_ms, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_rate():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for r, (rank, w, local, own, job, rate) in enumerate(got):
        assert (rank, w, local) == (r, world, r)
        assert job == 15.0                      # max over ranks, seen by every rank
        # 2 ranks x 32 tokens x 4 steps in 15 ms
        assert rate == pytest.approx(2 * 32 * 4 / 0.015)


def test_single_process_helpers():
    assert bench.Ranks(None, "cpu").max(3.5) == 3.5
    bench.Ranks(None, "cpu").barrier()
    assert bench.aggregate_rate(1, 32, 50, 1000.0) == pytest.approx(1600.0)


def test_reference_arm_prints_once_under_two_ranks():
    """`bench.py --impl reference` under torchrun: rank 0 alone times the oracle
    and prints one JSON line; the other rank exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "tiny"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["config"]["workload"] and d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"] and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_single_process():
    """`bench.py --impl reference` without torchrun: one JSON line with the
    contract's keys, the oracle timed on the host's cores."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2", "--warmup", "1",
           "--workload", "tiny"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["unit"] == "tokens/s"
    assert d["config"]["workload"].startswith("tiny") and d["dtype"] == "f64" and d["data"] == "synthetic"
    # a sampled step evaluates all 4 heads of the one query token: one token per step
    assert d["cpu_baseline"]["sample"].startswith("2 steps x 4 of 4 heads")
    assert d["value"] == pytest.approx(1 / (d["ms_per_step"] / 1e3), rel=1e-6)
