"""The N > 1 plumbing of bench.py, run as world-size-2 `gloo` ranks on the CPU.

The path shards with no data-path exchange (independent heads, sequences and
batches per GPU), so the only cross-rank steps are the barrier around the
timed region and the max-over-ranks reduction of the step time; the reference
arm is run by rank 0 alone.  Both are checked here on two CPU processes with
the same helpers bench.py uses under torchrun.
"""
import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, ms, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch
    import bench
    dist = bench.init_distributed(world, "gloo", timeout_s=60)
    try:
        dist.barrier()
        m = bench.max_over_ranks(ms, dist, torch.device("cpu"))
        v = bench.job_value(1e12, world, m)
        dist.barrier()
        q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo():
    world, port = 2, _free_port()
    per_rank_ms = [1.25, 3.5]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ps = [ctx.Process(target=_rank_main, args=(r, world, port, per_rank_ms[r], q)) for r in range(world)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout=180)
    codes = [p.exitcode for p in ps]
    for p in ps:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, m, v in got:
        # every rank reports the slowest rank's time, and the job value counts
        # the work of all ranks over that time
        assert m == max(per_rank_ms)
        assert v == pytest.approx(1e12 * world / (max(per_rank_ms) * 1e-3) / 1e12)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.init_distributed(1) is None
    assert bench.max_over_ranks(2.5, None, "cpu") == 2.5
    assert bench.job_value(2e12, 1, 1000.0) == pytest.approx(2.0)


def test_reference_arm_under_torchrun_two_cpu_ranks():
    """The driver's launch line for N=2, on the CPU: rank 0 alone prints one
    JSON line, the other rank exits 0 without output."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3", "--cpu-seconds", "0.2"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["n_gpus"] == 2 and j["steps"] == 1 and j["warmup"] == 3
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["value"] == j["value"] > 0
    assert j["e2e"] == {"value": j["value"], "unit": j["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    for key in ("metric", "unit", "ms_per_step", "higher_is_better", "scaling", "vs_baseline", "dtype", "data",
                "config"):
        assert key in j
