"""The N > 1 path on the CPU: world-size-2 process groups over gloo.

Sequences are independent, so N GPUs run N replicas with no data-path
collective; the only cross-rank steps are the harness's: the slowest rank's time
(max over ranks) and the whole-job rate (all ranks' units over that time).  The
reference arm under torchrun runs on rank 0 only and the other ranks exit 0.
"""
import datetime
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


def _rank_main(rank, world, port, times, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = bench.max_over_ranks(times[rank], world)
        q.put((rank, ms, bench.whole_job_rate(world, 512 * 4, ms)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run_ranks(times):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, len(times), port, times, q)) for r in range(len(times))]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(out)


def test_max_over_ranks_and_whole_job_rate_world2():
    """Both ranks see the slower rank's time; the rate counts both ranks' units."""
    out = _run_ranks([12.5, 20.0])
    assert [r for r, _, _ in out] == [0, 1]
    for _, ms, rate in out:
        assert ms == 20.0
        assert rate == pytest.approx(2 * 512 * 4 / 0.020)


def test_max_over_ranks_is_identity_for_one_process():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.25, 1) == 7.25
    assert bench.whole_job_rate(1, 1000, 500.0) == pytest.approx(2000.0)


def test_reference_arm_under_torchrun_world2_prints_once():
    """torchrun with 2 ranks: rank 0 runs the oracle and prints one line; rank 1 exits 0."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["value"] > 0
