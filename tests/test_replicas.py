"""Multi-process host logic of bench.py on CPU (gloo, world size 2).

The hot path shards with no exchange step, so N GPUs run N independent
replicas; the only collectives are the barrier around the timed region and
the max over ranks of the measured time.  These tests run that plumbing as
two gloo ranks, and the reference arm under torchrun, without a GPU."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    pg = bench.init_replicas(world, "gloo")
    pg.barrier()
    # rank r "measured" 10 (r + 1) ms for 5 steps of 1 TFLOP each
    total = bench.max_over_ranks(10.0 * (rank + 1), pg)
    value = bench.whole_job_tflops(world, 1e12, 5, total)
    pg.barrier()
    q.put((rank, total, value))
    pg.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, total, value in got:
        assert total == 20.0                      # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * 5 / 20e-3)   # both ranks' work over that time, in TFLOP/s


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.init_replicas(1) is None
    assert bench.max_over_ranks(3.5, None) == 3.5
    assert bench.whole_job_tflops(1, 2e12, 4, 8.0) == pytest.approx(1e3)


def test_reference_arm_under_torchrun_prints_one_line():
    """Rank 0 alone times the oracle and prints the JSON line; rank 1 exits 0
    without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["cpu_baseline"]["kind"] == "oracle"
    assert d["value"] > 0 and d["e2e"]["h2d_bytes_per_step"] == 0
