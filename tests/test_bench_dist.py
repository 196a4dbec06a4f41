"""Host logic of bench.py's multi-rank path on CPU: world size 2 over gloo.

Each rank is an independent replica of the layer (no data-path collective);
the job's throughput is all ranks' tokens over the slowest rank's time, and
the reference arm runs on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist(world, rank, rank, backend="gloo", timeout_s=60)
    d.barrier()
    # rank r processed 64 * (r + 1) tokens in 10 * (r + 1) ms
    value, ms, tokens = bench.job_throughput(d, 64.0 * (rank + 1), 10.0 * (rank + 1))
    d.barrier()
    d.close()
    q.put((rank, value, ms, tokens))


def test_job_throughput_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, value, ms, tokens in res:
        assert ms == 20.0                       # slowest rank
        assert tokens == 64.0 * 3               # both ranks' tokens
        assert value == pytest.approx(192.0 / 0.020)


def test_single_process_dist_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist(1, 0, 0, backend="gloo")
    assert bench.job_throughput(d, 128.0, 4.0) == (128.0 / 0.004, 4.0, 128.0)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "3", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
