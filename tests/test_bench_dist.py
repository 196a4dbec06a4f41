"""Host logic of bench.py on CPU: the multi-rank path at world size 2 over
gloo (each rank an independent replica, no data-path collective; the job's
throughput is all ranks' tokens over the slowest rank's time; the reference
arm runs on rank 0 only) and the roofline numerators."""
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


def test_algorithmic_work_closed_forms():
    """The roofline numerators against closed forms of the full layer: one
    touched expert's gate+up+down codes and scales are 23,598,720 bytes, and
    a forward's expert FLOPs are rows x 2 x 3 x 5120 x 1536."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import bench
    import gen
    wl = gen.WORKLOADS["decode"]
    sh = wl.shape
    T = 64
    rows = T * (sh.K + sh.S)
    offsets = np.zeros(sh.E + 2, np.int64)
    counts = np.zeros(sh.E + 1, np.int64)
    counts[:T * sh.K // 2] = 2        # 256 experts touched by 512 routed rows
    counts[sh.E] = T                  # the shared expert
    offsets[1:] = np.cumsum(counts)
    w = bench.algorithmic_work(wl, T, offsets)
    assert w["touched_groups"] == 257 and w["rows"] == rows
    act_gu = rows * (5120 + 160) + rows * (1536 + 48)
    act_dn = rows * (1536 + 48) + rows * 5120 * 2
    assert w["bytes"]["gate_up"] + w["bytes"]["down"] == 257 * 23_598_720 + act_gu + act_dn
    assert w["flops"]["gate_up"] + w["flops"]["down"] == rows * 47_185_920
    # a group with no rows costs nothing
    counts[5] = 0
    counts[6] = 4
    offsets[1:] = np.cumsum(counts)
    assert bench.algorithmic_work(wl, T, offsets)["touched_groups"] == 256
