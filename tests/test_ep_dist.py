"""Expert parallelism on CPU ranks over gloo: the library's orchestration
(fp8_expert_ffn_b200.ep: dispatch planning, count exchange, the three
all-to-alls and their split sizes) driven with CPU stand-ins for the
kernels, built from the oracle (test infrastructure). Each rank's output must
equal the oracle's single-rank layer on the same tokens, which holds only if
every row reaches the rank that owns its expert and comes back to its place.
The kernels themselves are checked on one GPU with emulated ranks
(tests/test_gpu_ep.py)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class HostOps:
    """The layer's steps on CPU (oracle arithmetic), in the interface of
    fp8_expert_ffn_b200.ep.CudaOps."""

    def __init__(self, layer, rank, ranks):
        import gen
        from oracle import moe
        self.moe, self.layer = moe, layer
        sh = layer.shape
        self.H, self.E, self.K, self.S, self.HB = sh.H, sh.E, sh.K, sh.S, sh.HB
        self.ranks, self.rank = ranks, rank
        self.El = sh.E // ranks
        self.device = "cpu"
        e0 = rank * self.El
        keep = list(range(e0, e0 + self.El)) + ([sh.E] if sh.S else [])
        ls = gen.LayerShape(H=sh.H, E=self.El, K=sh.K, F=sh.F, ld_f=sh.ld_f, S=sh.S)
        self.local = gen.Layer(ls, layer.router_w[e0:e0 + self.El], layer.w_gate[keep], layer.s_gate[keep],
                               layer.w_up[keep], layer.s_up[keep], layer.w_down[keep], layer.s_down[keep])

    def route_permute(self, x, T):
        m = self.moe
        r = m.route_layer(x, self.layer)
        p = m.permute(r.idx, self.E, self.S)
        tq, ts = m.quantize_tokens(x)
        return {"w": r.w, "inv": p.inv, "xq": tq[p.perm], "xs": ts[p.perm]}, p.offsets

    def send_buffers(self, st, T):
        R = T * self.K
        return torch.from_numpy(np.ascontiguousarray(st["xq"][:R])), torch.from_numpy(np.ascontiguousarray(st["xs"][:R]))

    def recv_buffers(self, n):
        return torch.empty((n, self.H), dtype=torch.uint8), torch.empty((n, self.HB), dtype=torch.float32)

    def experts(self, st, disp, recv_q, recv_s, T):
        P, El, R = self.ranks, self.El, T * self.K
        cnt = disp.recv                                     # [sender][local expert]
        start = np.concatenate([[0], np.cumsum(cnt.ravel())])[:-1].reshape(P, El)   # sender-major
        order = [np.arange(start[s, e], start[s, e] + cnt[s, e]) for e in range(El) for s in range(P)]
        order = np.concatenate(order).astype(np.int64) if order else np.zeros(0, np.int64)
        q = np.concatenate([recv_q.numpy()[order], st["xq"][R:R + T * self.S]])
        s = np.concatenate([recv_s.numpy()[order], st["xs"][R:R + T * self.S]])
        off = np.concatenate([[0], np.cumsum(cnt.sum(0)), [len(order) + T * self.S]]).astype(np.int64)
        y = self.moe.expert_ffn_rows(q, s, off, self.local)["y"]
        y_send = np.empty((disp.n_recv, self.H))
        y_send[order] = y[:len(order)]
        y_own = np.zeros((T * (self.K + self.S), self.H))
        y_own[R:] = y[len(order):]
        return torch.from_numpy(y_send), torch.from_numpy(y_own)

    def combine(self, st, y_own, T):
        return self.moe.combine(y_own.numpy(), st["inv"], st["w"], self.S)


def _worker(rank, world, port, T, q, idle_rank=-1):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import gen
        from fp8_expert_ffn_b200 import ep
        from oracle import moe
        _, layer, _ = gen.workload_inputs("toy")
        Tr = 0 if rank == idle_rank else T
        x = gen.make_x(Tr, layer.shape.H, 100 + rank, outliers=2)   # each rank has its own tokens
        out = ep.ep_forward(HostOps(layer, rank, world), ep.TorchExchange(), x, Tr)
        if Tr == 0:
            err = 0.0 if out.shape == (0, layer.shape.H) else 1.0
        else:
            ref = moe.layer_forward(x, layer)["out"]
            err = float(np.max(np.abs(out - ref)) / np.max(np.abs(ref)))
        sent = ep.plan_dispatch(moe.permute(moe.route_layer(x, layer).idx, layer.shape.E).offsets,
                                layer.shape.E, world)
        q.put((rank, err, int(sent.sum()) + (T * 4 if Tr == 0 else 0)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,idle", [(2, -1), (4, -1), (2, 1)])
def test_expert_parallel_forward_matches_single_rank(world, idle):
    """world ranks of 24 tokens each; with idle >= 0 that rank has no tokens
    (it still serves its experts and takes part in every exchange)."""
    T = 24
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, T, q, idle)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, err, sent in res:
        assert err <= 1e-12, (rank, err)
        assert sent == T * 4          # every routed row (T x top-4) is dispatched once


def test_plan_dispatch_splits_rows_by_owner():
    from fp8_expert_ffn_b200 import ep
    E, P = 8, 4
    counts = np.array([3, 0, 2, 5, 1, 1, 0, 4])
    offsets = np.concatenate([[0], np.cumsum(counts), [counts.sum() + 6]])
    plan = ep.plan_dispatch(offsets, E, P)
    assert plan.tolist() == [[3, 0], [2, 5], [1, 1], [0, 4]]
    d = ep.Dispatch(plan, plan[::-1].copy())
    assert d.send_rows == [3, 7, 2, 4] and d.recv_rows == [4, 2, 7, 3] and d.n_recv == 16
    with pytest.raises(ValueError):
        ep.local_experts(10, 4)


# ----------------------------------------------------------------------------- over peer memory

class HostPeerOps:
    """ep.PeerOps's interface on CPU: every rank's receive buffers are
    shared-memory tensors that all processes map (the stand-in for a peer
    GPU's memory), and the steps are the oracle's. The dispatch writes each
    routed row at the owner-side row that include/moe.h defines: owner p
    holds, for its local experts in turn, sender 0's rows, sender 1's, ...,
    then its own shared rows."""

    def __init__(self, layer, rank, ranks, bufs):
        self.base = HostOps(layer, rank, ranks)
        self.moe, self.layer, self.bufs = self.base.moe, layer, bufs
        self.E, self.K, self.S, self.H = self.base.E, self.base.K, self.base.S, self.base.H
        self.El, self.rank, self.ranks = self.base.El, rank, ranks

    def plan(self, x, T):
        m = self.moe
        r = m.route_layer(x, self.layer)
        p = m.permute(r.idx, self.E, self.S)
        tq, ts = m.quantize_tokens(x)
        st = {"idx": r.idx, "w": r.w, "inv": p.inv, "perm": p.perm, "offsets": p.offsets, "tq": tq, "ts": ts, "T": T}
        return st, torch.from_numpy(p.offsets.astype(np.int32))

    def dispatch(self, st, all_off, T):
        ao = np.asarray(all_off, np.int64)
        cnt = np.diff(ao[:, :self.E + 1], axis=1)              # [sender][expert]
        tot, pre = cnt.sum(0), cnt[:self.rank].sum(0)
        off, El = st["offsets"], self.El
        for g in range(self.E):
            p, b0 = g // El, (g // El) * El
            base = int(tot[b0:g].sum() + pre[g])
            rows = np.arange(off[g], off[g + 1])
            toks = st["perm"][rows]
            self.bufs[p]["q"][base:base + len(rows)] = torch.from_numpy(st["tq"][toks])
            self.bufs[p]["s"][base:base + len(rows)] = torch.from_numpy(st["ts"][toks])
            st.setdefault("where", {}).update({int(r): (p, base + i) for i, r in enumerate(rows)})
        mine = tot[self.rank * El:(self.rank + 1) * El]
        n_r = int(mine.sum())
        self.bufs[self.rank]["q"][n_r:n_r + T * self.S] = torch.from_numpy(st["tq"][:T])
        self.bufs[self.rank]["s"][n_r:n_r + T * self.S] = torch.from_numpy(st["ts"][:T])
        st["goff"] = np.concatenate([[0], np.cumsum(mine), [n_r + T * self.S]]).astype(np.int64)

    def experts(self, st):
        goff, n = st["goff"], int(st["goff"][-1])
        b = self.bufs[self.rank]
        y = self.moe.expert_ffn_rows(b["q"][:n].numpy(), b["s"][:n].numpy(), goff, self.base.local)["y"]
        b["y"][:n] = torch.from_numpy(y)

    def combine(self, st, T):
        R = T * self.K
        y_local = np.zeros((R + T * self.S, self.H))
        for r, (p, row) in st.get("where", {}).items():
            y_local[r] = self.bufs[p]["y"][row].numpy()
        n_r = int(st["goff"][self.El])
        y_local[R:] = self.bufs[self.rank]["y"][n_r:n_r + T * self.S].numpy()
        return self.moe.combine(y_local, st["inv"], st["w"], self.S)


class GlooSync:
    def all_gather(self, off):
        out = [torch.empty_like(off) for _ in range(dist.get_world_size())]
        dist.all_gather(out, off)
        return torch.stack(out)

    def barrier(self):
        dist.barrier()


def _peer_worker(rank, world, port, T, bufs, q, idle_rank=-1):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import gen
        from fp8_expert_ffn_b200 import ep
        from oracle import moe
        _, layer, _ = gen.workload_inputs("toy")
        Tr = 0 if rank == idle_rank else T
        x = gen.make_x(Tr, layer.shape.H, 100 + rank, outliers=2)
        ops = HostPeerOps(layer, rank, world, bufs)
        outs = [ep.ep_forward_peer(ops, GlooSync(), x, Tr) for _ in range(2)]   # buffers reused
        if Tr == 0:
            err = max(0.0 if o.shape == (0, layer.shape.H) else 1.0 for o in outs)
        else:
            ref = moe.layer_forward(x, layer)["out"]
            err = max(float(np.max(np.abs(o - ref)) / np.max(np.abs(ref))) for o in outs)
        q.put((rank, err))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,idle", [(2, -1), (4, -1), (4, 2)])
def test_peer_transport_forward_matches_single_rank(world, idle):
    """ep.ep_forward_peer's order of steps and collectives across processes,
    with the ranks' buffers in shared memory: every rank's output equals the
    oracle's single-rank layer, twice in a row on the same buffers."""
    from fp8_expert_ffn_b200 import ep
    import gen
    _, layer, _ = gen.workload_inputs("toy")
    sh = layer.shape
    T = 24
    cap = ep.peer_capacity(T, sh.K, sh.S, world)
    bufs = [{"q": torch.zeros((cap, sh.H), dtype=torch.uint8).share_memory_(),
             "s": torch.zeros((cap, sh.HB), dtype=torch.float64).share_memory_(),
             "y": torch.zeros((cap, sh.H), dtype=torch.float64).share_memory_()} for _ in range(world)]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_peer_worker, args=(r, world, port, T, bufs, q, idle)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, err in res:
        assert err <= 1e-12, (rank, err)


def _failing_worker(rank, world, port, T, bufs, q, dead_rank):
    """dead_rank leaves between steps (after the first forward, before the
    second: nothing of its own in flight); the others must see an error from
    their next collective, not hang."""
    import sys
    from datetime import timedelta
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=20))
    import gen
    from fp8_expert_ffn_b200 import ep
    _, layer, _ = gen.workload_inputs("toy")
    x = gen.make_x(T, layer.shape.H, 100 + rank, outliers=2)
    ops = HostPeerOps(layer, rank, world, bufs)
    ep.ep_forward_peer(ops, GlooSync(), x, T)
    if rank == dead_rank:
        os._exit(3)                      # the rank is gone: no goodbye to the others
    try:
        ep.ep_forward_peer(ops, GlooSync(), x, T)
        q.put((rank, "no error"))
    except Exception as e:               # noqa: BLE001 - the failure is the expected outcome
        q.put((rank, type(e).__name__))
    q.close()
    q.join_thread()                      # the message is sent before the process leaves
    os._exit(0)


def test_peer_transport_reports_a_dead_rank():
    """A rank that dies between forwards: every other rank's next forward
    fails in its first collective (the offsets all-gather) with an error
    instead of waiting for ever; no kernel is involved (host stand-ins)."""
    from fp8_expert_ffn_b200 import ep
    import gen
    import time
    _, layer, _ = gen.workload_inputs("toy")
    sh = layer.shape
    world, T, dead = 4, 16, 1
    cap = ep.peer_capacity(T, sh.K, sh.S, world)
    bufs = [{"q": torch.zeros((cap, sh.H), dtype=torch.uint8).share_memory_(),
             "s": torch.zeros((cap, sh.HB), dtype=torch.float64).share_memory_(),
             "y": torch.zeros((cap, sh.H), dtype=torch.float64).share_memory_()} for _ in range(world)]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_worker, args=(r, world, port, T, bufs, q, dead)) for r in range(world)]
    t0 = time.time()
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode is not None for p in procs), "a rank hung"
    assert procs[dead].exitcode == 3
    res = sorted(q.get(timeout=10) for _ in range(world - 1))
    assert [r for r, _ in res] == [r for r in range(world) if r != dead]
    assert all(outcome in ("RuntimeError", "DistBackendError", "DistNetworkError", "DistError") for _, outcome in res), res
    assert time.time() - t0 < 120
