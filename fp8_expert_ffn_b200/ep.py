"""Expert parallelism for the MoE layer across ranks (one process per GPU).

The SGLang cookbook "Dots3-Note" ("2. Configuration Tips") serves this
layer with expert parallelism across the GPUs of a node, DeepEP carrying the
dispatch and combine all-to-alls. Here the routed experts are split into P
contiguous blocks, rank p owning experts [p*El, (p+1)*El) with El = E/P; the
router and the shared expert are on every rank. One forward on rank r:

  1. route and permute its own T tokens (a routing-only handle over all E
     experts): its routed rows come out grouped by expert, so the rows for
     rank p are one contiguous range;
  2. exchange the per-(destination, local expert) row counts, then dispatch
     the FP8 rows and their scales (made row-major) with two all-to-alls;
  3. regroup what arrived (sender-major) into expert-major GEMM input with
     its own shared rows last, run the grouped gate/up and down GEMMs over
     its El experts plus the shared expert, and regroup the output back;
  4. return each sender's rows with a third all-to-all, into the sender's
     own permuted-row order, and combine.

Two transports. ep_forward + CudaOps: the rows cross in torch.distributed
all-to-alls (NCCL between GPUs, each rank's rows landing in its own memory
before any kernel reads them) and are regrouped by the library's kernels.
ep_forward_peer + PeerOps: the library's dispatch kernel writes every routed
row straight into its owner's receive buffer (a peer GPU's memory, mapped
with CUDA IPC through EpComm) at the row the owner's GEMMs read, and the
combine kernel reads the owners' output rows back; the only collectives are
an all-gather of the E+2 offsets of every rank and two barriers.

Host orchestration only: every step of the layer runs in the library's
kernels.
The orchestration takes the compute and the exchange as objects, so tests
can drive the same code with CPU ranks over gloo or with several emulated
ranks on one GPU.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


def local_experts(E: int, ranks: int) -> int:
    """Experts per rank (the routed experts are split evenly)."""
    if ranks < 1 or E % ranks:
        raise ValueError(f"{E} routed experts cannot be split evenly over {ranks} ranks")
    return E // ranks


def plan_dispatch(offsets, E: int, ranks: int) -> np.ndarray:
    """[ranks][El] rows this rank sends to each destination's local experts,
    from its permutation offsets (offsets[e] = first row of expert e)."""
    off = np.asarray(offsets, np.int64)
    return np.diff(off[:E + 1]).reshape(ranks, local_experts(E, ranks))


def rank_layers(layer, rank: int, ranks: int):
    """The two handles rank `rank` of `ranks` runs, built from a whole layer's
    device tensors: a routing-only handle over all E experts (the layer's
    router and its settings) and an expert handle over the rank's block
    [rank*El, (rank+1)*El) plus the shared expert, whose weights are copied
    out of the layer's (index_select) so that the block is contiguous."""
    import torch
    from . import LayerWeights, MoeLayer
    El = local_experts(layer.E, ranks)
    w = layer.weights
    route = MoeLayer(layer.H, layer.E, layer.K, layer.F, LayerWeights(None, None, None, None, None, None, w.router_w),
                     routed_scaling=layer.routed_scaling, n_shared=layer.S, n_group=layer.n_group,
                     topk_group=layer.topk_group, norm_topk=layer.norm_topk, router_bias=layer.router_bias)
    e0 = rank * El
    keep = torch.tensor(list(range(e0, e0 + El)) + ([layer.E] if layer.S else []), device=w.w_gate.device)
    pick = {k: getattr(w, k).index_select(0, keep).contiguous()
            for k in ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down")}
    experts = MoeLayer(layer.H, El, layer.K, layer.F, LayerWeights(router_w=w.router_w[e0:e0 + El].contiguous(), **pick),
                       ld_h=layer.ld_h, ld_f=layer.ld_f, n_shared=layer.S)
    return route, experts


@dataclass
class Dispatch:
    """Row counts of one forward on one rank."""
    send: np.ndarray        # [ranks][El] rows sent to (destination, its local expert)
    recv: np.ndarray        # [ranks][El] rows received from (sender, my local expert)

    @property
    def send_rows(self):
        return [int(v) for v in self.send.sum(1)]

    @property
    def recv_rows(self):
        return [int(v) for v in self.recv.sum(1)]

    @property
    def n_recv(self) -> int:
        return int(self.recv.sum())


class TorchExchange:
    """All-to-all over torch.distributed (NCCL for CUDA tensors, gloo for CPU)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.ranks = dist.get_world_size(group)

    def counts(self, send: np.ndarray, device) -> np.ndarray:
        import torch
        t = torch.from_numpy(np.ascontiguousarray(send, np.int32)).to(device)
        out = torch.empty_like(t)
        self.dist.all_to_all_single(out, t, group=self.group)
        return out.cpu().numpy().astype(np.int64)

    def rows(self, src, send_rows, recv_rows, out):
        """out (first dim sum(recv_rows)) <- the rows of src (first dim
        sum(send_rows)) that each rank sent to this one, in rank order."""
        self.dist.all_to_all_single(out, src, output_split_sizes=list(recv_rows),
                                    input_split_sizes=list(send_rows), group=self.group)
        return out


class CudaOps:
    """The layer's steps on this rank through the library (device tensors)."""

    def __init__(self, route_layer, expert_layer, ranks: int):
        import torch
        from . import torch_utils
        self.torch = torch
        self.tu = torch_utils
        self.route_layer, self.expert_layer, self.ranks = route_layer, expert_layer, ranks
        self.H, self.E, self.K, self.S = route_layer.H, route_layer.E, route_layer.K, route_layer.S
        self.HB = self.H // 128
        self.El = expert_layer.E
        assert self.El * ranks == self.E and expert_layer.S == self.S and expert_layer.K == self.K
        self.device = "cuda"

    def route_permute(self, x, T):
        from . import moe_permute, moe_route
        t, d = self.torch, self.device
        rows = T * (self.K + self.S)
        ws = self.tu.workspace(self.route_layer, T)
        idx = t.empty((T, self.K), dtype=t.int32, device=d)
        w = t.empty((T, self.K), dtype=t.float32, device=d)
        moe_route(self.route_layer, x, T, self.H, idx, w, None, ws, ws.numel())
        # zeros: with T = 0 the permutation writes nothing and the rank still
        # takes part in every exchange with empty sends
        st = {"w": w, "offsets": t.zeros(self.E + 2, dtype=t.int32, device=d),
              "perm": t.empty(rows, dtype=t.int32, device=d),
              "inv": t.empty((T, self.K), dtype=t.int32, device=d),
              "xq": t.empty((rows, self.H), dtype=t.uint8, device=d),
              "xs": t.empty((self.HB, rows), dtype=t.float32, device=d)}
        moe_permute(self.route_layer, x, T, self.H, idx, st["offsets"], st["perm"], st["inv"], st["xq"], st["xs"],
                    ws, ws.numel())
        return st, st["offsets"].cpu().numpy()

    def send_buffers(self, st, T):
        from . import moe_ep_pack_scales
        R = T * self.K
        xs_rows = self.torch.empty((R, self.HB), dtype=self.torch.float32, device=self.device)
        moe_ep_pack_scales(self.route_layer, st["xs"], T, xs_rows)
        return st["xq"][:R], xs_rows

    def recv_buffers(self, n):
        t = self.torch
        return (t.empty((n, self.H), dtype=t.uint8, device=self.device),
                t.empty((n, self.HB), dtype=t.float32, device=self.device))

    def experts(self, st, disp: Dispatch, recv_q, recv_s, T):
        """Regroup, grouped GEMMs over the local experts + shared, regroup back."""
        from . import moe_ep_regroup, moe_ep_unregroup, moe_grouped_down, moe_grouped_gate_up
        t, d = self.torch, self.device
        n = disp.n_recv
        rows = n + T * self.S
        seg = t.from_numpy(np.ascontiguousarray(disp.recv, np.int32)).to(d)
        gq = t.empty((rows, self.H), dtype=t.uint8, device=d)
        gs = t.empty((self.HB, rows), dtype=t.float32, device=d)
        goff = t.empty(self.El + 2, dtype=t.int32, device=d)
        moe_ep_regroup(self.expert_layer, self.ranks, seg, n, recv_q, recv_s, st["xq"], st["xs"], T, gq, gs, goff)
        FB = -(-self.expert_layer.F // 128)
        h = t.empty((rows, FB * 128), dtype=t.uint8, device=d)
        hs = t.empty((FB, rows), dtype=t.float32, device=d)
        y_g = t.empty((rows, self.H), dtype=t.bfloat16, device=d)
        moe_grouped_gate_up(self.expert_layer, gq, gs, goff, rows, h, hs)
        moe_grouped_down(self.expert_layer, h, hs, goff, rows, y_g)
        y_send = t.empty((n, self.H), dtype=t.bfloat16, device=d)
        y_own = t.empty((T * (self.K + self.S), self.H), dtype=t.bfloat16, device=d)
        moe_ep_unregroup(self.expert_layer, self.ranks, seg, n, y_g, T, y_send, y_own)
        return y_send, y_own

    def combine(self, st, y_own, T):
        from . import moe_combine
        out = self.torch.empty((T, self.H), dtype=self.torch.bfloat16, device=self.device)
        moe_combine(self.route_layer, y_own, st["inv"], st["w"], T, out, self.H)
        return out


def ep_forward(ops, exchange, x, T: int):
    """One expert-parallel forward of this rank's T tokens (see the module
    docstring); returns its [T][H] output."""
    st, offsets = ops.route_permute(x, T)
    send = plan_dispatch(offsets, ops.E, ops.ranks)
    disp = Dispatch(send, exchange.counts(send, ops.device))
    q_send, s_send = ops.send_buffers(st, T)
    recv_q, recv_s = ops.recv_buffers(disp.n_recv)
    exchange.rows(q_send, disp.send_rows, disp.recv_rows, recv_q)
    exchange.rows(s_send, disp.send_rows, disp.recv_rows, recv_s)
    y_send, y_own = ops.experts(st, disp, recv_q, recv_s, T)
    R = T * ops.K
    exchange.rows(y_send, disp.recv_rows, disp.send_rows, y_own[:R])
    return ops.combine(st, y_own, T)


# ----------------------------------------------------------------------------- over peer memory

class PeerOps:
    """The layer's steps on this rank with the dispatch and combine over
    peer memory (moe_ep_plan / moe_ep_dispatch / moe_ep_combine): routed
    rows are written straight into their owners' receive buffers and read
    back from the owners' output rows, so no row crosses an all-to-all and
    no regroup is needed. `comm` is this rank's connected EpComm."""

    def __init__(self, route_layer, expert_layer, comm, ranks: int):
        import torch
        from . import torch_utils
        self.torch, self.tu = torch, torch_utils
        self.route_layer, self.expert_layer, self.comm, self.ranks = route_layer, expert_layer, comm, ranks
        self.H, self.E, self.K, self.S = route_layer.H, route_layer.E, route_layer.K, route_layer.S
        self.El = expert_layer.E
        assert self.El * ranks == self.E and expert_layer.S == self.S and expert_layer.K == self.K
        assert comm.ranks == ranks
        cap = comm.capacity
        FB = -(-expert_layer.F // 128)
        d = "cuda"
        self.h = torch.empty((cap, FB * 128), dtype=torch.uint8, device=d)
        self.hs = torch.empty((FB, cap), dtype=torch.float32, device=d)
        self.goff = torch.empty(self.El + 2, dtype=torch.int32, device=d)
        self.device = d

    def _buffers(self, T):
        """Per-token buffers and the routing workspace, kept between forwards
        (stream order makes the reuse safe) and regrown for a larger T."""
        t = self.torch
        if getattr(self, "_T", -1) < T:
            self._T = T
            self._ws = self.tu.workspace(self.route_layer, T) if T else None
            self._idx = t.empty((T, self.K), dtype=t.int32, device=self.device)
            self._w = t.empty((T, self.K), dtype=t.float32, device=self.device)
            self._inv = t.empty((T, self.K), dtype=t.int32, device=self.device)
            self._off = t.empty(self.E + 2, dtype=t.int32, device=self.device)
        return self._ws, self._idx[:T], self._w[:T], self._inv[:T], self._off

    def plan(self, x, T):
        from . import moe_ep_plan, moe_route
        ws, idx, w, inv, off = self._buffers(T)
        st = {"x": x, "ws": ws if T else None, "idx": idx, "w": w, "inv": inv}
        nb = st["ws"].numel() if T else 0
        if T:
            moe_route(self.route_layer, x, T, self.H, st["idx"], st["w"], None, st["ws"], nb)
        moe_ep_plan(self.route_layer, st["idx"], T, off, st["ws"], nb)
        return st, off

    def dispatch(self, st, all_off, T):
        from . import moe_ep_dispatch
        nb = st["ws"].numel() if T else 0
        moe_ep_dispatch(self.route_layer, self.comm, st["x"], T, self.H, st["idx"], all_off, st["inv"], self.goff,
                        st["ws"], nb)

    def experts(self, st):
        from . import moe_grouped_down, moe_grouped_gate_up
        c = self.comm
        moe_grouped_gate_up(self.expert_layer, c.recv_q, c.recv_s, self.goff, c.capacity, self.h, self.hs)
        moe_grouped_down(self.expert_layer, self.h, self.hs, self.goff, c.capacity, c.y)

    def combine(self, st, T):
        from . import moe_ep_combine
        out = self.torch.empty((T, self.H), dtype=self.torch.bfloat16, device=self.device)
        moe_ep_combine(self.route_layer, self.comm, st["idx"], st["inv"], st["w"], self.goff, T, out, self.H)
        return out


class TorchSync:
    """The two collectives of the peer-memory forward over torch.distributed
    (NCCL: both are queued on the current stream, so no host wait): an
    all-gather of every rank's offsets and a barrier (an all-reduce of one
    word)."""

    def __init__(self, group=None, device="cuda"):
        import torch
        import torch.distributed as dist
        self.torch, self.dist, self.group = torch, dist, group
        self.ranks = dist.get_world_size(group)
        self.word = torch.zeros(1, dtype=torch.int32, device=device)

    def all_gather(self, off):
        out = self.torch.empty((self.ranks, off.numel()), dtype=off.dtype, device=off.device)
        self.dist.all_gather_into_tensor(out, off.contiguous(), group=self.group)
        return out

    def barrier(self):
        self.dist.all_reduce(self.word, group=self.group)


def connect_peers(comm, group=None):
    """Maps every other rank's exchange buffers into this one (EpComm):
    the ranks swap their buffer handles with torch.distributed (any backend)
    and each opens the others'. Call on every rank of the group together."""
    import torch.distributed as dist
    ranks = dist.get_world_size(group)
    if ranks != comm.ranks or dist.get_rank(group) != comm.rank:
        raise ValueError("the comm's rank and ranks must be this process's in the group")
    if ranks == 1:
        return comm
    handles = [None] * ranks
    dist.all_gather_object(handles, comm.export(), group=group)
    comm.connect(handles)
    return comm


def peer_capacity(tokens_per_rank: int, K: int, S: int, ranks: int) -> int:
    """Receive rows that always suffice: every rank's routed rows going to
    one owner, plus that owner's shared rows."""
    return max(1, ranks * tokens_per_rank * K + tokens_per_rank * S)


def ep_forward_peer(ops, sync, x, T: int):
    """One expert-parallel forward of this rank's T tokens over peer memory:
    plan, all-gather the offsets, dispatch into the owners' buffers, barrier,
    the grouped GEMMs on this rank's buffer, barrier, combine from the
    owners' output rows. Returns the [T][H] output."""
    st, off = ops.plan(x, T)
    all_off = sync.all_gather(off)
    ops.dispatch(st, all_off, T)
    sync.barrier()
    ops.experts(st)
    sync.barrier()
    return ops.combine(st, T)
