"""Expert parallelism through the library's kernels on one GPU: P emulated
ranks run as threads (both transports: the all-to-all one and the one over
peer memory, whose "peers" are then buffers on this GPU), each with a routing-only handle over all experts and
an expert handle over its own block of experts plus the shared expert; an
in-process exchange stands in for the all-to-alls (no collective, no kernel
waits on another). Each rank's output must be bit-identical to the
single-GPU forward of the whole layer on the same tokens: a row's GEMM
result does not depend on which rows share its tile, so any row sent to the
wrong expert or returned to the wrong place shows up."""
import threading

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import gen  # noqa: E402

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

import fp8_expert_ffn_b200 as fx  # noqa: E402
from fp8_expert_ffn_b200 import ep  # noqa: E402
from fp8_expert_ffn_b200 import torch_utils as tu  # noqa: E402


class LocalExchange:
    """The all-to-alls between emulated ranks (threads of this process)."""

    def __init__(self, ranks):
        self.ranks = ranks
        self.bar = threading.Barrier(ranks, timeout=300)
        self.box = [None] * ranks

    def view(self, rank):
        return _RankView(self, rank)


class _RankView:
    def __init__(self, ex, rank):
        self.ex, self.rank, self.ranks = ex, rank, ex.ranks

    def counts(self, send, device):
        self.ex.box[self.rank] = np.asarray(send)
        self.ex.bar.wait()
        recv = np.stack([self.ex.box[s][self.rank] for s in range(self.ranks)]).astype(np.int64)
        self.ex.bar.wait()
        return recv

    def rows(self, src, send_rows, recv_rows, out):
        torch.cuda.synchronize()
        self.ex.box[self.rank] = (src, list(send_rows))
        self.ex.bar.wait()
        o = 0
        for s in range(self.ranks):
            ssrc, ssend = self.ex.box[s]
            a, n = sum(ssend[:self.rank]), ssend[self.rank]
            assert n == recv_rows[s]
            if n:
                out[o:o + n].copy_(ssrc[a:a + n])
            o += n
        torch.cuda.synchronize()
        self.ex.bar.wait()
        return out


def _run(name, ranks, T, layer=None, xs=None):
    wl, layer0, _ = gen.workload_inputs(name)
    layer = layer0 if layer is None else layer
    sh = layer.shape
    dev = tu.upload_layer(layer)
    if xs is None:
        xs = [gen.make_x(T, sh.H, 200 + r, outliers=wl.outliers) for r in range(ranks)]
    refs = []
    for x in xs:
        xt = tu.bf16_tensor(x)
        o = torch.empty((T, sh.H), dtype=torch.bfloat16, device="cuda")
        ws = tu.workspace(dev, T)
        fx.moe_layer_forward(dev, xt, T, sh.H, o, sh.H, ws, ws.numel())
        refs.append(o)
    layers = [ep.rank_layers(dev, r, ranks) for r in range(ranks)]
    ex = LocalExchange(ranks)
    outs, errs = [None] * ranks, []

    def one(r):
        try:
            torch.cuda.set_device(0)
            ops = ep.CudaOps(layers[r][0], layers[r][1], ranks)
            outs[r] = ep.ep_forward(ops, ex.view(r), tu.bf16_tensor(xs[r]), T)
        except BaseException as e:   # noqa: BLE001 - re-raised below
            errs.append(e)
            ex.bar.abort()

    th = [threading.Thread(target=one, args=(r,)) for r in range(ranks)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    if errs:
        raise errs[0]
    for r in range(ranks):
        code, bits = fx.moe_get_device_status(layers[r][1])
        assert code == fx.MOE_OK, hex(bits)
        assert torch.equal(outs[r].view(torch.int16), refs[r].view(torch.int16)), f"rank {r} differs"


@pytest.mark.parametrize("ranks", [2, 4])
def test_expert_parallel_toy_layer_matches_single_gpu(ranks):
    _run("toy", ranks, 512)


def test_expert_parallel_full_layer_two_ranks():
    """256 routed experts split 128 + 128, 64 tokens per rank."""
    _run("decode", 2, 64)


def test_expert_parallel_rank_with_no_routed_rows():
    """A router whose top-4 always falls in rank 0's experts: rank 1 receives
    no routed rows (n_recv = 0) and runs only its own shared rows."""
    from oracle import moe
    wl, layer, _ = gen.workload_inputs("toy")
    sh = layer.shape
    router = layer.router_w.copy()
    router[sh.E // 2:, :] = 0.0
    router[sh.E // 2:, 0] = -30.0       # with x[:, 0] = 1: logit -30 for experts 8..15
    biased = gen.Layer(sh, router, layer.w_gate, layer.s_gate, layer.w_up, layer.s_up, layer.w_down, layer.s_down)
    T = 512
    xs = []
    for r in range(2):
        x = gen.make_x(T, sh.H, 200 + r, outliers=2)
        x[:, 0] = gen.f32_to_bf16_bits(np.float32([1.0]))[0]
        assert moe.route(x, router, sh.K).idx.max() < sh.E // 2
        xs.append(x)
    _run("toy", 2, T, layer=biased, xs=xs)


def test_routing_only_handle_refuses_gemm_calls():
    wl, layer, _ = gen.workload_inputs("toy")
    sh = layer.shape
    dev = tu.upload_layer(layer)
    route = fx.MoeLayer(sh.H, sh.E, sh.K, sh.F, fx.LayerWeights(None, None, None, None, None, None,
                                                                 dev.weights.router_w), n_shared=sh.S)
    T = 8
    # a routing-only handle's workspace is the route and permutation scratch alone
    assert 0 < fx.moe_workspace_size(route, 4096) < fx.moe_workspace_size(dev, 4096) // 10
    x = torch.zeros((T, sh.H), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(x)
    ws = tu.workspace(route, T)
    with pytest.raises(fx.MoeError) as e:
        fx.moe_layer_forward(route, x, T, sh.H, out, sh.H, ws, ws.numel())
    assert e.value.code == fx.MOE_ERR_INVALID_ARG


# ----------------------------------------------------------------------------- over peer memory

class LocalSync:
    """The offsets all-gather and the barriers between emulated ranks
    (threads of this process; every rank's kernels are finished before it
    reaches a barrier, so no kernel waits on another)."""

    def __init__(self, ranks):
        self.ranks = ranks
        self.bar = threading.Barrier(ranks, timeout=300)
        self.box = [None] * ranks

    def view(self, rank):
        return _SyncView(self, rank)


class _SyncView:
    def __init__(self, s, rank):
        self.s, self.rank = s, rank

    def all_gather(self, off):
        torch.cuda.synchronize()
        self.s.box[self.rank] = off
        self.s.bar.wait()
        out = torch.stack(list(self.s.box))
        self.s.bar.wait()
        return out

    def barrier(self):
        torch.cuda.synchronize()
        self.s.bar.wait()


def _run_peer(name, ranks, T, layer=None, xs=None, capacity=None, expect_overflow=False):
    wl, layer0, _ = gen.workload_inputs(name)
    layer = layer0 if layer is None else layer
    sh = layer.shape
    dev = tu.upload_layer(layer)
    if xs is None:
        xs = [gen.make_x(T, sh.H, 300 + r, outliers=wl.outliers) for r in range(ranks)]
    refs = []
    for x in xs:
        Tr = x.shape[0]
        o = torch.empty((Tr, sh.H), dtype=torch.bfloat16, device="cuda")
        if Tr:
            ws = tu.workspace(dev, Tr)
            fx.moe_layer_forward(dev, tu.bf16_tensor(x), Tr, sh.H, o, sh.H, ws, ws.numel())
        refs.append(o)
    layers = [ep.rank_layers(dev, r, ranks) for r in range(ranks)]
    cap = capacity or ep.peer_capacity(max(x.shape[0] for x in xs), sh.K, sh.S, ranks)
    comms = [fx.EpComm(layers[r][0], r, ranks, cap) for r in range(ranks)]
    fx.EpComm.connect_local(comms)
    sync = LocalSync(ranks)
    outs, errs = [None] * ranks, []

    def one(r):
        try:
            torch.cuda.set_device(0)
            ops = ep.PeerOps(layers[r][0], layers[r][1], comms[r], ranks)
            outs[r] = ep.ep_forward_peer(ops, sync.view(r), tu.bf16_tensor(xs[r]), xs[r].shape[0])
        except BaseException as e:   # noqa: BLE001 - re-raised below
            errs.append(e)
            sync.bar.abort()

    th = [threading.Thread(target=one, args=(r,)) for r in range(ranks)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    if errs:
        raise errs[0]
    for r in range(ranks):
        code, bits = fx.moe_get_device_status(layers[r][0])
        if expect_overflow:
            assert code == fx.MOE_ERR_DEVICE and bits == 0x10, hex(bits)
            continue
        assert code == fx.MOE_OK, hex(bits)
        assert fx.moe_get_device_status(layers[r][1])[0] == fx.MOE_OK
        assert torch.equal(outs[r].view(torch.int16), refs[r].view(torch.int16)), f"rank {r} differs"
    for c in comms:
        c.close()


@pytest.mark.parametrize("ranks", [1, 2, 4])
def test_peer_dispatch_toy_layer_matches_single_gpu(ranks):
    """Dispatch into the owners' buffers, grouped GEMMs on each owner's
    buffer, combine from the owners' rows: bit-identical to the single-GPU
    forward of the whole layer on every rank's tokens."""
    _run_peer("toy", ranks, 512)


def test_peer_dispatch_full_layer_two_ranks():
    """256 routed experts split 128 + 128, 64 tokens per rank (decode)."""
    _run_peer("decode", 2, 64)


def test_peer_dispatch_full_layer_eight_ranks_ragged():
    """8 ranks of 32 experts with different token counts per rank (one
    with none): owners receive from every sender, sizes not multiples of 32."""
    wl, layer, _ = gen.workload_inputs("decode")
    counts = [64, 1, 0, 37, 128, 5, 64, 33]
    xs = [gen.make_x(n, layer.shape.H, 400 + r, outliers=wl.outliers) for r, n in enumerate(counts)]
    _run_peer("decode", 8, None, xs=xs)


def test_peer_dispatch_overflow_is_flagged_and_dispatches_nothing():
    """A capacity below some owner's rows: every rank flags
    MOE_STATUS_EP_OVERFLOW, writes zero group offsets (the GEMMs do
    nothing) and no row is written out of bounds."""
    _run_peer("toy", 2, 64, capacity=16, expect_overflow=True)


@pytest.mark.parametrize("case", ["short_own_entry", "descending"])
def test_peer_dispatch_inconsistent_offsets_flag_bad_plan(case):
    """All-gathered offsets that do not match the plan: rows of this rank
    beyond its own entry are skipped (the rest still dispatched), and
    offsets that descend dispatch nothing; both set MOE_STATUS_BAD_PLAN and
    no store leaves the owners' buffers (the GEMMs and the combine then run
    normally on what is there)."""
    wl, layer, _ = gen.workload_inputs("toy")
    sh = layer.shape
    dev = tu.upload_layer(layer)
    ranks, T = 2, 64
    layers = [ep.rank_layers(dev, r, ranks) for r in range(ranks)]
    cap = ep.peer_capacity(T, sh.K, sh.S, ranks)
    comms = [fx.EpComm(layers[r][0], r, ranks, cap) for r in range(ranks)]
    fx.EpComm.connect_local(comms)
    ops = [ep.PeerOps(layers[r][0], layers[r][1], comms[r], ranks) for r in range(ranks)]
    xs = [tu.bf16_tensor(gen.make_x(T, sh.H, 600 + r, outliers=2)) for r in range(ranks)]
    plans = [ops[r].plan(xs[r], T) for r in range(ranks)]
    all_off = torch.stack([off for _, off in plans])
    bad = all_off.clone()
    if case == "short_own_entry":
        e = int(torch.argmax(torch.diff(all_off[0][:sh.E + 1])))   # rank 0's fullest expert
        bad[0, e + 1:] -= 1                # its count one short: one row of rank 0 is not its plan
    else:
        bad[1, 3] = bad[1, 4] + 5          # rank 1's offsets descend at expert 3
    for r in range(ranks):
        plans[r][0]["x"] = xs[r]
        ops[r].dispatch(plans[r][0], bad, T)
    torch.cuda.synchronize()
    bits = [fx.moe_get_device_status(layers[r][0])[1] for r in range(ranks)]
    if case == "short_own_entry":
        assert bits[0] == 0x8 and bits[1] == 0, [hex(b) for b in bits]
        inv0 = plans[0][0]["inv"]
        assert int((inv0 < 0).sum()) == 1          # exactly the one row beyond the entry skipped
    else:
        assert all(b == 0x8 for b in bits), [hex(b) for b in bits]
        assert all(int((ops[r].goff != 0).sum()) == 0 for r in range(ranks))
        assert all(bool((plans[r][0]["inv"] < 0).all()) for r in range(ranks))
    for r in range(ranks):
        ops[r].experts(plans[r][0])
        ops[r].combine(plans[r][0], T)
    torch.cuda.synchronize()
    for r in range(ranks):
        for h in layers[r]:
            assert fx.moe_get_device_status(h)[0] == fx.MOE_OK
    for c in comms:
        c.close()


def test_peer_dispatch_zipf_skewed_routing_four_ranks():
    """The Zipf-biased router of the long prefill (the hottest expert about
    ten times the mean load, some experts empty), 1024 tokens on each of 4
    ranks: the owners of the hot experts receive far more rows than the
    others, all within the default capacity."""
    wl, layer, _ = gen.workload_inputs("zipf")
    xs = [gen.make_x(1024, layer.shape.H, 700 + r, outliers=wl.outliers, zipf=True) for r in range(4)]
    _run_peer("zipf", 4, None, xs=xs)


@pytest.mark.parametrize("transport", ["peer", "all_to_all"])
def test_expert_parallel_router_variants(transport):
    """Group-limited top-k, a selection-only bias, norm_topk_prob off and
    routed_scaling 2 on the toy layer: the routing-only handle of every rank
    carries the layer's router settings (ep.rank_layers), so each rank's
    output stays bit-identical to the single-GPU forward."""
    wl, layer0, _ = gen.workload_inputs("toy")
    sh = layer0.shape
    layer = gen.Layer(sh, layer0.router_w, layer0.w_gate, layer0.s_gate, layer0.w_up, layer0.s_up,
                      layer0.w_down, layer0.s_down)
    layer.n_group, layer.topk_group, layer.norm_topk, layer.routed_scaling = 8, 3, False, 2.0
    layer.router_bias = np.random.default_rng(31).normal(0, 1.0 / sh.E, sh.E).astype(np.float32)
    xs = [gen.make_x(256, sh.H, 800 + r, outliers=2) for r in range(2)]
    if transport == "peer":
        _run_peer("toy", 2, None, layer=layer, xs=xs)
    else:
        _run("toy", 2, 256, layer=layer, xs=xs)


class _OneRank:
    def all_gather(self, off):
        return off.unsqueeze(0)

    def barrier(self):
        pass


def test_peer_forward_has_no_host_sync_and_replays_in_a_graph():
    """The peer-memory forward of one rank reads nothing back to the host: it
    captures into a CUDA graph (a host read would break the capture), and
    replays give the fused forward's bytes for new inputs."""
    wl, layer, _ = gen.workload_inputs("toy")
    sh, T = layer.shape, 256
    dev = tu.upload_layer(layer)
    route, experts = ep.rank_layers(dev, 0, 1)
    comm = fx.EpComm(route, 0, 1, ep.peer_capacity(T, sh.K, sh.S, 1))
    ops, sync = ep.PeerOps(route, experts, comm, 1), _OneRank()
    x = tu.bf16_tensor(gen.make_x(T, sh.H, 900, outliers=2))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        ep.ep_forward_peer(ops, sync, x, T)          # buffers allocated outside the capture
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        out = ep.ep_forward_peer(ops, sync, x, T)
    ref = torch.empty_like(out)
    ws = tu.workspace(dev, T)
    for seed in (901, 902):
        x.copy_(tu.bf16_tensor(gen.make_x(T, sh.H, seed, outliers=2)))
        g.replay()
        fx.moe_layer_forward(dev, x, T, sh.H, ref, sh.H, ws, ws.numel())
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    for h in (route, experts):
        assert fx.moe_get_device_status(h)[0] == fx.MOE_OK
    del g
    comm.close()
