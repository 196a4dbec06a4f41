"""Expert parallelism over peer memory across processes: two ranks as two
processes on one GPU, each mapping the other's exchange buffers through
CUDA IPC (EpComm.export / connect), exactly as ranks on separate GPUs do.
The all-gather and the barriers go over gloo on the host after a device
synchronise, so no kernel ever waits on another process. Each rank's
output must be bit-identical to the single-GPU forward of the whole layer
on its tokens."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class HostSync:
    """The peer-memory forward's collectives over gloo: the device work
    before each is finished first."""

    def __init__(self, dist):
        self.dist = dist
        self.ranks = dist.get_world_size()

    def all_gather(self, off):
        torch.cuda.synchronize()
        host = off.cpu()
        out = [torch.empty_like(host) for _ in range(self.ranks)]
        self.dist.all_gather(out, host)
        return torch.stack(out).cuda()

    def barrier(self):
        torch.cuda.synchronize()
        self.dist.barrier()


def _worker(rank, world, port, T, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        torch.cuda.set_device(0)
        import gen
        import fp8_expert_ffn_b200 as fx
        from fp8_expert_ffn_b200 import ep
        from fp8_expert_ffn_b200 import torch_utils as tu
        wl, layer, _ = gen.workload_inputs("toy")
        sh = layer.shape
        dev = tu.upload_layer(layer)
        x = tu.bf16_tensor(gen.make_x(T, sh.H, 500 + rank, outliers=2))
        ref = torch.empty((T, sh.H), dtype=torch.bfloat16, device="cuda")
        ws = tu.workspace(dev, T)
        fx.moe_layer_forward(dev, x, T, sh.H, ref, sh.H, ws, ws.numel())
        route, experts = ep.rank_layers(dev, rank, world)
        comm = ep.connect_peers(fx.EpComm(route, rank, world, ep.peer_capacity(T, sh.K, sh.S, world)))
        sync = HostSync(dist)
        ops = ep.PeerOps(route, experts, comm, world)
        outs = [ep.ep_forward_peer(ops, sync, x, T) for _ in range(2)]   # twice: buffers reused
        same = all(torch.equal(o.view(torch.int16), ref.view(torch.int16)) for o in outs)
        codes = [fx.moe_get_device_status(h)[0] for h in (route, experts)]
        dist.barrier()        # no rank unmaps while another still reads
        comm.close()
        q.put((rank, same, codes))
    finally:
        dist.destroy_process_group()


def test_peer_dispatch_across_processes_through_ipc():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, 256, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, same, codes in res:
        assert codes == [0, 0], (rank, codes)
        assert same, f"rank {rank} differs from the single-GPU forward"
