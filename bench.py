"""Benchmark of the FP8 MoE-layer forward (dots3-note preview shape) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode|prefill|zipf|edge|edge_f1500|...] [--no-workloads] [--ep]

One step = one whole forward of the layer (route, permute + quantise, gate/up
GEMM + SwiGLU + quantise, down GEMM, combine) over one batch of T tokens
whose inputs already sit in HBM, timed through moe_layer_forward (one call
captured in a CUDA graph, replayed once per step); a second
timed pass calls the stages one by one with CUDA events between them for the
per-stage times and the kernel rooflines. With N > 1 (torchrun, one rank per GPU) every
rank runs an independent replica of the layer on its own batch: the layer has
no exchange step on one node at this scale, so the job is weak-scaled and the
value is all ranks' tokens over the slowest rank's device time.

On one GPU the line also carries a `workloads` block: each of the seeded
workloads of the layer (decode T=64, prefill T=4096, Zipf long prefill
T=16384, edge T=4099 and its FFN=1500 variant) timed the same way, with both
roofline fractions (measured HBM copy bandwidth; dense FP8 = 2 x the measured
BF16 burst GEMM rate), its own clock sample and the C++ FP64 oracle timed on
that workload's own tokens. The toy layer is a parity case only.

With --ep the ranks run the layer expert-parallel instead (run_ep): a
separate line, not the replica measurement above.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s at T=64 and T=16384; % of HBM / dense-FP8 tensor roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FP8_OVER_BF16 = 2.0          # nominal dense FP8 / BF16 tensor throughput ratio on B200


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="decode",
                   choices=["decode", "prefill", "zipf", "edge", "edge_f1500", "decode_e64", "prefill_e32", "vision",
                            "dense"])
    p.add_argument("--no-workloads", action="store_true", help="time only --workload (no workloads block)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--ep", action="store_true",
                   help="expert parallelism over the ranks instead of replicas: the routed experts split into "
                        "equal blocks, one per rank")
    p.add_argument("--ep-transport", choices=["peer", "nccl"], default="peer",
                   help="peer: the library's dispatch/combine kernels over peer memory (CUDA IPC); nccl: "
                        "all-to-alls of the rows over torch.distributed with the regroup kernels")
    return p.parse_args()


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "gemm_traffic.json")
GEMM_SOURCE = os.path.join(ROOT, "fp8_expert_ffn_b200", "csrc", "gemm.cu")
GEMM_HOST_MARKER = "template <int MODE, int EPI>\ncudaError_t launch_gemm("


def measured_traffic(kernel: str, algorithmic_bytes: float):
    """DRAM bytes per launch from the committed ncu record (ratio of measured
    to algorithmic bytes on the profiling case), or None when the GEMM source
    has changed since the counters were taken."""
    import hashlib
    if not os.path.exists(TRAFFIC_FILE):
        return None
    rec = json.load(open(TRAFFIC_FILE))
    src = open(GEMM_SOURCE).read()
    cut = src.find(GEMM_HOST_MARKER)   # the kernel and its device helpers precede the host launch code
    sha = hashlib.sha256(src[:cut if cut >= 0 else len(src)].encode()).hexdigest()
    key = f"{kernel}_traffic_over_algorithmic"
    if sha != rec.get("kernel_source_sha256") or key not in rec:
        return None
    return round(rec[key] * algorithmic_bytes)


def peaks():
    if os.path.exists(PEAKS_FILE):
        d = json.load(open(PEAKS_FILE))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------- distributed plumbing

def dist_setup(n):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if n > 1 and world != n:
        raise SystemExit(f"--gpus {n} needs torchrun with {n} ranks (WORLD_SIZE={world})")
    return world, rank, local


class Dist:
    """One process per GPU; every rank runs its own replica of the layer. The
    only collectives are the barriers around the timed region and the
    reductions of the timing (max over ranks) and of the token count (sum)."""

    def __init__(self, world, rank, local, backend="nccl", timeout_s=600, group_always=False):
        import torch.distributed as dist
        self.world, self.rank, self.local = world, rank, local
        self.dist = dist if (world > 1 or group_always) else None
        self.device = "cuda" if backend == "nccl" else "cpu"
        if self.dist:
            from datetime import timedelta
            dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s))

    def barrier(self):
        if self.dist:
            self.dist.barrier()

    def _reduce(self, v: float, op) -> float:
        if not self.dist:
            return v
        import torch
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=op)
        return float(t.item())

    def max(self, v: float) -> float:
        return v if not self.dist else self._reduce(v, self.dist.ReduceOp.MAX)

    def sum(self, v: float) -> float:
        return v if not self.dist else self._reduce(v, self.dist.ReduceOp.SUM)

    def close(self):
        if self.dist:
            self.dist.destroy_process_group()


def job_throughput(d: "Dist", tokens_this_rank: float, ms_this_rank: float):
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    ms = d.max(ms_this_rank)
    tokens = d.sum(tokens_this_rank)
    return tokens / (ms / 1e3), ms, tokens


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons while running."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        self.proc.wait()
        rows = []
        for line in open(self.path):
            parts = [s.strip() for s in line.split(",")]
            if len(parts) == 8:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- workload

def algorithmic_work(layer, T, offsets):
    """Bytes and FLOPs of one forward, counted from the problem (not from the
    kernels): weights of the touched experts read once, activations and
    outputs once; FLOPs of the expert GEMMs only (2 * rows * N * K)."""
    sh = layer.shape
    H, F, E, K = sh.H, sh.F, sh.E, sh.K
    rows = T * (K + sh.S)
    counts = np.diff(offsets)
    touched = int(np.count_nonzero(counts[:E])) + (1 if counts[E] > 0 else 0)
    gu_w = 2 * F * H + 2 * sh.FB * sh.HB * 4          # gate + up codes and scales of one expert
    dn_w = H * F + sh.HB * sh.FB * 4                  # down codes and scales
    gu_bytes = touched * gu_w + rows * (H + 4 * sh.HB) + rows * (sh.FB * 128 + 4 * sh.FB)
    dn_bytes = touched * dn_w + rows * (sh.FB * 128 + 4 * sh.FB) + rows * H * 2
    route_bytes = E * H * 4 + T * H * 2 + T * K * 8
    permute_bytes = T * H * 2 + rows * (H + 4 * sh.HB) + T * K * 8 + rows * 4
    combine_bytes = rows * H * 2 + T * H * 2 + T * K * 8
    gu_flops = 2.0 * rows * (2 * F) * H
    dn_flops = 2.0 * rows * H * F
    return {"touched_groups": touched, "rows": rows,
            "bytes": {"route": route_bytes, "permute": permute_bytes, "gate_up": gu_bytes, "down": dn_bytes,
                      "combine": combine_bytes},
            "flops": {"gate_up": gu_flops, "down": dn_flops}}


_device_layers: dict = {}


def load_layer(name, d, rank):
    """Host inputs on every rank; with several ranks rank 0 generates the
    expert weights and broadcasts them over NCCL (same checkpoint everywhere).
    On one rank, workloads of the same layer (shape and weight seed) share
    the host and device copies of its experts; only the router differs."""
    import gen
    import torch
    from fp8_expert_ffn_b200 import torch_utils as tu
    import fp8_expert_ffn_b200 as fx
    wl = gen.WORKLOADS[name]
    sh = wl.shape
    if d.world == 1:
        wl, host, x = gen.workload_inputs(name)
        key = (sh, wl.w_seed)
        prev = _device_layers.get(key)
        dev = tu.upload_layer(host, share_experts=prev)
        if prev is None:
            for k in list(_device_layers):      # keep one layer's experts on the device at a time
                del _device_layers[k]
            torch.cuda.empty_cache()
            _device_layers[key] = dev
        return wl, host, dev, x
    x = gen.make_x(wl.T, sh.H, wl.x_seed + 1000 * rank, wl.outliers, wl.zipf)
    host = gen.make_layer(sh, wl.w_seed, zipf=wl.zipf) if rank == 0 else None
    shapes = {"w_gate": ((sh.E + sh.S, sh.F, sh.H), torch.uint8), "w_up": ((sh.E + sh.S, sh.F, sh.H), torch.uint8),
              "w_down": ((sh.E + sh.S, sh.H, sh.ld_f), torch.uint8),
              "s_gate": ((sh.E + sh.S, sh.FB, sh.HB), torch.float32), "s_up": ((sh.E + sh.S, sh.FB, sh.HB), torch.float32),
              "s_down": ((sh.E + sh.S, sh.HB, sh.FB), torch.float32), "router_w": ((sh.E, sh.H), torch.float32)}
    tens = {}
    for k, (shape, dt) in shapes.items():
        tens[k] = tu.to_device(getattr(host, k)) if rank == 0 else torch.empty(shape, dtype=dt, device="cuda")
        d.dist.broadcast(tens[k], 0)
    w = fx.LayerWeights(**tens)
    dev = fx.MoeLayer(sh.H, sh.E, sh.K, sh.F, w, ld_h=sh.H, ld_f=sh.ld_f, n_shared=sh.S)
    return wl, host, dev, x


class Stages:
    """Buffers and the per-stage calls of one forward (the same kernels that
    moe_layer_forward launches, with CUDA events between the stages)."""
    NAMES = ("route", "permute", "gate_up", "down", "combine")

    def __init__(self, dev, sh, T, x):
        import torch
        import fp8_expert_ffn_b200 as fx
        from fp8_expert_ffn_b200 import torch_utils as tu
        self.fx, self.dev, self.sh, self.T, self.x = fx, dev, sh, T, x
        K, E, H = sh.K, sh.E, sh.H
        rows = T * (K + sh.S)
        c = "cuda"
        self.ws = tu.workspace(dev, T)
        self.idx = torch.empty((T, K), dtype=torch.int32, device=c)
        self.w = torch.empty((T, K), dtype=torch.float32, device=c)
        self.offsets = torch.empty(E + 2, dtype=torch.int32, device=c)
        self.perm = torch.empty(rows, dtype=torch.int32, device=c)
        self.inv = torch.empty((T, K), dtype=torch.int32, device=c)
        self.xq = torch.empty((rows, H), dtype=torch.uint8, device=c)
        self.xs = torch.empty((sh.HB, rows), dtype=torch.float32, device=c)
        self.h = torch.empty((rows, sh.FB * 128), dtype=torch.uint8, device=c)
        self.hs = torch.empty((sh.FB, rows), dtype=torch.float32, device=c)
        self.y = torch.empty((rows, H), dtype=torch.bfloat16, device=c)
        self.out = torch.empty((T, H), dtype=torch.bfloat16, device=c)

    def step(self, ev=None):
        fx, d, T, H, nb = self.fx, self.dev, self.T, self.sh.H, self.ws.numel()
        if ev: ev[0].record()
        fx.moe_route(d, self.x, T, H, self.idx, self.w, None, self.ws, nb)
        if ev: ev[1].record()
        fx.moe_permute(d, self.x, T, H, self.idx, self.offsets, self.perm, self.inv, self.xq, self.xs, self.ws, nb)
        if ev: ev[2].record()
        fx.moe_gate_up(d, self.xq, self.xs, self.offsets, T, self.h, self.hs)
        if ev: ev[3].record()
        fx.moe_down(d, self.h, self.hs, self.offsets, T, self.y)
        if ev: ev[4].record()
        fx.moe_combine(d, self.y, self.inv, self.w, T, self.out, H)
        if ev: ev[5].record()


def time_stages(st: Stages, steps: int, warmup: int, d: Dist, sampler=None):
    import torch
    for _ in range(warmup):
        st.step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    d.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(steps):
        st.step(evs[i])
    t1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    d.barrier()
    torch.cuda.synchronize()
    total_ms = t0.elapsed_time(t1)
    per = {n: sum(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(steps)) / steps
           for j, n in enumerate(Stages.NAMES)}
    code, bits = st.fx.moe_get_device_status(st.dev)
    if code != 0:
        raise RuntimeError(f"device status {bits:#x}")
    return total_ms, per, clocks


def time_forward(st: Stages, steps: int, warmup: int, d: Dist, sampler=None):
    """The whole forward as a serving loop runs it: one moe_layer_forward
    captured once in a CUDA graph (its kernels chained by programmatic
    dependent launch, no event between them) and replayed once per step,
    CUDA events on the launching stream around the timed steps. The
    per-stage breakdown comes from time_stages, whose events between the
    stages break that chaining."""
    import torch
    fx, dev, T, H = st.fx, st.dev, st.T, st.sh.H

    def fwd():
        fx.moe_layer_forward(dev, st.x, T, H, st.out, H, st.ws, st.ws.numel())

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fwd()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fwd()
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    d.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        graph.replay()
    b.record()
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    d.barrier()
    torch.cuda.synchronize()
    del graph
    code, bits = fx.moe_get_device_status(dev)
    if code != 0:
        raise RuntimeError(f"device status {bits:#x}")
    return a.elapsed_time(b), clocks


def time_e2e(dev, sh, x_bits, steps, warmup, d: Dist):
    """Through moe_layer_forward with host buffers, pipelined the way a serving
    loop runs it: step i's input is copied from pinned host memory to the
    device, and step i's output back, on a copy stream, while the forwards
    run in order on the compute stream (double-buffered device input and
    output). Every step's two copies are inside the timed region, which runs
    from before the first upload to after the last download."""
    import torch
    import fp8_expert_ffn_b200 as fx
    from fp8_expert_ffn_b200 import torch_utils as tu
    T, H = x_bits.shape
    x_host = torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).view(torch.bfloat16).pin_memory()
    out_host = [torch.empty((T, H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_dev = [torch.empty((T, H), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    out_dev = [torch.empty((T, H), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    ws = tu.workspace(dev, T)
    comp, copy = torch.cuda.current_stream(), torch.cuda.Stream()
    h2d = [torch.cuda.Event() for _ in range(2)]
    fwd = [torch.cuda.Event() for _ in range(2)]
    d2h = [torch.cuda.Event() for _ in range(2)]

    def run(n, start=None, end=None):
        with torch.cuda.stream(copy):
            if start is not None:
                start.record(copy)
            x_dev[0].copy_(x_host, non_blocking=True)
            h2d[0].record(copy)
        for i in range(n):
            b = i & 1
            comp.wait_event(h2d[b])
            if i >= 2:
                comp.wait_event(d2h[b])          # out_dev[b]'s previous download is done
            fx.moe_layer_forward(dev, x_dev[b], T, H, out_dev[b], H, ws, ws.numel(), stream=comp)
            fwd[b].record(comp)
            with torch.cuda.stream(copy):
                if i + 1 < n:                   # next step's upload, overlapping this forward
                    if i >= 1:
                        copy.wait_event(fwd[1 - b])   # x_dev[1-b] was read by the previous forward
                    x_dev[1 - b].copy_(x_host, non_blocking=True)
                    h2d[1 - b].record(copy)
                copy.wait_event(fwd[b])
                out_host[b].copy_(out_dev[b], non_blocking=True)
                d2h[b].record(copy)
        if end is not None:
            end.record(copy)

    run(warmup)
    torch.cuda.synchronize()
    d.barrier()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(steps, a, b)
    torch.cuda.synchronize()
    d.barrier()
    pipelined = a.elapsed_time(b)
    # the same steps one after another on one stream (upload, forward,
    # download): what the copies cost when nothing hides them
    torch.cuda.synchronize()
    a.record(comp)
    for _ in range(steps):
        x_dev[0].copy_(x_host, non_blocking=True)
        fx.moe_layer_forward(dev, x_dev[0], T, H, out_dev[0], H, ws, ws.numel(), stream=comp)
        out_host[0].copy_(out_dev[0], non_blocking=True)
    b.record(comp)
    torch.cuda.synchronize()
    d.barrier()
    return pipelined, a.elapsed_time(b), T * H * 2, T * H * 2


ORACLE_TOKENS = 64     # tokens of one oracle sample (the whole decode batch)


def oracle_sample(host_layer, x_bits, first: int = 0):
    """One sample for the CPU baseline: the C++ FP64 oracle (plain loops,
    all host cores) through the whole layer -- route, permute, quantise,
    expert FFNs, combine -- on ORACLE_TOKENS consecutive tokens of the
    workload starting at `first` (wrapping). Returns (tokens, seconds)."""
    from oracle import cpp
    T = x_bits.shape[0]
    n = min(T, ORACLE_TOKENS)
    tok = (first + np.arange(n)) % T
    t = time.perf_counter()
    cpp.layer_forward(np.ascontiguousarray(x_bits[tok]), host_layer)
    return n, time.perf_counter() - t


def cpu_baseline(host_layer, x_bits, budget_s=10.0):
    """The oracle as it stands, timed on this host's cores: samples of
    oracle_sample until about budget_s seconds have passed."""
    from oracle import cpp
    tokens, secs, i = 0, 0.0, 0
    while secs < budget_s:
        n, dt = oracle_sample(host_layer, x_bits, first=i * ORACLE_TOKENS)
        tokens, secs, i = tokens + n, secs + dt, i + 1
    return {"value": round(tokens / secs, 3), "unit": "tokens/s", "cores": cpp.threads(), "kind": "oracle",
            "sample": f"C++ FP64 oracle, {i} x {min(x_bits.shape[0], ORACLE_TOKENS)} consecutive tokens of the "
                      f"workload through the whole layer (route, permute, quantise, expert FFNs, combine), "
                      f"{secs:.1f} s"}


def fractions(work, per, total_ms, pk):
    """Both roofline fractions of each GEMM and of the whole step: HBM
    (algorithmic bytes / time / measured copy bandwidth) and dense FP8
    (algorithmic FLOPs / time / (2 x measured BF16 burst rate); the sustained
    BF16 figure gives the sustained fraction beside it)."""
    fp8 = FP8_OVER_BF16 * pk["bf16_tflops"]
    fp8_sus = FP8_OVER_BF16 * pk["bf16_tflops_sustained"]
    out = {}
    step_bytes = sum(work["bytes"].values())
    step_flops = sum(work["flops"].values())
    for k, b, f, ms in (("gate_up", work["bytes"]["gate_up"], work["flops"]["gate_up"], per["gate_up"]),
                        ("down", work["bytes"]["down"], work["flops"]["down"], per["down"]),
                        ("step", step_bytes, step_flops, total_ms)):
        gbs = b / (ms / 1e3) / 1e9
        tfs = f / (ms / 1e3) / 1e12
        out[k] = {"ms": round(ms, 5), "hbm_gbs": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm_gbs"], 4),
                  "tflops": round(tfs, 1), "frac_fp8": round(tfs / fp8, 4), "frac_fp8_sustained": round(tfs / fp8_sus, 4)}
    ridge = fp8 * 1e12 / (pk["hbm_gbs"] * 1e9)
    out["binding"] = "hbm" if work["flops"]["gate_up"] / work["bytes"]["gate_up"] < ridge else "tensor"
    return out


def count_near_ties(st: Stages) -> int:
    """Tokens whose K-th and (K+1)-th routing probabilities (softmax of the
    library's FP32 logits, taken in FP64) are less than 1e-6 apart: the
    tokens whose choice of experts rounding may decide."""
    import torch
    sh, T = st.sh, st.T
    if sh.K >= sh.E:
        return 0
    logits = torch.empty((T, sh.E), dtype=torch.float32, device="cuda")
    st.fx.moe_route(st.dev, st.x, T, sh.H, st.idx, st.w, logits, st.ws, st.ws.numel())
    p = torch.softmax(logits.double(), dim=1)
    top = torch.topk(p, sh.K + 1, dim=1).values
    return int((top[:, sh.K - 1] - top[:, sh.K] < 1e-6).sum().item())


def measure_workload(name, d, rank, args, pk, sampler, oracle=True):
    """One workload: its stages timed over the same number of steps as the
    headline (at least 10; a timed region of 0.01-0.15 s, like the burst
    GEMM measurement behind the FP8 peak), with its own clock sample and the
    oracle on its own tokens."""
    from fp8_expert_ffn_b200 import torch_utils as tu
    wl, host, dev, x_bits = load_layer(name, d, rank)
    st = Stages(dev, wl.shape, wl.T, tu.bf16_tensor(x_bits))
    steps = max(10, args.steps)
    warm = max(3, min(args.warmup, 5))
    total_ms, clocks = time_forward(st, steps, warm, d, sampler)
    total_ms = d.max(total_ms)
    _, per, _ = time_stages(st, steps, warm, d)
    off = st.offsets.cpu().numpy()
    work = algorithmic_work(wl, wl.T, off)
    counts = np.diff(off)[:wl.shape.E]
    near_ties = count_near_ties(st)
    entry = {"workload": f"{wl.name}: {wl.note}", "T": wl.T, "steps": steps,
             "tokens_per_s": round(d.sum(float(wl.T * steps)) / (total_ms / 1e3), 1),
             "ms_per_step": round(total_ms / steps, 5), "stage_ms": {k: round(v, 5) for k, v in per.items()},
             "roofline": fractions(work, per, total_ms / steps, pk), "clocks": clocks,
             "touched_groups": work["touched_groups"],
             "load_max_over_mean": round(float(counts.max() / max(counts.mean(), 1e-9)), 2),
             "empty_experts": int((counts == 0).sum()), "near_tie_tokens": near_ties}
    if oracle and rank == 0:
        n, dt = oracle_sample(host, x_bits)
        entry["oracle"] = {"tokens_per_s": round(n / dt, 3), "tokens": n, "seconds": round(dt, 2),
                           "kind": "C++ FP64 oracle on this workload's first tokens, whole layer"}
    del st
    return entry


WORKLOADS = ("decode", "prefill", "zipf", "edge", "edge_f1500")


# ----------------------------------------------------------------------------- arms

def workload_config(wl, world, touched):
    """The config block of a line (the same in both arms)."""
    sh = wl.shape
    return {"workload": f"{wl.name}: {wl.note}", "T": wl.T, "hidden": sh.H, "experts": f"{sh.E}+{sh.S}",
            "top_k": sh.K, "ffn": sh.F, "weights": "FP8 E4M3, 128x128 fp32 block scales, seeded synthetic",
            "l2": "inputs larger than L2 (each step streams the touched experts' weights, GBs >> 126 MB)",
            "parallelism": f"replicas x{world}", "touched_groups": int(touched)}


def run_ours(args):
    import torch
    world, rank, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    d = Dist(world, rank, local)
    pk = peaks()
    wl, host, dev, x_bits = load_layer(args.workload, d, rank)
    from fp8_expert_ffn_b200 import torch_utils as tu
    sh = wl.shape
    T = wl.T
    x = tu.bf16_tensor(x_bits)
    st = Stages(dev, sh, T, x)
    visible = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    sampler = ClockSampler(visible.split(",")[local] if visible else local)
    total_ms, clocks = time_forward(st, args.steps, args.warmup, d, sampler)
    value, total_ms, tokens = job_throughput(d, float(T * args.steps), total_ms)
    _, per, _ = time_stages(st, args.steps, args.warmup, d)
    off = st.offsets.cpu().numpy()
    work = algorithmic_work(wl, T, off)
    # the dominant kernel: decode-sized batches are bound by streaming the
    # gate/up weights (HBM); large batches by the FP8 tensor pipe
    kern = max(("gate_up", "down"), key=lambda k: per[k])
    kern_ms = d.max(per[kern])
    fp8 = FP8_OVER_BF16 * pk["bf16_tflops"]
    hbm_bound = work["flops"][kern] / work["bytes"][kern] < (fp8 * 1e12) / (pk["hbm_gbs"] * 1e9)
    # both fractions of the dominant kernel; the non-binding one is reported
    # beside the roofline (it matters for mid-size batches such as T = 4096)
    hbm_frac = work["bytes"][kern] / (kern_ms / 1e3) / 1e9 / pk["hbm_gbs"]
    tensor_frac = work["flops"][kern] / (kern_ms / 1e3) / 1e12 / fp8
    other = {"bound": "tensor", "frac": round(tensor_frac, 4)} if hbm_bound else {"bound": "hbm",
                                                                                 "frac": round(hbm_frac, 4)}
    if hbm_bound:
        ach = work["bytes"][kern] / (kern_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "kernel": kern, "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / pk["hbm_gbs"], 4), "traffic": measured_traffic(kern, work["bytes"][kern]),
                "algorithmic_bytes_per_launch": work["bytes"][kern], "ms_per_launch": round(kern_ms, 5),
                "peak_source": f"{pk['source']} hbm_gbs"}
    else:
        ach = work["flops"][kern] / (kern_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "kernel": kern, "achieved": round(ach, 1), "peak": round(fp8, 1),
                "unit": "TFLOP/s", "frac": round(ach / fp8, 4), "traffic": None,
                "algorithmic_flops_per_launch": work["flops"][kern], "ms_per_launch": round(kern_ms, 5),
                "peak_source": f"{pk['source']} bf16_tflops (burst) x {FP8_OVER_BF16} (nominal FP8/BF16 ratio)",
                "frac_of_sustained": round(ach / (FP8_OVER_BF16 * pk["bf16_tflops_sustained"]), 4)}
    roof["other_bound"] = other
    e2e_ms, serial_ms, bi, bo = time_e2e(dev, sh, x_bits, args.steps, args.warmup, d)
    e2e_ms, serial_ms = d.max(e2e_ms), d.max(serial_ms)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 (fp32 accumulate)", "data": "synthetic",
        "config": workload_config(wl, world, work["touched_groups"]),
        "stage_ms": {k: round(v, 5) for k, v in per.items()},
        "roofline": roof,
        "e2e": {"value": round(tokens / (e2e_ms / 1e3), 1), "unit": "tokens/s", "h2d_bytes_per_step": bi,
                "d2h_bytes_per_step": bo, "ms_per_step": round(e2e_ms / args.steps, 5),
                "serial": {"value": round(tokens / (serial_ms / 1e3), 1),
                           "ms_per_step": round(serial_ms / args.steps, 5),
                           "how": "upload, forward, download one after another on one stream"}},
        # the library's own count for one forward (route 2, permute 2 or 4,
        # gate/up 1, down 1 or 2, combine 1)
        "gpu_launches": st.fx.moe_kernels_per_forward(dev, T) * args.steps,
        "launch": "one moe_layer_forward captured in a CUDA graph, replayed once per step",
        "clocks": clocks,
    }
    del st
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(host, x_bits)
    if world == 1 and not args.no_workloads:
        wls = {}
        for name in WORKLOADS:
            wls[name] = measure_workload(name, d, rank, args, pk, ClockSampler(sampler.gpu),
                                         oracle=not args.no_cpu_baseline)
        wls["toy"] = {"workload": "toy: T=32, hidden 512, 16+1 experts, top-4, FFN 256",
                      "purpose": "parity only (every value checked against the oracle), not timed"}
        line["workloads"] = wls
        wl_d, _, dev_d, xb_d = load_layer("decode", d, rank)
        line["expert_parallel_one_rank"] = measure_ep_one_rank(dev_d, wl_d.shape, wl_d.T, tu.bf16_tensor(xb_d),
                                                               max(10, args.steps), max(3, min(args.warmup, 5)), d)
        # the serving recipe's shape: 8 ranks of 128 tokens, emulated on this GPU
        line["expert_parallel_8_emulated"] = measure_ep_emulated(dev_d, wl_d.shape, wl_d, 8, 128,
                                                                 max(10, args.steps), 3)
        line["peaks"] = {"hbm_gbs": pk["hbm_gbs"], "fp8_tflops_burst": round(fp8, 1),
                         "fp8_tflops_sustained": round(FP8_OVER_BF16 * pk["bf16_tflops_sustained"], 1),
                         "source": f"{pk['source']}: HBM copy; FP8 = {FP8_OVER_BF16} x BF16 GEMM (nominal ratio)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    d.close()


def run_ep(args):
    """--ep: one expert-parallel forward per step on every rank (its own T
    tokens of the workload): route against all E experts, dispatch the FP8
    rows to the ranks that own their experts, grouped GEMMs over the rank's
    E/P experts plus the shared expert, return the rows, combine. With the
    peer transport (default; ep.ep_forward_peer) the library's kernels store
    and load the rows in the owners' memory and NCCL carries only the
    offsets and two barriers; with nccl (ep.ep_forward) the rows cross in
    torch.distributed all-to-alls. A one-rank group when run alone. Timed like the
    replica arm (CUDA events on the compute stream, barriers on both sides,
    max over ranks); the orchestration's two host reads of the counts are
    inside the timed region. Each rank's output is checked bit for bit
    against the single-GPU forward of the whole layer on the same tokens, and
    that forward's own time is reported beside it."""
    import torch
    from fp8_expert_ffn_b200 import ep
    from fp8_expert_ffn_b200 import torch_utils as tu
    import fp8_expert_ffn_b200 as fx
    world, rank, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    if world == 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", str(_free_port()))
        os.environ.setdefault("RANK", "0")
        os.environ.setdefault("WORLD_SIZE", "1")
    d = Dist(world, rank, local, group_always=True)
    wl, host, dev, x_bits = load_layer(args.workload, d, rank)
    sh, T = wl.shape, wl.T
    x = tu.bf16_tensor(x_bits)
    # the single-GPU forward of the whole layer: the parity reference and the
    # time the expert-parallel step is compared with
    ref = torch.empty((T, sh.H), dtype=torch.bfloat16, device="cuda")
    ws = tu.workspace(dev, T)
    fwd = lambda: fx.moe_layer_forward(dev, x, T, sh.H, ref, sh.H, ws, ws.numel())
    for _ in range(args.warmup):
        fwd()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        fwd()
    b.record()
    torch.cuda.synchronize()
    single_ms = d.max(a.elapsed_time(b)) / args.steps
    route, experts = ep.rank_layers(dev, rank, world)
    comm = None
    if args.ep_transport == "peer":
        comm = ep.connect_peers(fx.EpComm(route, rank, world, ep.peer_capacity(T, sh.K, sh.S, world)))
        ops, ex = ep.PeerOps(route, experts, comm, world), ep.TorchSync()
        step = lambda: ep.ep_forward_peer(ops, ex, x, T)
    else:
        ops, ex = ep.CudaOps(route, experts, world), ep.TorchExchange()
        step = lambda: ep.ep_forward(ops, ex, x, T)
    for _ in range(args.warmup):
        out = step()
    torch.cuda.synchronize()
    visible = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    sampler = ClockSampler(visible.split(",")[local] if visible else local)
    d.barrier()
    torch.cuda.synchronize()
    sampler.start()
    a.record()
    for _ in range(args.steps):
        out = step()
    b.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    d.barrier()
    torch.cuda.synchronize()
    value, total_ms, tokens = job_throughput(d, float(T * args.steps), a.elapsed_time(b))
    same = d.sum(0.0 if torch.equal(out.view(torch.int16), ref.view(torch.int16)) else 1.0)
    for h in (route, experts, dev):
        code, bits = fx.moe_get_device_status(h)
        if code != fx.MOE_OK:
            raise RuntimeError(f"device status {bits:#x}")
    if same != 0:
        raise RuntimeError(f"{int(same)} rank(s) differ from the single-GPU forward")
    stages = ep_peer_stages(ops, ex, x, T, args.steps, d, sh, world) if comm is not None else None
    line = {
        "metric": "expert-parallel MoE-layer tokens/s", "value": round(value, 1), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 (fp32 accumulate)",
        "data": "synthetic",
        "config": {"workload": f"{wl.name}: {wl.note}", "T_per_rank": T, "hidden": sh.H,
                   "experts": f"{sh.E}+{sh.S}", "experts_per_rank": sh.E // world, "top_k": sh.K, "ffn": sh.F,
                   "parallelism": f"ep{world}",
                   "exchange": ("dispatch/combine kernels over peer memory (CUDA IPC); NCCL all-gather of the "
                                "offsets and two barriers" if comm else
                                "torch.distributed all_to_all_single (NCCL) + regroup kernels")},
        "parity": "every rank's output bit-identical to the single-GPU forward of the whole layer",
        "single_gpu_forward_ms_per_step": round(single_ms, 5),
        "clocks": clocks,
    }
    if stages:
        line["stages"] = stages
    if rank == 0:
        print(json.dumps(line), flush=True)
    d.barrier()
    torch.cuda.synchronize()
    if comm is not None:
        comm.close()          # every rank is past its last read of the peers' buffers
    del ops, route, experts
    d.close()


class OneRankSync:
    """The peer-memory forward's collectives for a single rank: the
    all-gather is the rank's own offsets and there is nothing to wait for."""

    def all_gather(self, off):
        return off.unsqueeze(0)

    def barrier(self):
        pass


def measure_ep_one_rank(dev, sh, T, x, steps, warmup, d: Dist):
    """The expert-parallel forward over peer memory with one rank (every
    expert local, the exchange buffer its own): what its kernels cost over
    the fused forward, with the per-phase breakdown. Checked bit for bit
    against the fused forward."""
    import torch
    import fp8_expert_ffn_b200 as fx
    from fp8_expert_ffn_b200 import ep
    from fp8_expert_ffn_b200 import torch_utils as tu
    ref = torch.empty((T, sh.H), dtype=torch.bfloat16, device="cuda")
    ws = tu.workspace(dev, T)
    fx.moe_layer_forward(dev, x, T, sh.H, ref, sh.H, ws, ws.numel())
    route, experts = ep.rank_layers(dev, 0, 1)
    comm = fx.EpComm(route, 0, 1, ep.peer_capacity(T, sh.K, sh.S, 1))
    ops, sync = ep.PeerOps(route, experts, comm, 1), OneRankSync()
    for _ in range(warmup):
        out = ep.ep_forward_peer(ops, sync, x, T)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        out = ep.ep_forward_peer(ops, sync, x, T)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    same = torch.equal(out.view(torch.int16), ref.view(torch.int16))
    stages = ep_peer_stages(ops, sync, x, T, steps, d, sh, 1)
    for h in (route, experts):
        code, bits = fx.moe_get_device_status(h)
        if code != fx.MOE_OK:
            raise RuntimeError(f"device status {bits:#x}")
    if not same:
        raise RuntimeError("expert-parallel forward differs from the fused forward")
    comm.close()
    return {"ranks": 1, "transport": "dispatch/combine kernels over peer memory (one rank: its own buffer)",
            "ms_per_step": round(ms, 5), "tokens_per_s": round(T / (ms / 1e3), 1), "stages": stages,
            "parity": "bit-identical to the fused forward"}


def measure_ep_emulated(dev, sh, wl, ranks: int, T: int, steps: int, warmup: int):
    """The expert-parallel forward over peer memory with `ranks` ranks
    emulated on this one GPU (each rank's buffers in this GPU's memory, its
    tokens its own seeded batch): every phase runs for all ranks in turn on
    one stream, which orders the phases as the barriers would. Reports the
    time of one forward of all ranks, each phase summed over the ranks, and
    the owners' grouped-GEMM phase per rank against the weights it streams
    (its E/ranks experts plus the shared one). Each rank's output is checked
    bit for bit against the fused forward of the whole layer on its tokens.
    No NVLink is involved, so the exchange is not what this measures."""
    import torch
    import gen
    import fp8_expert_ffn_b200 as fx
    from fp8_expert_ffn_b200 import ep
    from fp8_expert_ffn_b200 import torch_utils as tu
    layers = [ep.rank_layers(dev, r, ranks) for r in range(ranks)]
    cap = ep.peer_capacity(T, sh.K, sh.S, ranks)
    comms = [fx.EpComm(layers[r][0], r, ranks, cap) for r in range(ranks)]
    fx.EpComm.connect_local(comms)
    ops = [ep.PeerOps(layers[r][0], layers[r][1], comms[r], ranks) for r in range(ranks)]
    xs = [tu.bf16_tensor(gen.make_x(T, sh.H, 5000 + r, wl.outliers, wl.zipf)) for r in range(ranks)]

    def forward(ev=None):
        plans = [ops[r].plan(xs[r], T) for r in range(ranks)]
        if ev: ev[0].record()
        all_off = torch.stack([off for _, off in plans])
        for r in range(ranks):
            ops[r].dispatch(plans[r][0], all_off, T)
        if ev: ev[1].record()
        for r in range(ranks):
            ops[r].experts(plans[r][0])
        if ev: ev[2].record()
        return [ops[r].combine(plans[r][0], T) for r in range(ranks)]

    for _ in range(warmup):
        outs = forward()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        outs = forward()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for i in range(steps):
        evs[i][3].record()
        forward(evs[i][:3])
    torch.cuda.synchronize()
    ph = {"route_plan": sum(evs[i][3].elapsed_time(evs[i][0]) for i in range(steps)) / steps,
          "dispatch": sum(evs[i][0].elapsed_time(evs[i][1]) for i in range(steps)) / steps,
          "experts": sum(evs[i][1].elapsed_time(evs[i][2]) for i in range(steps)) / steps}
    ws = tu.workspace(dev, T)
    ref = torch.empty((T, sh.H), dtype=torch.bfloat16, device="cuda")
    same = True
    for r in range(ranks):
        fx.moe_layer_forward(dev, xs[r], T, sh.H, ref, sh.H, ws, ws.numel())
        same &= torch.equal(outs[r].view(torch.int16), ref.view(torch.int16))
    for lr in layers:
        for h in lr:
            code, bits = fx.moe_get_device_status(h)
            if code != fx.MOE_OK:
                raise RuntimeError(f"device status {bits:#x}")
    if not same:
        raise RuntimeError("an emulated rank differs from the fused forward")
    for c in comms:
        c.close()
    El = sh.E // ranks
    owner_bytes = (El + sh.S) * (3 * sh.F * sh.H + 3 * sh.FB * sh.HB * 4)
    per_owner_ms = ph["experts"] / ranks
    return {"ranks": ranks, "tokens_per_rank": T, "transport": "dispatch/combine kernels over peer memory, ranks "
            "emulated on one GPU (their buffers in its memory)", "ms_per_forward_all_ranks": round(ms, 5),
            "phase_ms_all_ranks": {k: round(v, 5) for k, v in ph.items()},
            "owner_grouped_gemms_ms_per_rank": round(per_owner_ms, 5),
            "owner_weight_bytes_per_rank": owner_bytes,
            "owner_weight_stream_frac_hbm": round(owner_bytes / (per_owner_ms / 1e3) / 1e9 / peaks()["hbm_gbs"], 4),
            "parity": "every rank bit-identical to the fused forward on its tokens"}


EP_STAGES = ("route_plan", "all_gather", "dispatch", "barrier_1", "experts", "barrier_2", "combine")


def ep_peer_stages(ops, sync, x, T, steps, d: Dist, sh, world):
    """The peer-memory forward again with CUDA events between its phases
    (max over ranks of each phase's mean), and the dispatch and combine
    kernels' bytes over their times: the dispatch reads x and writes every
    token's K+S quantised rows with their scales (to the owners: over
    NVLink for the rows of other ranks), the combine reads the K+S output
    rows of every token and writes one; on one rank all of it is HBM
    traffic, so their fraction of the measured HBM copy is given then."""
    import torch
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(EP_STAGES) + 1)] for _ in range(steps)]
    d.barrier()
    torch.cuda.synchronize()
    for i in range(steps):
        e = evs[i]
        e[0].record()
        st, off = ops.plan(x, T)
        e[1].record()
        all_off = sync.all_gather(off)
        e[2].record()
        ops.dispatch(st, all_off, T)
        e[3].record()
        sync.barrier()
        e[4].record()
        ops.experts(st)
        e[5].record()
        sync.barrier()
        e[6].record()
        ops.combine(st, T)
        e[7].record()
    torch.cuda.synchronize()
    d.barrier()
    ms = {n: d.max(sum(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(steps)) / steps)
          for j, n in enumerate(EP_STAGES)}
    rows = T * (sh.K + sh.S)
    disp_bytes = T * sh.H * 2 + rows * (sh.H + 4 * sh.HB) + T * sh.K * 8
    comb_bytes = rows * sh.H * 2 + T * sh.H * 2 + T * sh.K * 12
    out = {"ms": {k: round(v, 5) for k, v in ms.items()},
           "dispatch_gbs": round(disp_bytes / (ms["dispatch"] / 1e3) / 1e9, 1),
           "combine_gbs": round(comb_bytes / (ms["combine"] / 1e3) / 1e9, 1),
           "bytes": {"dispatch": disp_bytes, "combine": comb_bytes}}
    if world == 1:
        hbm = peaks()["hbm_gbs"]
        out["dispatch_frac_hbm"] = round(out["dispatch_gbs"] / hbm, 4)
        out["combine_frac_hbm"] = round(out["combine_gbs"] / hbm, 4)
    return out


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def run_reference(args):
    """The C++ FP64 oracle timed on this host's cores as the reference arm
    (rank 0 only): each step is one oracle_sample of the workload (the same
    sampling rule as the cpu_baseline of the other arm)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import gen
    from oracle import cpp
    from oracle import moe
    wl, host, x_bits = gen.workload_inputs(args.workload)
    cpp.build()
    # the groups the whole batch touches (routed experts chosen by the
    # oracle's router, plus the shared expert), as in the other arm's config
    touched = len(np.unique(moe.route_layer(x_bits, host).idx)) + wl.shape.S
    for i in range(args.warmup):
        oracle_sample(host, x_bits, first=i * ORACLE_TOKENS)
    tokens, secs = 0, 0.0
    for i in range(args.steps):
        n, dt = oracle_sample(host, x_bits, first=(args.warmup + i) * ORACLE_TOKENS)
        tokens, secs = tokens + n, secs + dt
    value = tokens / secs
    n1 = min(wl.T, ORACLE_TOKENS)
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, world, touched),
            "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "kind": "oracle", "cores": cpp.threads(),
                             "sample": f"C++ FP64 oracle, {n1} consecutive tokens of the workload per step "
                                       f"through the whole layer"},
            "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.ep:
        run_ep(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
