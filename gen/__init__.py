"""Seeded synthetic inputs for the FP8 MoE-layer forward (shared by the CUDA
path's tests and bench and by the CPU oracle).

Holds no arithmetic of the layer's forward pass: it draws Gaussian
activations and weights with a counter-based generator (Philox4x32-10) and
writes the weights out as a fine-grained FP8 checkpoint (E4M3 codes plus one
fp32 scale per 128 x 128 block), the storage format that the model card of
dots-studio/dots3-note-prev ("Model Overview": BF16 and FP8 precision) and
transformers PR #47844 ("What does this PR do?": E4M3 weights, 128 x 128
weight blocks) describe. Real checkpoints are not used.

Layer shapes follow the Dots3NoteTextConfig defaults of the transformers docs
page "Dots 3 Note Preview" (hidden_size 5120, n_routed_experts 256,
n_shared_experts 1, num_experts_per_tok 8, moe_intermediate_size 1536).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moegen.cpp")
_LIB = os.path.join(_HERE, "libmoegen.so")

# Streams separate the kinds of tensors drawn from one seed.
STREAM_X = 1
STREAM_ROUTER = 2
STREAM_GATE = 3
STREAM_UP = 4
STREAM_DOWN = 5
STREAM_OUTLIER = 6
STREAM_ZIPF = 7


def build(force: bool = False) -> str:
    """Compile libmoegen.so in-tree (g++, a second or two)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-o", tmp, _SRC, "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        L.moegen_philox4x32_10.argtypes = [ctypes.c_void_p] * 3
        L.moegen_normal_f32.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_float,
                                        ctypes.c_void_p, ctypes.c_int]
        L.moegen_u32.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_void_p]
        L.moegen_e4m3_encode.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_void_p]
        L.moegen_fp8_blocks.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        L.moegen_fp8_blocks.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags.c_contiguous
    return a.ctypes.data


def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.asarray(ctr, dtype=np.uint32).copy()
    k = np.asarray(key, dtype=np.uint32).copy()
    out = np.zeros(4, np.uint32)
    lib().moegen_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def normal_f32(seed: int, stream: int, n: int, sigma: float = 1.0, nthreads: int = 0) -> np.ndarray:
    out = np.empty(n, np.float32)
    lib().moegen_normal_f32(seed, stream, n, sigma, _ptr(out), nthreads)
    return out


def u32(seed: int, stream: int, n: int) -> np.ndarray:
    out = np.empty(n, np.uint32)
    lib().moegen_u32(seed, stream, n, _ptr(out))
    return out


def e4m3_encode_gen(v: np.ndarray) -> np.ndarray:
    """The generator's own E4M3 encoder (exposed only so tests can pin it)."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().moegen_e4m3_encode(_ptr(v), v.size, _ptr(out))
    return out


def fp8_blocks(seed: int, stream: int, nmat: int, rows: int, cols: int, ld: int, sigma: float,
               nthreads: int = 0):
    """Synthetic checkpoint matrices: codes uint8 [nmat, rows, ld], scales f32
    [nmat, ceil(rows/128), ceil(cols/128)]; columns >= cols of codes are 0."""
    codes = np.empty((nmat, rows, ld), np.uint8)
    scales = np.empty((nmat, -(-rows // 128), -(-cols // 128)), np.float32)
    rc = lib().moegen_fp8_blocks(seed, stream, nmat, rows, cols, ld, sigma, _ptr(codes), _ptr(scales), nthreads)
    if rc != 0:
        raise ValueError("moegen_fp8_blocks: bad arguments")
    return codes, scales


def f32_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns the uint16 bit patterns."""
    b = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def seeded_choice(seed: int, stream: int, n: int, k: int, lo: int = 0) -> np.ndarray:
    """k distinct integers from [lo, n): a partial Fisher-Yates shuffle driven by u32 words."""
    pool = np.arange(lo, n, dtype=np.int64)
    words = u32(seed, stream, k)
    for i in range(k):
        j = i + int(words[i]) % (len(pool) - i)
        pool[i], pool[j] = pool[j], pool[i]
    return pool[:k].copy()


def seeded_permutation(seed: int, stream: int, n: int) -> np.ndarray:
    return seeded_choice(seed, stream, n, n)


# ---------------------------------------------------------------------------
# Workloads
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class LayerShape:
    H: int          # hidden size
    E: int          # routed experts (the shared expert is index E)
    K: int          # experts per token
    F: int          # expert FFN width (routed and shared)
    ld_f: int       # row stride (bytes) of the down-projection codes, >= F, multiple of 16
    S: int = 1      # shared experts (0 or 1); the shared expert is index E

    @property
    def FB(self) -> int:
        return -(-self.F // 128)

    @property
    def HB(self) -> int:
        return -(-self.H // 128)


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    shape: LayerShape
    x_seed: int
    w_seed: int
    outliers: int = 0        # number of x channels scaled by 20
    zipf: bool = False       # skewed router bias (long-prefill workload)
    note: str = ""


DOTS3 = LayerShape(H=5120, E=256, K=8, F=1536, ld_f=1536)
DOTS3_F1500 = LayerShape(H=5120, E=256, K=8, F=1500, ld_f=1536)
TOY = LayerShape(H=512, E=16, K=4, F=256, ld_f=256)

# Zipf workload constants: rank r gets router bias -ZIPF_ALPHA * ZIPF_S * ln(r);
# the ZIPF_EMPTY lowest-ranked experts get ZIPF_OFF and are never chosen.
# ZIPF_ALPHA was set with tests/golden/make_zipf_alpha.py (the oracle router on the
# seeded T=16384 tokens) so that the busiest expert takes about 10x the mean.
ZIPF_S = 1.1
ZIPF_ALPHA = 0.5508
ZIPF_EMPTY = 16
ZIPF_OFF = -1000.0
ZIPF_CHANNEL = 0   # x[:, 0] = 1 carries the bias through the router GEMM

WORKLOADS = {
    "toy": Workload("toy", 32, TOY, x_seed=0, w_seed=0,
                    note="T=32, hidden 512, 16+1 experts, top-4, FFN 256"),
    # the toy layer at a batch with several row tiles per group (about 600
    # rows each), checked on every token
    "toy_t2048": Workload("toy_t2048", 2048, TOY, x_seed=9, w_seed=0,
                          note="T=2048, hidden 512, 16+1 experts, top-4, FFN 256"),
    "decode": Workload("decode", 64, DOTS3, x_seed=1, w_seed=1, outliers=8,
                       note="T=64, dots3-note MoE layer, balanced router"),
    "prefill": Workload("prefill", 4096, DOTS3, x_seed=2, w_seed=1, outliers=8,
                        note="T=4096, balanced router"),
    "zipf": Workload("zipf", 16384, DOTS3, x_seed=3, w_seed=1, outliers=8, zipf=True,
                     note="T=16384, Zipf(1.1)-biased router"),
    "edge": Workload("edge", 4099, DOTS3, x_seed=4, w_seed=1, outliers=8,
                     note="T=4099 (ragged)"),
    "edge_f1500": Workload("edge_f1500", 4099, DOTS3_F1500, x_seed=4, w_seed=2, outliers=8,
                           note="T=4099 on the FFN=1500 variant (partial 128x128 blocks)"),
    # vision MoE of the ViT encoder (Dots3NoteVisionConfig: hidden_size 1536,
    # num_local_experts 64, moe_intermediate_size 2112 = 16.5 x 128, no
    # shared expert; top-k unstated, read as 2)
    "vision": Workload("vision", 4096, LayerShape(H=1536, E=64, K=2, F=2112, ld_f=2112, S=0), x_seed=6, w_seed=4,
                       note="T=4096 patch tokens, vision MoE: hidden 1536, 64 experts, top-2, FFN 2112, no shared"),
    # the dense FFN layer of the language model (Dots3NoteTextConfig
    # intermediate_size 13824 = 108 x 128) as a one-expert, top-1 layer
    "dense": Workload("dense", 64, LayerShape(H=5120, E=1, K=1, F=13824, ld_f=13824, S=0), x_seed=7, w_seed=5,
                      outliers=8, note="T=64, dense FP8 FFN 5120 -> 2 x 13824 -> 5120 (one expert, weight 1)"),
    # a smaller decode-shaped case (64 routed experts, 1.5 GB of weights) for
    # profiler captures that must stay a few GB on the device
    "decode_e64": Workload("decode_e64", 16, LayerShape(H=5120, E=64, K=8, F=1536, ld_f=1536), x_seed=5,
                           w_seed=3, outliers=8, note="T=16, 64+1 experts, hidden 5120, FFN 1536 (profiling case)"),
    # a prefill-shaped case with several row tiles per expert (about 1000
    # rows each, like the busier experts of the long prefill) whose weights
    # and activations stay near 1 GB, for full profiler captures
    "prefill_e32": Workload("prefill_e32", 4096, LayerShape(H=5120, E=32, K=8, F=1536, ld_f=1536), x_seed=8,
                            w_seed=6, outliers=8,
                            note="T=4096, 32+1 experts, hidden 5120, FFN 1536 (profiling case)"),
}


@dataclass
class Layer:
    """One synthetic FP8 MoE layer (host copies). Shared expert = index E."""
    shape: LayerShape
    router_w: np.ndarray   # f32 [E, H]
    w_gate: np.ndarray     # u8 [E+1, F, H]
    s_gate: np.ndarray     # f32 [E+1, FB, HB]
    w_up: np.ndarray       # u8 [E+1, F, H]
    s_up: np.ndarray       # f32 [E+1, FB, HB]
    w_down: np.ndarray     # u8 [E+1, H, ld_f]
    s_down: np.ndarray     # f32 [E+1, HB, FB]
    meta: dict = field(default_factory=dict)


def make_experts(shape: LayerShape, w_seed: int, nthreads: int = 0):
    """Expert checkpoint (gate, up, down codes and block scales) of one layer."""
    H, E, F = shape.H, shape.E, shape.F
    n = E + shape.S
    wg, sg = fp8_blocks(w_seed, STREAM_GATE, n, F, H, H, 1.0 / math.sqrt(H), nthreads)
    wu, su = fp8_blocks(w_seed, STREAM_UP, n, F, H, H, 1.0 / math.sqrt(H), nthreads)
    wd, sd = fp8_blocks(w_seed, STREAM_DOWN, n, H, F, shape.ld_f, 1.0 / math.sqrt(F), nthreads)
    return wg, sg, wu, su, wd, sd


def make_router(shape: LayerShape, w_seed: int, zipf: bool = False) -> np.ndarray:
    """Router weight f32 [E, H] ~ N(0, 0.02); with zipf, column ZIPF_CHANNEL holds the bias."""
    router = normal_f32(w_seed, STREAM_ROUTER, shape.E * shape.H, 0.02).reshape(shape.E, shape.H)
    if zipf:
        router[:, ZIPF_CHANNEL] = zipf_bias(w_seed, shape.E)
    return router


def make_layer(shape: LayerShape, w_seed: int, zipf: bool = False, nthreads: int = 0, experts=None) -> Layer:
    wg, sg, wu, su, wd, sd = make_experts(shape, w_seed, nthreads) if experts is None else experts
    meta = {"w_seed": w_seed, "zipf": zipf}
    return Layer(shape, make_router(shape, w_seed, zipf), wg, sg, wu, su, wd, sd, meta)


def zipf_bias(seed: int, E: int, alpha: float = None) -> np.ndarray:
    """Per-expert router bias whose popularity profile follows Zipf(ZIPF_S):
    a seeded permutation assigns ranks 1..E; bias = -alpha*s*ln(rank); the
    ZIPF_EMPTY lowest ranks are switched off."""
    alpha = ZIPF_ALPHA if alpha is None else alpha
    perm = seeded_permutation(seed, STREAM_ZIPF, E)   # perm[i] = expert with rank i+1
    rank = np.empty(E, np.int64)
    rank[perm] = np.arange(1, E + 1)
    bias = (-alpha * ZIPF_S * np.log(rank.astype(np.float64))).astype(np.float32)
    bias[rank > E - ZIPF_EMPTY] = np.float32(ZIPF_OFF)
    return bias


def make_x(T: int, H: int, seed: int, outliers: int = 0, zipf: bool = False) -> np.ndarray:
    """Activations as bf16 bit patterns (uint16 [T, H]): N(0,1); `outliers`
    seeded channels scaled by 20; with zipf, channel ZIPF_CHANNEL is 1.0."""
    z = normal_f32(seed, STREAM_X, T * H).reshape(T, H)
    if outliers:
        ch = seeded_choice(seed, STREAM_OUTLIER, H, outliers, lo=1)
        z[:, ch] *= np.float32(20.0)
    if zipf:
        z[:, ZIPF_CHANNEL] = np.float32(1.0)
    return f32_to_bf16_bits(z)


def outlier_channels(seed: int, H: int, outliers: int) -> np.ndarray:
    return seeded_choice(seed, STREAM_OUTLIER, H, outliers, lo=1)


_expert_cache: dict = {}


def workload_inputs(name: str, T: int = None, cache: bool = True):
    """(workload, layer, x_bits) for a named workload; T overrides the token count.
    Expert weights are generated once per (shape, seed) and shared between workloads."""
    wl = WORKLOADS[name]
    key = (wl.shape, wl.w_seed)
    experts = _expert_cache.get(key) if cache else None
    if experts is None:
        experts = make_experts(wl.shape, wl.w_seed)
        if cache:
            _expert_cache[key] = experts
    layer = make_layer(wl.shape, wl.w_seed, zipf=wl.zipf, experts=experts)
    x = make_x(wl.T if T is None else T, wl.shape.H, wl.x_seed, wl.outliers, wl.zipf)
    return wl, layer, x
