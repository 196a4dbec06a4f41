"""The C++ FP64 oracle (moe_oracle.cpp, plain loops) behind the numpy
oracle's function names, so that the same pins and cross-checks run on both.

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline legs may import this module. It shares no code with the CUDA path
and none with the numpy oracle (moe.py): this file only marshals arrays into
and out of the C library, whose loops do all the arithmetic.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.cpp")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

GROUP = 128
NEAR_TIE = 1e-6


def build(force: bool = False) -> str:
    """Compile libmoe_oracle.so in-tree (g++, a few seconds)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread", "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


class _Layer(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("E", ctypes.c_int), ("S", ctypes.c_int), ("K", ctypes.c_int),
                ("F", ctypes.c_int), ("ld_f", ctypes.c_int),
                ("w_gate", ctypes.c_void_p), ("s_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p),
                ("s_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p), ("s_down", ctypes.c_void_p)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        sig = {
            "oracle_threads": ([], I),
            "oracle_e4m3_table": ([P], None),
            "oracle_e4m3_encode": ([P, I64, P], None),
            "oracle_round_bf16": ([P, I64, P], None),
            "oracle_silu": ([P, I64, P], None),
            "oracle_quantize_rows": ([P, I64, I, P, P], None),
            "oracle_dequant_rows": ([P, I64, P, I64, I, P], None),
            "oracle_dequant_block": ([P, I64, P, I, I, P], None),
            "oracle_router_logits": ([P, I, I, P, I, P], None),
            "oracle_softmax": ([P, I, I, P], None),
            "oracle_select_topk": ([P, I, I, I, D, I, I, P, I, P, P, P], None),
            "oracle_permute": ([P, I, I, I, I, P, P, P], None),
            "oracle_expert_ffn_rows": ([P, P, P, P, P, I, P, P, P, P], None),
            "oracle_expert_down_rows": ([P, P, P, P, P, I, P], None),
            "oracle_combine": ([P, I, P, P, I, I, I, P], None),
            "oracle_token_outputs": ([P, P, I, P, P, P], None),
            "oracle_layer_forward_bf16": ([P, P, I, P, P, P], None),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: np.ndarray) -> int:
    return a.ctypes.data


def threads() -> int:
    return lib().oracle_threads()


# ------------------------------------------------------------------ E4M3 and numbers

def e4m3_table() -> np.ndarray:
    out = np.empty(256, np.float64)
    lib().oracle_e4m3_table(_p(out))
    return out


def e4m3_decode(codes) -> np.ndarray:
    return e4m3_table()[np.asarray(codes, np.uint8)]


def e4m3_encode(v) -> np.ndarray:
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().oracle_e4m3_encode(_p(v), v.size, _p(out))
    return out


def bf16_to_f64(bits) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16_f64(v) -> np.ndarray:
    v = _c(v, np.float64)
    out = np.empty(v.shape, np.float64)
    lib().oracle_round_bf16(_p(v), v.size, _p(out))
    return out


def silu(g) -> np.ndarray:
    g = _c(g, np.float64)
    out = np.empty(g.shape, np.float64)
    lib().oracle_silu(_p(g), g.size, _p(out))
    return out


# ------------------------------------------------------------------ quantisation

def quantize_rows(v):
    v = _c(v, np.float32)
    rows, C = v.shape
    codes = np.empty((rows, C), np.uint8)
    scales = np.empty((rows, -(-C // GROUP)), np.float32)
    lib().oracle_quantize_rows(_p(v), rows, C, _p(codes), _p(scales))
    return codes, scales


def dequant_rows(codes, scales, C: int = None) -> np.ndarray:
    codes = _c(codes, np.uint8)
    C = codes.shape[1] if C is None else C
    scales = _c(np.asarray(scales, np.float32)[:, :-(-C // GROUP)], np.float32)
    out = np.empty((codes.shape[0], C), np.float64)
    lib().oracle_dequant_rows(_p(codes), codes.shape[1], _p(scales), codes.shape[0], C, _p(out))
    return out


def dequant_block(codes, scales, rows: int, cols: int) -> np.ndarray:
    codes = _c(codes, np.uint8)
    scales = _c(np.asarray(scales, np.float32)[:-(-rows // GROUP), :-(-cols // GROUP)], np.float32)
    out = np.empty((rows, cols), np.float64)
    lib().oracle_dequant_block(_p(codes), codes.shape[1], _p(scales), rows, cols, _p(out))
    return out


# ------------------------------------------------------------------ routing

@dataclass
class Route:
    logits: np.ndarray
    probs: np.ndarray
    idx: np.ndarray
    w: np.ndarray
    gap: np.ndarray
    near_tie: np.ndarray


def router_logits(x_bits, router_w) -> np.ndarray:
    x = _c(x_bits, np.uint16)
    wr = _c(router_w, np.float32)
    T, H = x.shape
    out = np.empty((T, wr.shape[0]), np.float64)
    lib().oracle_router_logits(_p(x), T, H, _p(wr), wr.shape[0], _p(out))
    return out


def softmax(logits) -> np.ndarray:
    lg = _c(logits, np.float64)
    out = np.empty(lg.shape, np.float64)
    lib().oracle_softmax(_p(lg), lg.shape[0], lg.shape[1], _p(out))
    return out


def select_topk(probs, K: int, routed_scaling: float = 1.0, n_group: int = 1, topk_group: int = 1, bias=None,
                norm_topk: bool = True):
    p = _c(probs, np.float64)
    T, E = p.shape
    b = None if bias is None else _c(bias, np.float64)
    idx = np.empty((T, K), np.int32)
    w = np.empty((T, K), np.float64)
    gap = np.empty(T, np.float64)
    lib().oracle_select_topk(_p(p), T, E, K, float(routed_scaling), n_group, topk_group,
                             None if b is None else _p(b), int(bool(norm_topk)), _p(idx), _p(w), _p(gap))
    return idx, w, gap


def route(x_bits, router_w, K: int, routed_scaling: float = 1.0, n_group: int = 1, topk_group: int = 1,
          bias=None, norm_topk: bool = True) -> Route:
    logits = router_logits(x_bits, router_w)
    probs = softmax(logits)
    idx, w, gap = select_topk(probs, K, routed_scaling, n_group, topk_group, bias, norm_topk)
    return Route(logits, probs, idx, w, gap, gap < NEAR_TIE)


def router_options(layer) -> dict:
    return {"routed_scaling": getattr(layer, "routed_scaling", 1.0), "n_group": getattr(layer, "n_group", 1),
            "topk_group": getattr(layer, "topk_group", 1), "bias": getattr(layer, "router_bias", None),
            "norm_topk": getattr(layer, "norm_topk", True)}


def route_layer(x_bits, layer) -> Route:
    return route(x_bits, layer.router_w, layer.shape.K, **router_options(layer))


# ------------------------------------------------------------------ permutation

@dataclass
class Perm:
    offsets: np.ndarray
    perm: np.ndarray
    inv: np.ndarray


def permute(idx, E: int, S: int = 1) -> Perm:
    idx = _c(idx, np.int32)
    T, K = idx.shape
    offsets = np.empty(E + 2, np.int32)
    perm = np.empty(T * K + T * S, np.int32)
    inv = np.empty((T, K), np.int32)
    lib().oracle_permute(_p(idx), T, K, E, S, _p(offsets), _p(perm), _p(inv))
    return Perm(offsets, perm, inv)


# ------------------------------------------------------------------ expert FFN, combine, layer

class _LayerRef:
    """The C struct of a layer plus the contiguous arrays it points into."""

    def __init__(self, layer):
        sh = layer.shape
        self.keep = [_c(layer.w_gate, np.uint8), _c(layer.s_gate, np.float32), _c(layer.w_up, np.uint8),
                     _c(layer.s_up, np.float32), _c(layer.w_down, np.uint8), _c(layer.s_down, np.float32)]
        self.s = _Layer(sh.H, sh.E, sh.S, sh.K, sh.F, sh.ld_f, *[_p(a) for a in self.keep])

    @property
    def ptr(self):
        return ctypes.byref(self.s)


def _groups(layer, groups):
    E1 = layer.shape.E + layer.shape.S
    return _c(np.arange(E1) if groups is None else np.asarray(list(groups)), np.int32)


def expert_ffn_rows(xq, xs, offsets, layer, groups=None) -> dict:
    sh = layer.shape
    xq, xs = _c(xq, np.uint8), _c(xs, np.float32)
    off = _c(offsets, np.int32)
    rows = int(off[-1])
    h = np.zeros((rows, sh.F), np.float64)
    hq = np.zeros((rows, sh.F), np.uint8)
    hs = np.zeros((rows, sh.FB), np.float32)
    y = np.zeros((rows, sh.H), np.float64)
    g = _groups(layer, groups)
    L = _LayerRef(layer)
    lib().oracle_expert_ffn_rows(L.ptr, _p(xq), _p(xs), _p(off), _p(g), len(g), _p(h), _p(hq), _p(hs), _p(y))
    return {"h": h, "hq": hq, "hs": hs, "y": y}


def expert_down_rows(hq, hs, offsets, layer, groups=None) -> np.ndarray:
    sh = layer.shape
    hq = _c(np.asarray(hq)[:, :sh.F], np.uint8)
    hs = _c(hs, np.float32)
    off = _c(offsets, np.int32)
    y = np.zeros((int(off[-1]), sh.H), np.float64)
    g = _groups(layer, groups)
    L = _LayerRef(layer)
    lib().oracle_expert_down_rows(L.ptr, _p(hq), _p(hs), _p(off), _p(g), len(g), _p(y))
    return y


def combine(y, inv, w, S: int = 1) -> np.ndarray:
    y, inv, w = _c(y, np.float64), _c(inv, np.int32), _c(w, np.float64)
    T, K = inv.shape
    out = np.empty((T, y.shape[1]), np.float64)
    lib().oracle_combine(_p(y), y.shape[1], _p(inv), _p(w), T, K, S, _p(out))
    return out


def quantize_tokens(x_bits):
    return quantize_rows(bf16_to_f64(x_bits).astype(np.float32))


def gather_rows(tok_codes, tok_scales, perm):
    return tok_codes[perm], tok_scales[perm]


def layer_forward(x_bits, layer) -> dict:
    """Whole layer: route -> permute -> quantise/gather -> expert FFNs -> combine."""
    sh = layer.shape
    r = route_layer(x_bits, layer)
    p = permute(r.idx, sh.E, sh.S)
    tq, ts = quantize_tokens(x_bits)
    xq, xs = gather_rows(tq, ts, p.perm)
    f = expert_ffn_rows(xq, xs, p.offsets, layer)
    out = combine(f["y"], p.inv, r.w, sh.S)
    return {"route": r, "perm": p, "xq": xq, "xs": xs, **f, "out": out}


def _routing(x_bits, layer, tokens, idx, w):
    tokens = np.asarray(tokens)
    xb = _c(np.asarray(x_bits)[tokens], np.uint16)
    if idx is None:
        r = route_layer(xb, layer)
        return xb, _c(r.idx, np.int32), _c(r.w, np.float64)
    return xb, _c(np.asarray(idx)[tokens], np.int32), _c(np.asarray(w, np.float64)[tokens], np.float64)


def token_outputs(x_bits, layer, tokens, idx=None, w=None) -> np.ndarray:
    """Direct per-token evaluation (no permutation) of the given tokens."""
    xb, idx_s, w_s = _routing(x_bits, layer, tokens, idx, w)
    out = np.empty((xb.shape[0], layer.shape.H), np.float64)
    L = _LayerRef(layer)
    lib().oracle_token_outputs(L.ptr, _p(xb), xb.shape[0], _p(idx_s), _p(w_s), _p(out))
    return out


def layer_forward_bf16(x_bits, layer, tokens=None, idx=None, w=None) -> np.ndarray:
    """BF16-checkpoint path: W = bf16(q s), no activation or h quantisation."""
    T = np.asarray(x_bits).shape[0]
    xb, idx_s, w_s = _routing(x_bits, layer, np.arange(T) if tokens is None else tokens, idx, w)
    out = np.empty((xb.shape[0], layer.shape.H), np.float64)
    L = _LayerRef(layer)
    lib().oracle_layer_forward_bf16(L.ptr, _p(xb), xb.shape[0], _p(idx_s), _p(w_s), _p(out))
    return out
