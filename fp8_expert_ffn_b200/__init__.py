"""Python binding of libfp8moe.so: argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; this module only
turns tensors into device pointers and calls the C entry points of
include/moe.h by the same names. There is no CPU path: if the shared library
cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

HERE = os.path.dirname(os.path.abspath(__file__))
# FP8MOE_CHECKED=1 selects the bounds-checked build (-DMOE_CHECKS)
CHECKED = os.environ.get("FP8MOE_CHECKED", "") == "1"
LIB_PATH = os.path.join(HERE, "libfp8moe_checked.so" if CHECKED else "libfp8moe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_MISALIGNED, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, \
    MOE_ERR_DEVICE = range(7)

ENTRY_POINTS = ("moe_status_string", "moe_layer_create", "moe_layer_destroy", "moe_workspace_size", "moe_route",
                "moe_permute", "moe_expert_ffn", "moe_combine", "moe_layer_forward", "moe_get_device_status",
                "moe_gate_up", "moe_down", "moe_test_grouped_gemm_f32", "moe_permute_noalloc",
                "moe_kernels_per_forward", "moe_test_inject_stall", "moe_grouped_gate_up", "moe_grouped_down",
                "moe_ep_pack_scales", "moe_ep_regroup", "moe_ep_unregroup", "moe_ep_comm_create",
                "moe_ep_comm_export", "moe_ep_comm_connect", "moe_ep_comm_connect_local", "moe_ep_comm_buffers",
                "moe_ep_comm_destroy", "moe_ep_plan", "moe_ep_dispatch", "moe_ep_combine")

MOE_EP_HANDLE_BYTES = 64        # include/moe.h

MOE_NOALLOC_MAX_TOKENS = 4096   # include/moe.h


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int, text: str):
        super().__init__(f"{fn}: {text} (status {code})")
        self.code = code


class moe_layer_desc(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("n_routed", ctypes.c_int), ("n_shared", ctypes.c_int),
                ("top_k", ctypes.c_int), ("ffn", ctypes.c_int), ("shared_ffn", ctypes.c_int),
                ("block", ctypes.c_int), ("routed_scaling", ctypes.c_float), ("norm_topk", ctypes.c_int),
                ("n_group", ctypes.c_int), ("topk_group", ctypes.c_int)]


class moe_weights(ctypes.Structure):
    _fields_ = [("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p),
                ("s_gate", ctypes.c_void_p), ("s_up", ctypes.c_void_p), ("s_down", ctypes.c_void_p),
                ("router_w", ctypes.c_void_p), ("ld_h", ctypes.c_int), ("ld_f", ctypes.c_int),
                ("router_bias", ctypes.c_void_p)]


_lib = None


def lib(build_if_missing: bool = True):
    """Load libfp8moe.so (building it in-tree first if it is missing or stale)."""
    global _lib
    if _lib is not None:
        return _lib
    if build_if_missing:
        from . import build as _build
        if _build.stale(CHECKED):
            _build.build(checked=CHECKED)
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"fp8_expert_ffn_b200: CUDA library not built ({LIB_PATH})")
    L = ctypes.CDLL(LIB_PATH)
    P, I, S, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    L.moe_status_string.argtypes = [I]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_layer_create.argtypes = [ctypes.POINTER(moe_layer_desc), ctypes.POINTER(moe_weights), ctypes.POINTER(P)]
    L.moe_layer_destroy.argtypes = [P]
    L.moe_workspace_size.argtypes = [P, I]
    L.moe_workspace_size.restype = S
    L.moe_route.argtypes = [P, P, I, I, P, P, P, P, S, P]
    L.moe_permute.argtypes = [P, P, I, I, P, P, P, P, P, P, P, S, P]
    L.moe_expert_ffn.argtypes = [P, P, P, P, I, P, P, S, P]
    L.moe_combine.argtypes = [P, P, P, P, I, P, I, P]
    L.moe_layer_forward.argtypes = [P, P, I, I, P, I, P, S, P]
    L.moe_get_device_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32)]
    L.moe_gate_up.argtypes = [P, P, P, P, I, P, P, P]
    L.moe_permute_noalloc.argtypes = [P, P, I, I, P, P, P, P, P, P, P]
    L.moe_down.argtypes = [P, P, P, P, I, P, P]
    L.moe_test_grouped_gemm_f32.argtypes = [P, I, P, P, P, I, P, P]
    L.moe_kernels_per_forward.argtypes = [P, I]
    L.moe_test_inject_stall.argtypes = [P, ctypes.c_ulonglong]
    L.moe_grouped_gate_up.argtypes = [P, P, P, P, I, P, P, P]
    L.moe_grouped_down.argtypes = [P, P, P, P, I, P, P]
    L.moe_ep_pack_scales.argtypes = [P, P, I, P, P]
    L.moe_ep_regroup.argtypes = [P, I, P, I, P, P, P, P, I, P, P, P, P]
    L.moe_ep_unregroup.argtypes = [P, I, P, I, P, I, P, P, P]
    L.moe_ep_comm_create.argtypes = [P, I, I, I, ctypes.POINTER(P)]
    L.moe_ep_comm_export.argtypes = [P, ctypes.c_char_p]
    L.moe_ep_comm_connect.argtypes = [P, ctypes.c_char_p]
    L.moe_ep_comm_connect_local.argtypes = [ctypes.POINTER(P), I]
    L.moe_ep_comm_buffers.argtypes = [P, ctypes.POINTER(P), ctypes.POINTER(P), ctypes.POINTER(P)]
    L.moe_ep_comm_destroy.argtypes = [P]
    L.moe_ep_plan.argtypes = [P, P, I, P, P, S, P]
    L.moe_ep_dispatch.argtypes = [P, P, P, I, I, P, P, P, P, P, S, P]
    L.moe_ep_combine.argtypes = [P, P, P, P, P, P, I, P, I, P]
    for name in ENTRY_POINTS:
        if name not in ("moe_status_string", "moe_workspace_size"):
            getattr(L, name).restype = I
    _lib = L
    return L


def status_string(code: int) -> str:
    return lib().moe_status_string(code).decode()


def _check(fn: str, code: int):
    if code != MOE_OK:
        raise MoeError(fn, code, status_string(code))


def _ptr(t) -> int:
    if t is None:
        return 0
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


@dataclass
class LayerWeights:
    """Device tensors of one layer (uint8 codes, float32 scales/router)."""
    w_gate: object
    w_up: object
    w_down: object
    s_gate: object
    s_up: object
    s_down: object
    router_w: object


class MoeLayer:
    """Owns a moe_layer_t; keeps the weight tensors alive while it exists."""

    def __init__(self, hidden, n_routed, top_k, ffn, weights: LayerWeights, ld_h=None, ld_f=None,
                 routed_scaling=1.0, n_shared=1, n_group=1, topk_group=1, norm_topk=True, router_bias=None):
        """router_bias: device fp32 [E] selection-only bias (copied at creation) or None."""
        self.H, self.E, self.K, self.F = hidden, n_routed, top_k, ffn
        self.weights = weights
        self.S = n_shared
        self.ld_h = hidden if ld_h is None else ld_h
        self.ld_f = ffn if ld_f is None else ld_f
        self.routed_scaling, self.n_group, self.topk_group = routed_scaling, n_group, topk_group
        self.norm_topk, self.router_bias = bool(norm_topk), router_bias
        d = moe_layer_desc(hidden, n_routed, n_shared, top_k, ffn, ffn, 128, routed_scaling, int(bool(norm_topk)),
                           n_group, topk_group)
        w = moe_weights(_ptr(weights.w_gate), _ptr(weights.w_up), _ptr(weights.w_down), _ptr(weights.s_gate),
                        _ptr(weights.s_up), _ptr(weights.s_down), _ptr(weights.router_w),
                        hidden if ld_h is None else ld_h, ffn if ld_f is None else ld_f, _ptr(router_bias))
        h = ctypes.c_void_p()
        _check("moe_layer_create", lib().moe_layer_create(ctypes.byref(d), ctypes.byref(w), ctypes.byref(h)))
        self.handle = h.value

    def close(self):
        if getattr(self, "handle", None):
            lib().moe_layer_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def rows(self, T: int) -> int:
        return T * (self.K + self.S)


def moe_kernels_per_forward(layer: MoeLayer, T: int) -> int:
    return int(lib().moe_kernels_per_forward(layer.handle, T))


def moe_grouped_gate_up(layer, xq, xs, offsets, rows, h, hs, stream=None):
    _check("moe_grouped_gate_up", lib().moe_grouped_gate_up(layer.handle, _ptr(xq), _ptr(xs), _ptr(offsets), rows,
                                                            _ptr(h), _ptr(hs), _stream(stream)))


def moe_grouped_down(layer, h, hs, offsets, rows, y, stream=None):
    _check("moe_grouped_down", lib().moe_grouped_down(layer.handle, _ptr(h), _ptr(hs), _ptr(offsets), rows, _ptr(y),
                                                      _stream(stream)))


def moe_ep_pack_scales(layer, xs, T, xs_rows, stream=None):
    _check("moe_ep_pack_scales", lib().moe_ep_pack_scales(layer.handle, _ptr(xs), T, _ptr(xs_rows), _stream(stream)))


def moe_ep_regroup(layer, ranks, seg_counts, n_recv, recv_q, recv_s, own_q, own_s, T, out_q, out_s, out_offsets,
                   stream=None):
    _check("moe_ep_regroup", lib().moe_ep_regroup(layer.handle, ranks, _ptr(seg_counts), n_recv, _ptr(recv_q),
                                                  _ptr(recv_s), _ptr(own_q), _ptr(own_s), T, _ptr(out_q),
                                                  _ptr(out_s), _ptr(out_offsets), _stream(stream)))


def moe_ep_unregroup(layer, ranks, seg_counts, n_recv, y_g, T, y_send, y_own, stream=None):
    _check("moe_ep_unregroup", lib().moe_ep_unregroup(layer.handle, ranks, _ptr(seg_counts), n_recv, _ptr(y_g), T,
                                                      _ptr(y_send), _ptr(y_own), _stream(stream)))


class EpComm:
    """One rank's exchange buffers for the expert-parallel dispatch and
    combine over peer memory (moe_ep_comm_*); `capacity` rows each."""

    def __init__(self, layer: MoeLayer, rank: int, ranks: int, capacity: int):
        h = ctypes.c_void_p()
        _check("moe_ep_comm_create", lib().moe_ep_comm_create(layer.handle, rank, ranks, capacity, ctypes.byref(h)))
        self.handle = h.value
        self.rank, self.ranks, self.capacity = rank, ranks, capacity
        q, s, y = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
        _check("moe_ep_comm_buffers", lib().moe_ep_comm_buffers(self.handle, ctypes.byref(q), ctypes.byref(s),
                                                                ctypes.byref(y)))
        self.recv_q, self.recv_s, self.y = q.value, s.value, y.value   # device addresses

    def export(self) -> bytes:
        buf = ctypes.create_string_buffer(MOE_EP_HANDLE_BYTES)
        _check("moe_ep_comm_export", lib().moe_ep_comm_export(self.handle, buf))
        return buf.raw

    def connect(self, handles):
        """handles: every rank's export(), in rank order."""
        blob = b"".join(handles)
        if len(blob) != MOE_EP_HANDLE_BYTES * self.ranks:
            raise ValueError("one handle per rank expected")
        _check("moe_ep_comm_connect", lib().moe_ep_comm_connect(self.handle, blob))

    @staticmethod
    def connect_local(comms):
        arr = (ctypes.c_void_p * len(comms))(*[c.handle for c in comms])
        _check("moe_ep_comm_connect_local", lib().moe_ep_comm_connect_local(arr, len(comms)))

    def close(self):
        if getattr(self, "handle", None):
            lib().moe_ep_comm_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_ep_plan(layer, topk_idx, T, offsets, ws, ws_bytes, stream=None):
    _check("moe_ep_plan", lib().moe_ep_plan(layer.handle, _ptr(topk_idx), T, _ptr(offsets), _ptr(ws), ws_bytes,
                                            _stream(stream)))


def moe_ep_dispatch(layer, comm: EpComm, x, T, ldx, topk_idx, all_offsets, inv_ep, group_offsets, ws, ws_bytes,
                    stream=None):
    _check("moe_ep_dispatch", lib().moe_ep_dispatch(layer.handle, comm.handle, _ptr(x), T, ldx, _ptr(topk_idx),
                                                    _ptr(all_offsets), _ptr(inv_ep), _ptr(group_offsets), _ptr(ws),
                                                    ws_bytes, _stream(stream)))


def moe_ep_combine(layer, comm: EpComm, topk_idx, inv_ep, topk_w, group_offsets, T, out, ldo, stream=None):
    _check("moe_ep_combine", lib().moe_ep_combine(layer.handle, comm.handle, _ptr(topk_idx), _ptr(inv_ep),
                                                  _ptr(topk_w), _ptr(group_offsets), T, _ptr(out), ldo,
                                                  _stream(stream)))


def moe_test_inject_stall(layer: MoeLayer, wait_limit_ns: int):
    _check("moe_test_inject_stall", lib().moe_test_inject_stall(layer.handle, int(wait_limit_ns)))


def moe_workspace_size(layer: MoeLayer, T: int) -> int:
    return int(lib().moe_workspace_size(layer.handle, T))


def moe_route(layer, x, T, ldx, topk_idx, topk_w, router_logits, ws, ws_bytes, stream=None):
    _check("moe_route", lib().moe_route(layer.handle, _ptr(x), T, ldx, _ptr(topk_idx), _ptr(topk_w),
                                        _ptr(router_logits), _ptr(ws), ws_bytes, _stream(stream)))


def moe_permute(layer, x, T, ldx, topk_idx, offsets, perm, inv, xq, xs, ws, ws_bytes, stream=None):
    _check("moe_permute", lib().moe_permute(layer.handle, _ptr(x), T, ldx, _ptr(topk_idx), _ptr(offsets),
                                            _ptr(perm), _ptr(inv), _ptr(xq), _ptr(xs), _ptr(ws), ws_bytes,
                                            _stream(stream)))


def moe_expert_ffn(layer, xq, xs, offsets, T, y, ws, ws_bytes, stream=None):
    _check("moe_expert_ffn", lib().moe_expert_ffn(layer.handle, _ptr(xq), _ptr(xs), _ptr(offsets), T, _ptr(y),
                                                  _ptr(ws), ws_bytes, _stream(stream)))


def moe_combine(layer, y, inv, topk_w, T, out, ldo, stream=None):
    _check("moe_combine", lib().moe_combine(layer.handle, _ptr(y), _ptr(inv), _ptr(topk_w), T, _ptr(out), ldo,
                                            _stream(stream)))


def moe_layer_forward(layer, x, T, ldx, out, ldo, ws, ws_bytes, stream=None):
    _check("moe_layer_forward", lib().moe_layer_forward(layer.handle, _ptr(x), T, ldx, _ptr(out), ldo, _ptr(ws),
                                                        ws_bytes, _stream(stream)))


def moe_get_device_status(layer, stream=None):
    """(status code, raw bits); synchronises the stream."""
    bits = ctypes.c_uint32(0)
    code = lib().moe_get_device_status(layer.handle, _stream(stream), ctypes.byref(bits))
    return code, bits.value


def moe_gate_up(layer, xq, xs, offsets, T, h, hs, stream=None):
    _check("moe_gate_up", lib().moe_gate_up(layer.handle, _ptr(xq), _ptr(xs), _ptr(offsets), T, _ptr(h), _ptr(hs),
                                            _stream(stream)))


def moe_down(layer, h, hs, offsets, T, y, stream=None):
    _check("moe_down", lib().moe_down(layer.handle, _ptr(h), _ptr(hs), _ptr(offsets), T, _ptr(y), _stream(stream)))


def moe_test_grouped_gemm_f32(layer, which, a, a_scales, offsets, T, out, stream=None):
    _check("moe_test_grouped_gemm_f32",
           lib().moe_test_grouped_gemm_f32(layer.handle, which, _ptr(a), _ptr(a_scales), _ptr(offsets), T,
                                           _ptr(out), _stream(stream)))


def moe_permute_noalloc(layer, x, T, ldx, topk_idx, offsets, perm, inv, xq, xs, stream=None):
    """moe_permute without a workspace (scratch in a library-owned device
    array; T <= MOE_NOALLOC_MAX_TOKENS; calls that overlap on the GPU race)."""
    _check("moe_permute_noalloc",
           lib().moe_permute_noalloc(layer.handle, _ptr(x), T, ldx, _ptr(topk_idx), _ptr(offsets), _ptr(perm),
                                     _ptr(inv), _ptr(xq), _ptr(xs), _stream(stream)))
