"""Shared pieces of the GPU parity tests: runs every stage of the CUDA path on
one seeded workload and keeps the device results, so that each test can
compare one stage against the oracle fed with the GPU's upstream outputs
(teacher forcing)."""
from __future__ import annotations

import numpy as np
import torch

import fp8_expert_ffn_b200 as fx
from fp8_expert_ffn_b200 import torch_utils as tu
from oracle import e4m3, moe

# Output tolerance: relative Frobenius error and max-abs error relative to the
# oracle output's rms (the layer's stated parity bar).
REL_FRO = 5e-3
MAX_ABS_RMS = 2e-2


class Case:
    """Runs route -> permute -> expert_ffn -> combine through the C ABI."""

    def __init__(self, host_layer, x_bits: np.ndarray, device_layer=None):
        self.host = host_layer
        sh = host_layer.shape
        self.sh = sh
        self.T = x_bits.shape[0]
        self.x_bits = x_bits
        self.dev = device_layer if device_layer is not None else tu.upload_layer(host_layer)
        T, K, E, H = self.T, sh.K, sh.E, sh.H
        rows = T * (K + sh.S)
        self.rows = rows
        d = "cuda"
        self.x = tu.bf16_tensor(x_bits)
        self.ws = tu.workspace(self.dev, T)
        nb = self.ws.numel()
        self.idx = torch.empty((T, K), dtype=torch.int32, device=d)
        self.w = torch.empty((T, K), dtype=torch.float32, device=d)
        self.logits = torch.empty((T, E), dtype=torch.float32, device=d)
        fx.moe_route(self.dev, self.x, T, H, self.idx, self.w, self.logits, self.ws, nb)
        self.offsets = torch.empty(E + 2, dtype=torch.int32, device=d)
        self.perm = torch.empty(rows, dtype=torch.int32, device=d)
        self.inv = torch.empty((T, K), dtype=torch.int32, device=d)
        self.xq = torch.empty((rows, H), dtype=torch.uint8, device=d)
        self.xs = torch.empty((sh.HB, rows), dtype=torch.float32, device=d)
        fx.moe_permute(self.dev, self.x, T, H, self.idx, self.offsets, self.perm, self.inv, self.xq, self.xs,
                       self.ws, nb)
        self.hq = torch.empty((rows, sh.FB * 128), dtype=torch.uint8, device=d)
        self.hs = torch.empty((sh.FB, rows), dtype=torch.float32, device=d)
        fx.moe_gate_up(self.dev, self.xq, self.xs, self.offsets, T, self.hq, self.hs)
        self.y = torch.empty((rows, H), dtype=torch.bfloat16, device=d)
        fx.moe_down(self.dev, self.hq, self.hs, self.offsets, T, self.y)
        self.out = torch.empty((T, H), dtype=torch.bfloat16, device=d)
        fx.moe_combine(self.dev, self.y, self.inv, self.w, T, self.out, H)
        code, bits = fx.moe_get_device_status(self.dev)
        assert code == fx.MOE_OK, f"device status {bits:#x}"

    # host copies
    def np(self, name):
        t = getattr(self, name)
        if t.dtype == torch.bfloat16:
            return tu.bf16_bits(t)
        return t.cpu().numpy()


def bf16_f64(bits):
    return moe.bf16_to_f64(bits)


def rows_of_tokens(inv: np.ndarray, T: int, K: int, tokens, S: int = 1) -> np.ndarray:
    tokens = np.asarray(tokens)
    return np.concatenate([inv[tokens].ravel(), T * K + tokens]) if S else inv[tokens].ravel()


def oracle_ffn_on_rows(layer, rows, xq, xs_rows_major, offsets):
    """Oracle expert FFN for a subset of permuted rows (each row keeps its own
    group); returns dict of h/hq/hs/y for those rows, in the order given."""
    rows = np.asarray(rows)
    groups = np.searchsorted(offsets, rows, side="right") - 1
    order = np.argsort(groups, kind="stable")
    g_sorted = groups[order]
    E1 = layer.shape.E + 1
    off = np.zeros(E1 + 1, np.int64)
    off[1:] = np.cumsum(np.bincount(g_sorted, minlength=E1)[:E1])
    f = moe.expert_ffn_rows(xq[rows[order]], xs_rows_major[rows[order]], off, layer,
                            groups=np.unique(g_sorted))
    inv_order = np.empty_like(order)
    inv_order[order] = np.arange(len(order))
    return {k: v[inv_order] for k, v in f.items()}


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    """Half a unit in the last place of bf16 (8 significant bits) at |v|."""
    a = np.maximum(np.abs(np.asarray(v, np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 8)


def assert_output_close(got: np.ndarray, ref: np.ndarray, what: str, rel_fro=REL_FRO, max_abs_rms=MAX_ABS_RMS):
    """The layer's parity bar on a bf16 output against the unrounded FP64
    oracle: relative Frobenius error <= rel_fro, and max-abs error <=
    max_abs_rms * rms(ref) applied to the value before its one rounding to
    bf16, i.e. |got - ref| <= max_abs_rms * rms + half a bf16 ulp of ref.
    (Without the half ulp no bf16 output could pass once |ref| > 5.1 rms.)"""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    rms = np.sqrt(np.mean(ref ** 2))
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    err = np.abs(got - ref)
    excess = err - bf16_half_ulp(ref)
    mx = float(np.max(excess)) if got.size else 0.0
    assert rel <= rel_fro, f"{what}: relative Frobenius error {rel:.3e} > {rel_fro}"
    assert mx <= max_abs_rms * rms, \
        f"{what}: max abs error beyond bf16 rounding {mx:.3e} > {max_abs_rms} * rms {rms:.3e}" \
        f" (raw max abs {err.max():.3e})"
    return rel, mx / rms


def e4m3_step_diff(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance between E4M3 codes in representable steps (sign-aware)."""
    def ordinal(c):
        c = c.astype(np.int64)
        mag = c & 0x7F
        return np.where(c & 0x80, -mag, mag)
    return np.abs(ordinal(a) - ordinal(b))
