"""Parity of the whole forward on layer shapes beyond the named workloads:
expert counts that are not multiples of 32 (router tiles and top-K lanes
partly empty), top-K from 1 to 8, FFN widths with partial 128-blocks and
down-projection row strides padded to 16 bytes, hidden sizes of one to
twelve 128-channel groups, with and without the shared expert, and token
counts around the tile and bitmap-word edges. Every token is compared with
the oracle's direct per-token evaluation (tokens whose top-K gap is below
1e-6 excluded): within the output bar of the oracle that keeps each expert
row in bf16 as the layer does, and within the relative bar of the all-FP64
oracle. The stage calls must give the fused call's bytes."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import gen  # noqa: E402
from oracle import moe  # noqa: E402

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

import fp8_expert_ffn_b200 as fx  # noqa: E402
from fp8_expert_ffn_b200 import torch_utils as tu  # noqa: E402
import gpu_case as gc  # noqa: E402

# (H, E, K, F, S, T)
SHAPES = [
    (128, 3, 1, 200, 1, 1),
    (256, 7, 2, 128, 0, 33),
    (384, 40, 6, 320, 1, 129),
    (512, 33, 8, 96, 1, 257),
    (1024, 100, 4, 1000, 0, 300),
    (1536, 256, 8, 136, 1, 95),
]


def _ld(F):
    return -(-F // 16) * 16


@pytest.mark.parametrize("H,E,K,F,S,T", SHAPES)
def test_forward_on_shape(H, E, K, F, S, T):
    sh = gen.LayerShape(H=H, E=E, K=K, F=F, ld_f=_ld(F), S=S)
    seed = 1000 + H + E + K + F
    layer = gen.make_layer(sh, seed)
    x_bits = gen.make_x(T, H, seed + 1, outliers=2)
    dev = tu.upload_layer(layer)
    x = tu.bf16_tensor(x_bits)
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    ws = tu.workspace(dev, T)
    fx.moe_layer_forward(dev, x, T, H, out, H, ws, ws.numel())
    code, bits = fx.moe_get_device_status(dev)
    assert code == fx.MOE_OK, hex(bits)
    r = moe.route(x_bits, layer.router_w, K)
    keep = np.nonzero(~r.near_tie)[0]
    got = moe.bf16_to_f64(tu.bf16_bits(out))[keep]
    what = f"shape H={H} E={E} K={K} F={F} S={S} T={T}"
    # against the oracle with the layer's bf16 expert rows (y is a bf16
    # tensor): the full bar; against the all-FP64 oracle: the relative error
    # (a lone expert row several times the output rms carries its own bf16
    # rounding, which the max-abs bar on the output does not allow for)
    ref_y = moe.token_outputs(x_bits, layer, keep, y_bf16=True)
    gc.assert_output_close(got, ref_y, what + " (bf16 expert rows)")
    ref = moe.token_outputs(x_bits, layer, keep)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel <= gc.REL_FRO, f"{what}: relative Frobenius error {rel:.3e} against the FP64 oracle"
    # the stage calls give the fused call's bytes
    rows = T * (K + S)
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    fx.moe_route(dev, x, T, H, idx, w, None, ws, ws.numel())
    assert np.array_equal(idx.cpu().numpy()[keep], r.idx[keep])
    off = torch.empty(E + 2, dtype=torch.int32, device="cuda")
    perm = torch.empty(rows, dtype=torch.int32, device="cuda")
    inv = torch.empty((T, K), dtype=torch.int32, device="cuda")
    xq = torch.empty((rows, H), dtype=torch.uint8, device="cuda")
    xs = torch.empty((sh.HB, rows), dtype=torch.float32, device="cuda")
    fx.moe_permute(dev, x, T, H, idx, off, perm, inv, xq, xs, ws, ws.numel())
    p = moe.permute(idx.cpu().numpy(), E, S)
    assert np.array_equal(off.cpu().numpy(), p.offsets) and np.array_equal(perm.cpu().numpy(), p.perm)
    y = torch.empty((rows, H), dtype=torch.bfloat16, device="cuda")
    fx.moe_expert_ffn(dev, xq, xs, off, T, y, ws, ws.numel())
    o2 = torch.empty_like(out)
    fx.moe_combine(dev, y, inv, w, T, o2, H)
    assert torch.equal(o2.view(torch.int16), out.view(torch.int16))
    assert fx.moe_get_device_status(dev)[0] == fx.MOE_OK
