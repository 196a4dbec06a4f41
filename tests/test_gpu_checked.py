"""The bounds-checked build (libfp8moe_checked.so, -DMOE_CHECKS, loaded with
FP8MOE_CHECKED=1) in a child process: its forward is bit-identical to the
normal build's, and a row index from the inputs that falls outside its
buffer (a corrupted inv given to moe_combine) sets MOE_STATUS_BOUNDS and is
skipped, the other slots combining as before. The corrupted input is only
ever given to the checked build, whose own check turns it into a status."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available() and __name__ != "__main__":
    pytest.skip("needs a GPU", allow_module_level=True)


def _forward_bits(fx, tu, layer, x_bits):
    sh = layer.shape
    dev = tu.upload_layer(layer)
    T = x_bits.shape[0]
    out = torch.empty((T, sh.H), dtype=torch.bfloat16, device="cuda")
    ws = tu.workspace(dev, T)
    fx.moe_layer_forward(dev, tu.bf16_tensor(x_bits), T, sh.H, out, sh.H, ws, ws.numel())
    assert fx.moe_get_device_status(dev)[0] == fx.MOE_OK
    return dev, tu.bf16_bits(out)


def _child(outdir):
    sys.path.insert(0, ROOT)
    import fp8_expert_ffn_b200 as fx
    from fp8_expert_ffn_b200 import torch_utils as tu
    import gen
    assert fx.CHECKED and fx.LIB_PATH.endswith("libfp8moe_checked.so")
    fx.lib()
    torch.cuda.set_device(0)
    wl, layer, x_bits = gen.workload_inputs("toy")
    dev, bits = _forward_bits(fx, tu, layer, x_bits)
    np.save(os.path.join(outdir, "forward.npy"), bits)
    # a combine whose inv points past the y rows: flagged and skipped
    sh, T = layer.shape, x_bits.shape[0]
    rows = T * (sh.K + sh.S)
    x = tu.bf16_tensor(x_bits)
    ws = tu.workspace(dev, T)
    idx = torch.empty((T, sh.K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, sh.K), dtype=torch.float32, device="cuda")
    fx.moe_route(dev, x, T, sh.H, idx, w, None, ws, ws.numel())
    off = torch.empty(sh.E + 2, dtype=torch.int32, device="cuda")
    perm = torch.empty(rows, dtype=torch.int32, device="cuda")
    inv = torch.empty((T, sh.K), dtype=torch.int32, device="cuda")
    xq = torch.empty((rows, sh.H), dtype=torch.uint8, device="cuda")
    xs = torch.empty((sh.HB, rows), dtype=torch.float32, device="cuda")
    fx.moe_permute(dev, x, T, sh.H, idx, off, perm, inv, xq, xs, ws, ws.numel())
    y = torch.empty((rows, sh.H), dtype=torch.bfloat16, device="cuda")
    fx.moe_expert_ffn(dev, xq, xs, off, T, y, ws, ws.numel())
    skipped = inv.clone()
    skipped[3, 1] = -1
    bad = inv.clone()
    bad[3, 1] = rows + 5
    ref = torch.empty((T, sh.H), dtype=torch.bfloat16, device="cuda")
    got = torch.empty_like(ref)
    fx.moe_combine(dev, y, skipped, w, T, ref, sh.H)
    clean = fx.moe_get_device_status(dev)
    fx.moe_combine(dev, y, bad, w, T, got, sh.H)
    flagged = fx.moe_get_device_status(dev)
    res = {"clean": list(clean), "flagged": list(flagged),
           "same": bool(torch.equal(got.view(torch.int16), ref.view(torch.int16)))}
    print(json.dumps(res), flush=True)


def test_checked_build_matches_and_flags_out_of_range_rows(tmp_path):
    import fp8_expert_ffn_b200 as fx
    from fp8_expert_ffn_b200 import build
    from fp8_expert_ffn_b200 import torch_utils as tu
    import gen
    build.build(checked=True)
    env = dict(os.environ, FP8MOE_CHECKED="1")
    r = subprocess.run([sys.executable, os.path.abspath(__file__), "child", str(tmp_path)], env=env, cwd=ROOT,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert res["clean"] == [fx.MOE_OK, 0]
    assert res["flagged"] == [fx.MOE_ERR_DEVICE, 0x20], res
    assert res["same"], "the other slots must combine as with the bad slot skipped"
    wl, layer, x_bits = gen.workload_inputs("toy")
    _, bits = _forward_bits(fx, tu, layer, x_bits)
    assert np.array_equal(np.load(tmp_path / "forward.npy"), bits), "checked build changed the output"


if __name__ == "__main__" and len(sys.argv) > 2 and sys.argv[1] == "child":
    _child(sys.argv[2])
