"""moe_permute_noalloc: the permutation for callers that cannot allocate
device memory (a runtime whose HBM is all handed to its own pools, a stream
being captured where cudaMalloc is not allowed, a path that cannot afford
cudaMalloc's implicit synchronisation). Its scratch is a library-owned
device array instead of a caller workspace.

Checked through the C ABI against moe_permute (the workspace entry point) on
two calls in a row: a large batch, then a small one, so that state left in
the shared array by the first call would show up in the second. The
permutation's outputs are integer maps and quantised bytes, so the bar is
bit-exact, as for moe_permute against the oracle.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import gen  # noqa: E402

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

import fp8_expert_ffn_b200 as fx  # noqa: E402
from fp8_expert_ffn_b200 import torch_utils as tu  # noqa: E402


def _run_both(dev, sh, x, idx, T):
    rows = T * (sh.K + 1)
    c = "cuda"
    outs = []
    for fn in ("workspace", "noalloc"):
        off = torch.full((sh.E + 2,), -1, dtype=torch.int32, device=c)
        perm = torch.full((rows,), -1, dtype=torch.int32, device=c)
        inv = torch.full((T, sh.K), -1, dtype=torch.int32, device=c)
        xq = torch.zeros((rows, sh.H), dtype=torch.uint8, device=c)
        xs = torch.zeros((sh.HB, rows), dtype=torch.float32, device=c)
        if fn == "workspace":
            ws = tu.workspace(dev, T)
            fx.moe_permute(dev, x, T, sh.H, idx, off, perm, inv, xq, xs, ws, ws.numel())
        else:
            fx.moe_permute_noalloc(dev, x, T, sh.H, idx, off, perm, inv, xq, xs)
        outs.append([t.cpu().numpy() for t in (off, perm, inv, xq, xs)])
    code, bits = fx.moe_get_device_status(dev)
    assert code == fx.MOE_OK, hex(bits)
    return outs


def test_noalloc_permute_matches_workspace_permute_twice():
    wl, layer, _ = gen.workload_inputs("toy")
    sh = layer.shape
    dev = tu.upload_layer(layer)
    ws = tu.workspace(dev, fx.MOE_NOALLOC_MAX_TOKENS)
    for T, seed in ((fx.MOE_NOALLOC_MAX_TOKENS, 21), (37, 22)):   # two calls in a row, large then small
        x = tu.bf16_tensor(gen.make_x(T, sh.H, seed, outliers=2))
        idx = torch.empty((T, sh.K), dtype=torch.int32, device="cuda")
        w = torch.empty((T, sh.K), dtype=torch.float32, device="cuda")
        fx.moe_route(dev, x, T, sh.H, idx, w, None, ws, ws.numel())
        ref, got = _run_both(dev, sh, x, idx, T)
        for name, a, b in zip(("offsets", "perm", "inv", "xq", "xs"), ref, got):
            assert np.array_equal(a.view(np.uint8), b.view(np.uint8)), f"T={T}: {name} differs"


def test_noalloc_permute_full_layer_at_the_size_limit():
    """The 256-expert layer at T = MOE_NOALLOC_MAX_TOKENS: bitmap, prefix
    words and counts of the shared array all at their largest, twice."""
    wl, layer, x_bits = gen.workload_inputs("prefill")
    sh = layer.shape
    T = fx.MOE_NOALLOC_MAX_TOKENS
    assert sh.E == 256 and x_bits.shape[0] >= T
    dev = tu.upload_layer(layer)
    ws = tu.workspace(dev, T)
    for first in (0, 1):    # two calls in a row on different tokens
        x = tu.bf16_tensor(np.ascontiguousarray(np.roll(x_bits, -first, axis=0)[:T]))
        idx = torch.empty((T, sh.K), dtype=torch.int32, device="cuda")
        w = torch.empty((T, sh.K), dtype=torch.float32, device="cuda")
        fx.moe_route(dev, x, T, sh.H, idx, w, None, ws, ws.numel())
        ref, got = _run_both(dev, sh, x, idx, T)
        for name, a, b in zip(("offsets", "perm", "inv", "xq", "xs"), ref, got):
            assert np.array_equal(a.view(np.uint8), b.view(np.uint8)), f"call {first}: {name} differs"
    del dev


def test_noalloc_permute_rejects_too_many_tokens():
    wl, layer, _ = gen.workload_inputs("toy")
    sh = layer.shape
    dev = tu.upload_layer(layer)
    T = fx.MOE_NOALLOC_MAX_TOKENS + 1
    rows = T * (sh.K + 1)
    x = torch.zeros((T, sh.H), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((T, sh.K), dtype=torch.int32, device="cuda")
    off = torch.empty(sh.E + 2, dtype=torch.int32, device="cuda")
    perm = torch.empty(rows, dtype=torch.int32, device="cuda")
    inv = torch.empty((T, sh.K), dtype=torch.int32, device="cuda")
    xq = torch.empty((rows, sh.H), dtype=torch.uint8, device="cuda")
    xs = torch.empty((sh.HB, rows), dtype=torch.float32, device="cuda")
    with pytest.raises(fx.MoeError) as e:
        fx.moe_permute_noalloc(dev, x, T, sh.H, idx, off, perm, inv, xq, xs)
    assert e.value.code == fx.MOE_ERR_UNSUPPORTED
