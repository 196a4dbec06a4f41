"""The two oracles against each other: the numpy one (BLAS-backed FP64
matmuls on dequantised operands) and the plain-loop C++ one (FP64 sums in
index order, E4M3 through its 256-entry table). They share no arithmetic
code, so agreement here pins each against a second, independent reading of
the same definitions: routing indices, permutation maps and every quantised
byte must be identical, FP64 results equal to 1e-12 relative."""
import numpy as np
import pytest

import gen
from oracle import cpp, moe


def _close(a, b, tol=1e-12):
    return np.max(np.abs(a - b)) <= tol * max(np.max(np.abs(a)), 1e-300)


def test_whole_layer_toy():
    _, layer, x = gen.workload_inputs("toy")
    a, b = moe.layer_forward(x, layer), cpp.layer_forward(x, layer)
    assert np.array_equal(a["route"].idx, b["route"].idx)
    assert _close(a["route"].w, b["route"].w) and _close(a["route"].logits, b["route"].logits)
    for f in ("offsets", "perm", "inv"):
        assert np.array_equal(getattr(a["perm"], f), getattr(b["perm"], f))
    for k in ("xq", "xs", "hq", "hs"):
        assert np.array_equal(a[k], b[k]), k
    for k in ("h", "y", "out"):
        assert _close(a[k], b[k]), k


def test_toy_router_variants():
    _, layer, x = gen.workload_inputs("toy")
    rng = np.random.default_rng(3)
    for opts in ({"n_group": 4, "topk_group": 2}, {"bias": rng.uniform(-0.02, 0.02, layer.shape.E)},
                 {"norm_topk": False, "routed_scaling": 2.5}):
        ra = moe.route(x, layer.router_w, layer.shape.K, **opts)
        rb = cpp.route(x, layer.router_w, layer.shape.K, **opts)
        assert np.array_equal(ra.idx, rb.idx) and _close(ra.w, rb.w) and _close(ra.gap, rb.gap, 1e-9)


def test_full_layer_four_decode_tokens():
    """Four tokens of the decode workload through the 256+1-expert layer."""
    _, layer, x = gen.workload_inputs("decode")
    tok = np.array([0, 17, 42, 63])
    ra, rb = moe.route_layer(x[tok], layer), cpp.route_layer(x[tok], layer)
    assert np.array_equal(ra.idx, rb.idx) and _close(ra.w, rb.w)
    qa, sa = moe.quantize_tokens(x[tok])
    qb, sb = cpp.quantize_tokens(x[tok])
    assert np.array_equal(qa, qb) and np.array_equal(sa, sb)
    assert _close(moe.token_outputs(x, layer, tok), cpp.token_outputs(x, layer, tok))


def test_bf16_path_toy():
    _, layer, x = gen.workload_inputs("toy")
    assert _close(moe.layer_forward_bf16(x, layer), cpp.layer_forward_bf16(x, layer))


def test_partial_block_layer_rows():
    """F = 1500-style partial blocks on a small layer: h bytes and y agree."""
    sh = gen.LayerShape(H=256, E=4, K=2, F=250, ld_f=256)
    layer = gen.make_layer(sh, 11)
    x = gen.make_x(40, 256, 3)
    a, b = moe.layer_forward(x, layer), cpp.layer_forward(x, layer)
    assert np.array_equal(a["hq"], b["hq"]) and np.array_equal(a["hs"], b["hs"])
    assert _close(a["out"], b["out"])
