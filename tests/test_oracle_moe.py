"""Pins of the oracle's MoE-layer steps against closed forms, brute force,
invariants and library routines (torch's float8 cast, torch's silu), so that
a dropped term, a wrong sign or index, or a transposed operand in the oracle
fails one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import gen
from oracle import e4m3, moe

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers

def torch_decode(codes) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8))
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def torch_encode(v32: np.ndarray) -> np.ndarray:
    v = np.clip(np.asarray(v32, np.float32), -448, 448)
    return torch.from_numpy(np.ascontiguousarray(v)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def textbook_quant_row(v):
    """One row, groups of 128: fp32 amax/448, fp32 divide, torch's RNE cast."""
    v = np.asarray(v, np.float32)
    codes, scales = [], []
    for g0 in range(0, len(v), 128):
        blk = v[g0:g0 + 128]
        amax = np.float32(max(abs(float(t)) for t in blk))
        s = np.float32(amax / np.float32(448))
        scales.append(s)
        codes.extend([0] * len(blk) if amax == 0 else list(torch_encode(blk / s)))
    return np.array(codes, np.uint8), np.array(scales, np.float32)


def textbook_ffn(x_row_f64, wg, sg, wu, su, wd, sd, F, H):
    """One token through one SwiGLU expert with explicit loops over every index."""
    q, s = textbook_quant_row(x_row_f64.astype(np.float32))
    xd = torch_decode(q)
    a = [xd[k] * float(s[k // 128]) for k in range(H)]
    dg, du, dd = torch_decode(wg), torch_decode(wu), torch_decode(wd)
    h = np.zeros(F)
    for n in range(F):
        g = sum(a[k] * dg[n, k] * float(sg[n // 128, k // 128]) for k in range(H))
        u = sum(a[k] * du[n, k] * float(su[n // 128, k // 128]) for k in range(H))
        h[n] = g / (1.0 + math.exp(-g)) * u
    hq, hs = textbook_quant_row(h.astype(np.float32))
    hd = torch_decode(hq)
    b = [hd[n] * float(hs[n // 128]) for n in range(F)]
    y = np.zeros(H)
    for m in range(H):
        y[m] = sum(b[n] * dd[m, n] * float(sd[m // 128, n // 128]) for n in range(F))
    return y


def small_layer(H=256, E=6, K=2, F=130, ld_f=144, seed=5):
    sh = gen.LayerShape(H=H, E=E, K=K, F=F, ld_f=ld_f)
    return gen.make_layer(sh, seed), sh


# ---------------------------------------------------------------- config

def test_layer_shape_matches_pages(O):
    cfg = json.load(open(os.path.join(GOLDEN, "dots3_text_config.json")))
    s = gen.DOTS3
    assert (s.H, s.E, s.K, s.F) == (cfg["hidden_size"], cfg["n_routed_experts"],
                                    cfg["num_experts_per_tok"], cfg["moe_intermediate_size"])
    assert cfg["shared_experts_intermediate_size"] == s.F and cfg["n_shared_experts"] == 1
    assert cfg["weight_block_size"] == [O.GROUP, O.GROUP]
    assert cfg["routed_scaling_factor"] == 1.0 and cfg["norm_topk_prob"] is True
    assert cfg["hidden_act"] == "silu" and cfg["mlp_bias"] is False


# ---------------------------------------------------------------- quantiser

def test_quantize_matches_textbook_rows(O):
    rng = np.random.default_rng(2)
    v = (rng.standard_normal((5, 300)) * np.exp(rng.uniform(-3, 3, (5, 1)))).astype(np.float32)
    v[1, 128:256] = 0.0                       # an all-zero group
    v[2, 256:] = 0.0; v[2, 299] = -7.5        # partial last group (44 channels)
    q, s = O.quantize_rows(v)
    for r in range(5):
        tq, ts = textbook_quant_row(v[r])
        assert np.array_equal(q[r], tq) and np.array_equal(s[r], ts)
    assert s[1, 1] == 0 and not q[1, 128:256].any()
    assert s[2, 2] == np.float32(np.float32(7.5) / np.float32(448))


def test_quantize_error_bound_and_amax_code(O):
    rng = np.random.default_rng(3)
    v = (rng.standard_normal((64, 512)) * 3).astype(np.float32)
    q, s = O.quantize_rows(v)
    d = O.dequant_rows(q, s)
    # RNE to 3 mantissa bits: |error| <= 2^-4 |value| + half the subnormal step
    bound = np.abs(v) * 2.0 ** -4 + np.repeat(s, 128, axis=1) * 2.0 ** -10 * 1.0001
    assert np.all(np.abs(d - v) <= bound)
    # the amax element of every group lands on +-448
    for g in range(4):
        j = np.argmax(np.abs(v[:, g * 128:(g + 1) * 128]), axis=1) + g * 128
        assert np.all(np.abs(O.e4m3_table()[q[np.arange(64), j]]) == 448.0)


def test_quantize_power_of_two_invariance(O):
    rng = np.random.default_rng(4)
    v = rng.standard_normal((8, 256)).astype(np.float32)
    q0, s0 = O.quantize_rows(v)
    for k in (-20, -3, 5, 30):
        q1, s1 = O.quantize_rows(v * np.float32(2.0 ** k))
        assert np.array_equal(q0, q1)
        assert np.array_equal(s1, s0 * np.float32(2.0 ** k))


# ---------------------------------------------------------------- routing

def test_topk_vs_full_sort_with_ties(O):
    rng = np.random.default_rng(5)
    E, K = 24, 5
    logits = rng.standard_normal((200, E)).round(1)       # many exact ties
    probs = O.softmax(logits)
    idx, w, gap = O.select_topk(probs, K)
    for t in range(200):
        ref = sorted(range(E), key=lambda e: (-probs[t, e], e))
        assert list(idx[t]) == sorted(ref[:K])
        assert gap[t] == probs[t, ref[K - 1]] - probs[t, ref[K]]


def test_route_weights_closed_form(O):
    rng = np.random.default_rng(6)
    logits = rng.standard_normal((50, 32)) * 2
    probs = O.softmax(logits)
    idx, w, _ = O.select_topk(probs, 8)
    assert np.allclose(w.sum(1), 1.0, atol=1e-15)
    sel = np.take_along_axis(logits, idx.astype(np.int64), 1)
    closed = np.exp(sel - sel.max(1, keepdims=True))
    closed /= closed.sum(1, keepdims=True)
    assert np.allclose(w, closed, rtol=1e-13, atol=0)
    assert np.allclose(O.softmax(logits), torch.softmax(torch.from_numpy(logits), 1).numpy(), rtol=1e-14)


def test_route_zero_input(O):
    sh = gen.TOY
    x = np.zeros((4, sh.H), np.uint16)
    r = O.route(x, gen.make_router(sh, 0), sh.K)
    assert np.array_equal(r.idx, np.tile(np.arange(sh.K), (4, 1)))
    assert np.all(r.w == 1.0 / sh.K)


def test_near_tie_flag(O):
    sh = gen.TOY
    router = np.zeros((sh.E, sh.H), np.float32)
    router[:, 0] = np.linspace(1.0, -1.0, sh.E).astype(np.float32)
    router[sh.K, 0] = router[sh.K - 1, 0]                # 4th and 5th exactly tied
    x = np.zeros((2, sh.H), np.uint16)
    x[:, 0] = gen.f32_to_bf16_bits(np.float32([1.0]))[0]
    r = O.route(x, router, sh.K)
    assert r.near_tie.all() and np.all(r.gap == 0)
    assert list(r.idx[0]) == list(range(sh.K))          # tie -> lower id
    router[sh.K, 0] = -1.0
    assert not O.route(x, router, sh.K).near_tie.any()


# ---------------------------------------------------------------- permutation

def brute_permute(idx, E):
    T, K = idx.shape
    counts = [0] * E
    for t in range(T):
        for k in range(K):
            counts[idx[t, k]] += 1
    offsets = [0]
    for e in range(E):
        offsets.append(offsets[-1] + counts[e])
    offsets.append(offsets[-1] + T)
    cursor = offsets[:E]
    perm = [None] * (T * K + T)
    inv = np.zeros((T, K), np.int64)
    for t in range(T):
        for k in range(K):
            e = idx[t, k]
            perm[cursor[e]] = t
            inv[t, k] = cursor[e]
            cursor[e] += 1
    for t in range(T):
        perm[T * K + t] = t
    return np.array(offsets), np.array(perm), inv


def test_permute_vs_brute_and_invariants(O):
    rng = np.random.default_rng(7)
    T, K, E = 123, 4, 16
    idx = np.sort(np.array([rng.choice(E, K, replace=False) for _ in range(T)]), axis=1)
    p = O.permute(idx, E)
    o, pr, iv = brute_permute(idx, E)
    assert np.array_equal(p.offsets, o) and np.array_equal(p.perm, pr) and np.array_equal(p.inv, iv)
    R = T * K
    assert sorted(p.inv.ravel().tolist()) == list(range(R))                 # bijection onto [0, R)
    assert np.all(p.perm[p.inv] == np.arange(T)[:, None])                   # perm o inv = token
    grp = np.searchsorted(p.offsets, p.inv, side="right") - 1
    assert np.array_equal(grp, idx)                                         # row lies in its expert's group
    for e in range(E):
        seg = p.perm[p.offsets[e]:p.offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)                                     # token order inside a group
    assert p.offsets[E] == R and p.offsets[E + 1] == R + T
    assert np.array_equal(p.perm[R:], np.arange(T))


def test_permute_empty_and_all_to_one(O):
    p = O.permute(np.zeros((0, 4), np.int32), 8)
    assert p.offsets.tolist() == [0] * 10 and len(p.perm) == 0
    idx = np.tile(np.array([[3, 5]]), (6, 1))
    p = O.permute(idx, 8)
    assert p.offsets.tolist() == [0, 0, 0, 0, 6, 6, 12, 12, 12, 18]


# ---------------------------------------------------------------- expert FFN

def test_silu_matches_torch(O):
    g = np.linspace(-80, 80, 1001)
    assert np.allclose(O.silu(g), torch.nn.functional.silu(torch.from_numpy(g)).numpy(), rtol=1e-15, atol=1e-300)


def test_expert_ffn_vs_textbook_loops(O):
    layer, sh = small_layer()
    rng = np.random.default_rng(8)
    # scales vary block to block so a transposed scale index shows up
    for name in ("s_gate", "s_up", "s_down"):
        arr = getattr(layer, name)
        arr *= rng.uniform(0.5, 2.0, arr.shape).astype(np.float32)
    x = gen.f32_to_bf16_bits(rng.standard_normal((3, sh.H)).astype(np.float32) * 2)
    xf = O.bf16_to_f64(x)
    e = 4
    tq, ts = O.quantize_tokens(x)
    f = O.expert_ffn_rows(tq, ts, np.array([0] * (e + 1) + [3] * (sh.E + 1 - e)), layer, groups=[e])
    for r in range(3):
        ref = textbook_ffn(xf[r], layer.w_gate[e], layer.s_gate[e], layer.w_up[e], layer.s_up[e],
                           layer.w_down[e], layer.s_down[e], sh.F, sh.H)
        assert np.allclose(f["y"][r], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_gemm_exact_integers(O):
    """Scales 1 and codes with values in {-4..4}: every dot product is an exact integer."""
    rng = np.random.default_rng(9)
    vals = np.array([0x00, 0x38, 0x40, 0x44, 0x48, 0xB8, 0xC0, 0xC4, 0xC8], np.uint8)  # 0,1,2,3,4,-1,-2,-3,-4
    ints = np.array([0, 1, 2, 3, 4, -1, -2, -3, -4])
    ia, ib = rng.integers(0, 9, (7, 384)), rng.integers(0, 9, (200, 384))
    a = O.dequant_rows(vals[ia], np.ones((7, 3), np.float32))
    w = O.dequant_block(vals[ib], np.ones((2, 3), np.float32), 200, 384)
    assert np.array_equal(a @ w.T, (ints[ia] @ ints[ib].T).astype(np.float64))


def test_dequant_block_index_order(O):
    codes = np.full((256, 384), 0x38, np.uint8)           # all 1.0
    s = np.arange(6, dtype=np.float32).reshape(2, 3) + 1  # s[n_blk, k_blk]
    w = O.dequant_block(codes, s, 200, 300)
    assert w[0, 0] == 1 and w[0, 299] == 3 and w[199, 0] == 4 and w[130, 260] == 6


def test_combine_closed_form(O):
    T, K, H = 3, 2, 4
    y = np.arange((T * K + T) * H, dtype=np.float64).reshape(T * K + T, H)
    inv = np.array([[4, 0], [1, 5], [2, 3]])
    w = np.array([[0.25, 0.75], [0.5, 0.5], [1.0, 0.0]])
    out = O.combine(y, inv, w)
    for t in range(T):
        ref = sum(w[t, k] * y[inv[t, k]] for k in range(K)) + y[T * K + t]
        assert np.array_equal(out[t], ref)


# ---------------------------------------------------------------- whole layer

def test_zero_input_gives_zero_output(O, toy):
    _, layer, _ = toy
    x = np.zeros((5, layer.shape.H), np.uint16)
    r = O.layer_forward(x, layer)
    assert np.all(r["out"] == 0.0) and np.all(r["xs"] == 0) and not r["xq"].any()


def test_one_hot_router_selects_one_expert(O, toy):
    _, layer0, x = toy
    sh = layer0.shape
    estar, c0 = 11, 0
    router = np.zeros((sh.E, sh.H), np.float32)
    router[estar, c0] = 200.0
    layer = gen.Layer(sh, router, layer0.w_gate, layer0.s_gate, layer0.w_up, layer0.s_up,
                      layer0.w_down, layer0.s_down)
    xs = x[:3].copy()
    xs[:, c0] = gen.f32_to_bf16_bits(np.float32([1.0]))[0]
    r = O.layer_forward(xs, layer)
    assert np.array_equal(r["route"].idx, np.tile([0, 1, 2, estar], (3, 1)))
    assert np.all(r["route"].w[:, 3] == 1.0) and np.all(r["route"].w[:, :3] < 1e-80)
    xf = O.bf16_to_f64(xs)
    for t in range(3):
        ref = sum(textbook_ffn(xf[t], layer.w_gate[g], layer.s_gate[g], layer.w_up[g], layer.s_up[g],
                               layer.w_down[g], layer.s_down[g], sh.F, sh.H) for g in (estar, sh.E))
        assert np.allclose(r["out"][t], ref, rtol=1e-11, atol=1e-11 * np.abs(ref).max())


def test_permuted_path_equals_direct_per_token(O, toy):
    _, layer, x = toy
    r = O.layer_forward(x, layer)
    d = O.token_outputs(x, layer, np.arange(x.shape[0]))
    assert np.max(np.abs(d - r["out"])) <= 1e-12 * np.max(np.abs(r["out"]))


def test_direct_path_with_bf16_expert_rows_equals_combine_of_rounded_y(toy):
    """token_outputs(y_bf16=True) rounds each expert's output row to bf16
    before weighting it: equal to the permuted path's combine applied to the
    bf16-rounded y rows (the pinned f64 -> bf16 rounding), and different
    from the unrounded sum."""
    from oracle import moe
    _, layer, x = toy
    r = moe.layer_forward(x, layer)
    want = moe.combine(moe.f64_to_bf16_f64(r["y"]), r["perm"].inv, r["route"].w, layer.shape.S)
    got = moe.token_outputs(x, layer, np.arange(x.shape[0]), y_bf16=True)
    assert np.max(np.abs(got - want)) <= 1e-12 * np.max(np.abs(want))
    assert np.max(np.abs(got - r["out"])) > 1e-6 * np.max(np.abs(want))


def test_partial_blocks_equal_zero_padded_layer(O):
    """F=250 (not a multiple of 128) equals the same layer zero-padded to F=256."""
    layer, sh = small_layer(H=256, E=4, K=2, F=250, ld_f=256, seed=11)
    sp = gen.LayerShape(H=256, E=4, K=2, F=256, ld_f=256)
    pad = lambda a, axis: np.concatenate([a, np.zeros(a.shape[:axis] + (256 - a.shape[axis],) + a.shape[axis + 1:], a.dtype)], axis)
    lp = gen.Layer(sp, layer.router_w, pad(layer.w_gate, 1), layer.s_gate, pad(layer.w_up, 1), layer.s_up,
                   layer.w_down.copy(), layer.s_down)
    lp.w_down[:, :, 250:] = 0
    x = gen.make_x(9, 256, 3)
    a, b = O.layer_forward(x, layer)["out"], O.layer_forward(x, lp)["out"]
    assert np.max(np.abs(a - b)) <= 1e-13 * np.max(np.abs(a))
    # the tail scale block was taken over the real rows only
    w = gen.normal_f32(11, gen.STREAM_GATE, 5 * 250 * 256, 1 / 16).reshape(5, 250, 256)
    assert layer.s_gate[2, 1, 0] == np.float32(np.abs(w[2, 128:250, :128]).max() / np.float32(448))


def test_bf16_checkpoint_cross_check(O, toy):
    _, layer, x = toy
    a = O.layer_forward(x, layer)["out"]
    b = O.layer_forward_bf16(x, layer)
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert 1e-4 < rel < 8e-2


def test_no_shared_expert_and_single_expert_layer(O):
    """S = 0: no shared rows; E = 1, K = 1: the layer is that expert's FFN."""
    rng = np.random.default_rng(12)
    idx = np.sort(np.array([rng.choice(8, 2, replace=False) for _ in range(10)]), axis=1)
    p = O.permute(idx, 8, S=0)
    assert p.offsets[8] == p.offsets[9] == 20 and len(p.perm) == 20
    y = rng.standard_normal((20, 3))
    w = rng.uniform(size=(10, 2))
    out = O.combine(y, p.inv, w, S=0)
    assert np.array_equal(out, sum(w[:, k:k + 1] * y[p.inv[:, k]] for k in range(2)))
    sh = gen.LayerShape(H=256, E=1, K=1, F=200, ld_f=208, S=0)
    layer = gen.make_layer(sh, 9)
    assert layer.w_gate.shape[0] == 1
    x = gen.make_x(5, 256, 2)
    r = O.layer_forward(x, layer)
    assert np.all(r["route"].idx == 0) and np.all(r["route"].w == 1.0)
    xf = O.bf16_to_f64(x)
    for t in range(5):
        ref = textbook_ffn(xf[t], layer.w_gate[0], layer.s_gate[0], layer.w_up[0], layer.s_up[0],
                           layer.w_down[0], layer.s_down[0], sh.F, sh.H)
        assert np.allclose(r["out"][t], ref, rtol=1e-11, atol=1e-11 * np.abs(ref).max())


def test_routed_scaling_in_oracle(O):
    sh = gen.TOY
    x = gen.make_x(6, sh.H, 1)
    r1 = O.route(x, gen.make_router(sh, 0), sh.K)
    r2 = O.route(x, gen.make_router(sh, 0), sh.K, routed_scaling=2.5)
    assert np.array_equal(r1.idx, r2.idx) and np.allclose(r2.w, 2.5 * r1.w, rtol=1e-15)


# ----------------------------------------------------------------------------- router variants

def test_group_limited_hand_example(O):
    """8 experts in 4 groups of 2, two groups eligible, top-3 (worked by hand):
    group maxima 0.30, 0.20, 0.03, 0.25 keep groups 0 and 3, so expert 2
    (0.20, group 1) loses to expert 6 (0.04); ungrouped the top-3 is 0, 2, 7."""
    p = np.array([[0.30, 0.01, 0.20, 0.15, 0.02, 0.03, 0.04, 0.25]])
    idx, w, gap = O.select_topk(p, 3, n_group=4, topk_group=2)
    assert idx.tolist() == [[0, 6, 7]]
    np.testing.assert_allclose(w[0], np.array([0.30, 0.04, 0.25]) / 0.59, rtol=1e-15)
    assert gap[0] == pytest.approx(min(0.04 - 0.01, 0.25 - 0.20))
    idx0, _, _ = O.select_topk(p, 3)
    assert idx0.tolist() == [[0, 2, 7]]


def test_group_limited_reduces_to_ungrouped(O):
    rng = np.random.default_rng(21)
    p = rng.dirichlet(np.ones(16), size=64)
    ref = O.select_topk(p, 4)
    # every group eligible
    got = O.select_topk(p, 4, n_group=4, topk_group=4)
    assert np.array_equal(got[0], ref[0]) and np.allclose(got[1], ref[1])
    # one expert per group, K groups eligible: the K best experts
    got = O.select_topk(p, 4, n_group=16, topk_group=4)
    assert np.array_equal(got[0], ref[0]) and np.allclose(got[1], ref[1])


def test_group_limited_properties(O):
    """Checked on the output only: at most topk_group groups are used, every
    dropped group's best member is no better than every kept group's, and no
    eligible expert left out beats a selected one."""
    rng = np.random.default_rng(22)
    E, G, TG, K = 64, 8, 3, 6
    p = rng.dirichlet(np.ones(E) * 0.3, size=200)
    idx, w, _ = O.select_topk(p, K, n_group=G, topk_group=TG)
    gs = E // G
    for t in range(len(p)):
        used = set(int(e) // gs for e in idx[t])
        assert len(used) <= TG
        gmax = p[t].reshape(G, gs).max(axis=1)
        # the kept groups: the used ones plus (if fewer) the next best
        kept = sorted(range(G), key=lambda g: (-gmax[g], g))[:TG]
        assert used <= set(kept)
        for g in set(range(G)) - set(kept):
            assert gmax[g] <= min(gmax[k] for k in kept)
        elig = [e for e in range(E) if e // gs in kept]
        left = [e for e in elig if e not in idx[t]]
        assert max(p[t, left]) <= min(p[t, idx[t]])
        assert w[t].sum() == pytest.approx(1.0)


def test_selection_bias_selects_but_does_not_weight(O):
    rng = np.random.default_rng(23)
    E, K = 32, 4
    logits = rng.normal(0, 1, (50, E))
    p = np.exp(logits - logits.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    ref = O.select_topk(p, K)
    # a constant bias changes nothing
    got = O.select_topk(p, K, bias=np.full(E, 0.7))
    assert np.array_equal(got[0], ref[0]) and np.allclose(got[1], ref[1], rtol=1e-14)
    # a large negative bias removes an expert, a large positive one forces one in
    b = np.zeros(E)
    b[5] = -1000.0
    b[9] = 1000.0
    idx, w, _ = O.select_topk(p, K, bias=b)
    assert (idx != 5).all() and (idx == 9).any(axis=1).all()
    for t in range(len(p)):
        # the weights are the unbiased probabilities of the selected experts,
        # renormalised (softmax of their logits)
        sel = idx[t]
        ex = np.exp(logits[t, sel] - logits[t, sel].max())
        np.testing.assert_allclose(w[t], ex / ex.sum(), rtol=1e-12)


def test_norm_topk_off_keeps_the_softmax_weights(O):
    import scipy.special
    rng = np.random.default_rng(24)
    sh = gen.TOY
    x = gen.make_x(9, sh.H, 2)
    router = gen.make_router(sh, 0)
    r = O.route(x, router, sh.K, routed_scaling=2.0, norm_topk=False)
    full = scipy.special.softmax(O.bf16_to_f64(x) @ router.astype(np.float64).T, axis=1)
    np.testing.assert_allclose(r.w, 2.0 * np.take_along_axis(full, r.idx.astype(np.int64), 1), rtol=1e-12)
    assert (r.w.sum(1) < 2.0).all()
    r1 = O.route(x, router, sh.K)
    assert np.array_equal(r.idx, r1.idx)


def test_route_layer_reads_the_layer_options(O):
    sh = gen.TOY
    x = gen.make_x(10, sh.H, 1)
    wl, layer, _ = gen.workload_inputs("toy")
    a = O.route_layer(x, layer)
    b = O.route(x, layer.router_w, sh.K)
    assert np.array_equal(a.idx, b.idx) and np.array_equal(a.w, b.w)


# ----------------------------------------------------------------------------- BF16 cross-check path

def _torch_bf16_via_f32(v64: np.ndarray) -> np.ndarray:
    """torch's own casts, f64 -> f32 -> bf16 (each round to nearest even), back to f64."""
    t = torch.from_numpy(np.ascontiguousarray(v64, np.float64))
    return t.to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()


def test_bf16_rounding_matches_torch_cast_bit_for_bit(O):
    """f64_to_bf16_f64 against torch's cast on a stride sweep of every finite
    fp32 bit pattern, every tie pattern (low half 0x8000, both parities of the
    kept last bit), the patterns one below and one above each tie, subnormals
    and the values that round up to infinity. A truncating cast, or one that
    breaks ties away from zero, fails the tie and round-up cases."""
    sweep = np.arange(0, 0x7F800000, 4099, dtype=np.uint64).astype(np.uint32)
    hi = (np.arange(0, 0x7F80, 37, dtype=np.uint32) << 16)
    ties = np.concatenate([hi | 0x8000, (hi | 0x10000) | 0x8000])            # even and odd kept bit
    near = np.concatenate([ties - 1, ties + 1])
    sub = np.arange(1, 0x00800000, 997, dtype=np.uint32)                      # fp32 subnormals
    top = np.arange(0x7F7F0000, 0x7F800000, 97, dtype=np.uint32)              # includes round-up to inf
    bits = np.concatenate([sweep, ties, near, sub, top])
    bits = np.concatenate([bits, bits | 0x80000000])                          # both signs
    v32 = bits.view(np.float32)
    got = O.f64_to_bf16_f64(v32.astype(np.float64))
    want = _torch_bf16_via_f32(v32.astype(np.float64))
    assert np.array_equal(got.view(np.uint64), want.view(np.uint64))
    # ties go to the even bf16 mantissa: 1 + 2^-8 -> 1, 1 + 3 * 2^-8 -> 1 + 2^-6
    assert O.f64_to_bf16_f64(np.array([1 + 2.0 ** -8]))[0] == 1.0
    assert O.f64_to_bf16_f64(np.array([1 + 3 * 2.0 ** -8]))[0] == 1 + 2.0 ** -6
    # f64 values between fp32 numbers are rounded to fp32 first (the checkpoint's fp32 dequantisation)
    rng = np.random.default_rng(31)
    v64 = rng.standard_normal(20000) * np.exp(rng.uniform(-30, 30, 20000))
    assert np.array_equal(O.f64_to_bf16_f64(v64).view(np.uint64), _torch_bf16_via_f32(v64).view(np.uint64))


def _bf16_weight(codes, scales, n, k):
    """W[n', k'] = bf16(fp32(decode(codes) * scale of its 128 x 128 block)) with explicit indices."""
    d = torch_decode(codes)
    w = np.zeros((n, k))
    for i in range(n):
        for j in range(k):
            p = np.float32(np.float32(d[i, j]) * np.float32(scales[i // 128, j // 128]))
            w[i, j] = float(torch.tensor(float(p), dtype=torch.float32).to(torch.bfloat16).item())
    return w


def test_bf16_layer_path_vs_textbook_loops(O):
    """layer_forward_bf16 against loops over every index: weights bf16(q s),
    no activation or h quantisation, FP64 sums, shared expert added with 1."""
    layer, sh = small_layer(H=256, E=4, K=2, F=130, ld_f=144, seed=21)
    rng = np.random.default_rng(22)
    for name in ("s_gate", "s_up", "s_down"):
        arr = getattr(layer, name)
        arr *= rng.uniform(0.5, 2.0, arr.shape).astype(np.float32)
    x = gen.f32_to_bf16_bits(rng.standard_normal((3, sh.H)).astype(np.float32))
    got = O.layer_forward_bf16(x, layer)
    r = O.route_layer(x, layer)
    xf = O.bf16_to_f64(x)
    Wg = [_bf16_weight(layer.w_gate[g], layer.s_gate[g], sh.F, sh.H) for g in range(sh.E + 1)]
    Wu = [_bf16_weight(layer.w_up[g], layer.s_up[g], sh.F, sh.H) for g in range(sh.E + 1)]
    Wd = [_bf16_weight(layer.w_down[g], layer.s_down[g], sh.H, sh.F) for g in range(sh.E + 1)]
    for t in range(3):
        ref = np.zeros(sh.H)
        for g, wt in [(int(r.idx[t, k]), float(r.w[t, k])) for k in range(sh.K)] + [(sh.E, 1.0)]:
            h = np.zeros(sh.F)
            for n in range(sh.F):
                gsum = sum(xf[t, k] * Wg[g][n, k] for k in range(sh.H))
                usum = sum(xf[t, k] * Wu[g][n, k] for k in range(sh.H))
                h[n] = gsum / (1.0 + math.exp(-gsum)) * usum
            for m in range(sh.H):
                ref[m] += wt * sum(h[n] * Wd[g][m, n] for n in range(sh.F))
        assert np.allclose(got[t], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_expert_down_rows_vs_textbook_loops(O):
    """expert_down_rows over a multi-group offset vector (with empty groups and
    a partial F block): each row uses its own group's down weights and scales."""
    layer, sh = small_layer(H=256, E=5, K=2, F=130, ld_f=144, seed=23)
    rng = np.random.default_rng(24)
    layer.s_down *= rng.uniform(0.5, 2.0, layer.s_down.shape).astype(np.float32)
    counts = np.array([2, 0, 3, 1, 0, 2])                # groups 0..E (E = shared)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rows = int(off[-1])
    hq = rng.integers(0, 256, (rows, sh.F)).astype(np.uint8)
    hq[(hq & 0x7F) == 0x7F] = 0x3C                       # no NaN codes
    hs = rng.uniform(0.01, 0.1, (rows, sh.FB)).astype(np.float32)
    y = O.expert_down_rows(hq, hs, off, layer)
    hd = torch_decode(hq)
    for r in range(rows):
        g = int(np.searchsorted(off, r, side="right") - 1)
        dd = torch_decode(layer.w_down[g])
        sd = layer.s_down[g]
        ref = np.array([sum(hd[r, n] * float(hs[r, n // 128]) * dd[m, n] * float(sd[m // 128, n // 128])
                            for n in range(sh.F)) for m in range(sh.H)])
        assert np.allclose(y[r], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max()), f"row {r} (group {g})"
