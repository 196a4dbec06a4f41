"""Parity of the CUDA path (through the C ABI) with the FP64 oracle.

Each stage is checked with teacher forcing: the oracle gets the GPU's own
upstream outputs. Routing indices, permutation maps and quantised activation
bytes must match bit-exactly (tokens whose top-K gap is below 1e-6 are
excluded from the routing comparison); the layer output must be within
relative Frobenius 5e-3 and max-abs 2e-2 * rms of the oracle.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import gen  # noqa: E402
from oracle import moe  # noqa: E402

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines, never run there
    pytest.skip("needs a GPU", allow_module_level=True)

import fp8_expert_ffn_b200 as fx  # noqa: E402
from fp8_expert_ffn_b200 import torch_utils as tu  # noqa: E402
import gpu_case as gc  # noqa: E402

RNG = np.random.default_rng(1234)


# ----------------------------------------------------------------------------- fixtures

_cases = {}


def get_case(name):
    if name not in _cases:
        wl, layer, x = gen.workload_inputs(name)
        dev = _device_layers.get((wl.shape, wl.w_seed, wl.zipf))
        if dev is None:
            same_experts = [d for (s, w, z), d in _device_layers.items() if (s, w) == (wl.shape, wl.w_seed)]
            dev = tu.upload_layer(layer, share_experts=same_experts[0] if same_experts else None)
            _device_layers[(wl.shape, wl.w_seed, wl.zipf)] = dev
        _cases[name] = (wl, layer, gc.Case(layer, x, dev))
    return _cases[name]


_device_layers = {}

FULL = ["toy", "toy_t2048", "decode", "dense"]   # every token / row checked
SAMPLED = ["prefill", "zipf", "edge", "edge_f1500", "vision"]
ALL = FULL + SAMPLED


def token_sample(T, n):
    if T <= n:
        return np.arange(T)
    s = RNG.choice(T, n, replace=False)
    return np.sort(np.concatenate([s, [0, T - 1]]))


# ----------------------------------------------------------------------------- routing

@pytest.mark.parametrize("name", ALL)
def test_route(name):
    wl, layer, c = get_case(name)
    r = moe.route(c.x_bits, layer.router_w, layer.shape.K)
    keep = ~r.near_tie
    idx = c.np("idx")
    assert np.array_equal(idx[keep], r.idx[keep]), \
        f"{np.sum(np.any(idx[keep] != r.idx[keep], axis=1))} unflagged tokens routed differently"
    w = c.np("w")
    assert np.allclose(w[keep], r.w[keep], rtol=2e-5, atol=1e-6)
    assert np.allclose(w.sum(1), 1.0, atol=2e-6)
    lg = c.np("logits")
    assert np.max(np.abs(lg - r.logits)) <= 1e-4 * max(1.0, np.abs(r.logits).max())


# ----------------------------------------------------------------------------- permutation

@pytest.mark.parametrize("name", ALL)
def test_permute(name):
    wl, layer, c = get_case(name)
    sh, T = layer.shape, c.T
    p = moe.permute(c.np("idx"), sh.E, sh.S)
    assert np.array_equal(c.np("offsets"), p.offsets)
    assert np.array_equal(c.np("perm"), p.perm)
    assert np.array_equal(c.np("inv"), p.inv)
    tq, ts = moe.quantize_tokens(c.x_bits)
    perm = p.perm
    rows = np.arange(c.rows) if name in FULL else np.sort(RNG.choice(c.rows, min(c.rows, 8192), replace=False))
    xq = c.xq[torch.from_numpy(rows).cuda()].cpu().numpy()
    assert np.array_equal(xq, tq[perm[rows]]), "quantised activation bytes differ"
    xs = c.np("xs")[:, rows].T
    assert np.array_equal(xs.view(np.uint32), ts[perm[rows]].view(np.uint32)), "activation scales differ"


# ----------------------------------------------------------------------------- expert FFN

@pytest.mark.parametrize("name", ALL)
def test_expert_ffn(name):
    wl, layer, c = get_case(name)
    sh, T = layer.shape, c.T
    toks = np.arange(T) if name in FULL else token_sample(T, 40)
    rows = np.unique(gc.rows_of_tokens(c.np("inv"), T, sh.K, toks, sh.S))
    off = c.np("offsets")
    xq = c.xq[torch.from_numpy(rows).cuda()].cpu().numpy()
    xs = c.np("xs")[:, rows].T.copy()
    ref = gc.oracle_ffn_on_rows(layer, np.arange(len(rows)), xq, xs,
                                np.searchsorted(rows, off).astype(np.int64))
    # h bytes: not gated bit-exactly (FP32 vs FP64 accumulation), but nearly all
    # equal and the rest one E4M3 step away
    hq = c.hq[torch.from_numpy(rows).cuda()].cpu().numpy()[:, :sh.F]
    match = np.mean(hq == ref["hq"])
    assert match >= 0.995, f"h code match {match:.5f}"
    assert gc.e4m3_step_diff(hq, ref["hq"]).max() <= 1
    # y against the oracle fed with the GPU's h (teacher forcing of the down GEMM)
    hs = c.hs.cpu().numpy()[:, rows].T.copy()
    E1 = sh.E + 1
    groups = np.searchsorted(off, rows, side="right") - 1
    sub_off = np.zeros(E1 + 1, np.int64)
    sub_off[1:] = np.cumsum(np.bincount(groups, minlength=E1)[:E1])
    y_tf = moe.expert_down_rows(hq, hs, sub_off, layer, groups=np.unique(groups))
    y = tu.bf16_bits(c.y[torch.from_numpy(rows).cuda()])
    yg = moe.bf16_to_f64(y)
    rms = np.sqrt(np.mean(y_tf ** 2))
    assert np.all(np.abs(yg - y_tf) <= 2.0 ** -8 * np.abs(y_tf) + 1e-4 * rms), "y differs beyond bf16 rounding"
    # and against the oracle's own h
    gc.assert_output_close(yg, ref["y"], f"{name}: y")


# ----------------------------------------------------------------------------- combine and layer

@pytest.mark.parametrize("name", ALL)
def test_combine(name):
    wl, layer, c = get_case(name)
    T = c.T
    toks = np.arange(T) if name in FULL else token_sample(T, 2048)
    y = moe.bf16_to_f64(tu.bf16_bits(c.y))
    ref = moe.combine(y, c.np("inv"), c.np("w").astype(np.float64), layer.shape.S)[toks]
    out = moe.bf16_to_f64(c.np("out"))[toks]
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.all(np.abs(out - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5 * rms)


@pytest.mark.parametrize("name", ALL)
def test_layer_end_to_end(name):
    wl, layer, c = get_case(name)
    T = c.T
    toks = np.arange(T) if name in FULL else token_sample(T, 48)
    r = moe.route(c.x_bits[toks], layer.router_w, layer.shape.K)
    keep = toks[~r.near_tie]
    ref = moe.token_outputs(c.x_bits, layer, keep)
    out = moe.bf16_to_f64(c.np("out"))[keep]
    gc.assert_output_close(out, ref, f"{name}: layer output")
    # the composed entry points give the same bytes as the stage calls
    ws = tu.workspace(c.dev, T)
    o2 = torch.empty_like(c.out)
    fx.moe_layer_forward(c.dev, c.x, T, layer.shape.H, o2, layer.shape.H, ws, ws.numel())
    assert torch.equal(o2.view(torch.int16), c.out.view(torch.int16))
    y2 = torch.empty_like(c.y)
    fx.moe_expert_ffn(c.dev, c.xq, c.xs, c.offsets, T, y2, ws, ws.numel())
    assert torch.equal(y2.view(torch.int16), c.y.view(torch.int16))


def _check_rows_teacher_forced(name, rows):
    """h codes against the oracle fed the GPU's xq/xs, and y against the
    oracle fed the GPU's h, on every one of the given permuted rows."""
    wl, layer, c = get_case(name)
    sh = layer.shape
    rows = np.unique(rows)
    off = c.np("offsets")
    rt = torch.from_numpy(rows).cuda()
    xq = c.xq[rt].cpu().numpy()
    xs = c.np("xs")[:, rows].T.copy()
    ref = gc.oracle_ffn_on_rows(layer, np.arange(len(rows)), xq, xs, np.searchsorted(rows, off).astype(np.int64))
    hq = c.hq[rt].cpu().numpy()[:, :sh.F]
    match = np.mean(hq == ref["hq"])
    assert match >= 0.995, f"{name}: h code match {match:.5f} over {len(rows)} rows"
    assert gc.e4m3_step_diff(hq, ref["hq"]).max() <= 1
    hs = c.hs.cpu().numpy()[:, rows].T.copy()
    E1 = sh.E + 1
    groups = np.searchsorted(off, rows, side="right") - 1
    sub_off = np.zeros(E1 + 1, np.int64)
    sub_off[1:] = np.cumsum(np.bincount(groups, minlength=E1)[:E1])
    y_tf = moe.expert_down_rows(hq, hs, sub_off, layer, groups=np.unique(groups))
    yg = moe.bf16_to_f64(tu.bf16_bits(c.y[rt]))
    rms = np.sqrt(np.mean(y_tf ** 2))
    bad = np.abs(yg - y_tf) > 2.0 ** -8 * np.abs(y_tf) + 1e-4 * rms
    assert not bad.any(), f"{name}: y differs beyond bf16 rounding on {np.unique(np.nonzero(bad)[0]).size} rows"


def test_zipf_hottest_group_and_partial_tiles_every_row():
    """Long prefill with Zipf routing, full size: every row of the busiest
    expert's group (about 40 row tiles, several chunks of the tile order) and
    every row of every group's partial last tile (the rows the GEMM epilogues
    store without the bulk tensor path) -- h codes and y, teacher forced."""
    wl, layer, c = get_case("zipf")
    off = c.np("offsets").astype(np.int64)
    counts = np.diff(off)[:layer.shape.E]
    hot = int(np.argmax(counts))
    rows = [np.arange(off[hot], off[hot + 1])]
    for g in range(layer.shape.E + 1):
        n = off[g + 1] - off[g]
        if n % 128:
            rows.append(np.arange(off[g] + (n // 128) * 128, off[g + 1]))
    rows = np.concatenate(rows)
    assert counts[hot] >= 10 * 128 and len(rows) > counts[hot] + 1000
    _check_rows_teacher_forced("zipf", rows)


def test_edge_last_tokens_end_to_end():
    """The last 3 tokens of the ragged T=4099 batch (beyond the last full
    128-token block), end to end against the oracle."""
    wl, layer, c = get_case("edge")
    toks = np.arange(c.T - 3, c.T)
    r = moe.route(c.x_bits[toks], layer.router_w, layer.shape.K)
    keep = toks[~r.near_tie]
    assert len(keep) >= 2
    ref = moe.token_outputs(c.x_bits, layer, keep)
    gc.assert_output_close(moe.bf16_to_f64(c.np("out"))[keep], ref, "edge: last tokens")
    rows = gc.rows_of_tokens(c.np("inv"), c.T, layer.shape.K, toks, layer.shape.S)
    _check_rows_teacher_forced("edge", rows)


def test_bf16_checkpoint_cross_check():
    """FP8 path vs the oracle's BF16-weight path (no activation quantisation)
    on the F=1500 variant: catches a wrong dequantisation (scale index or
    partial block) that both FP8 paths could share."""
    wl, layer, c = get_case("edge_f1500")
    toks = token_sample(c.T, 24)
    r = moe.route(c.x_bits[toks], layer.router_w, layer.shape.K)
    keep = toks[~r.near_tie]
    ref = moe.layer_forward_bf16(c.x_bits, layer, tokens=keep)
    out = moe.bf16_to_f64(c.np("out"))[keep]
    rel = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert rel < 8e-2, rel


# ----------------------------------------------------------------------------- GEMM promotion

def _integer_layer():
    """Toy-shaped layer whose codes decode to integers in [-4, 4] with every
    scale 1: all products and sums are exact in FP32."""
    sh = gen.TOY
    rng = np.random.default_rng(7)
    vals = np.array([0x00, 0x38, 0x40, 0x44, 0x48, 0xB8, 0xC0, 0xC4, 0xC8], np.uint8)
    pick = lambda shape: vals[rng.integers(0, 9, shape)]
    E1 = sh.E + 1
    return gen.Layer(sh, gen.make_router(sh, 0), pick((E1, sh.F, sh.H)), np.ones((E1, sh.FB, sh.HB), np.float32),
                     pick((E1, sh.F, sh.H)), np.ones((E1, sh.FB, sh.HB), np.float32),
                     pick((E1, sh.H, sh.ld_f)), np.ones((E1, sh.HB, sh.FB), np.float32)), vals


def _group_offsets(sh, T, rng):
    rows = T * (sh.K + 1)
    sizes = np.zeros(sh.E + 1, np.int64)
    sizes[3] = 150          # two row tiles
    sizes[0] = 0            # empty groups
    rest = rows - sizes.sum()
    cuts = np.sort(rng.choice(rest + 1, sh.E - 2, replace=True))
    parts = np.diff(np.concatenate([[0], cuts, [rest]]))
    sizes[[g for g in range(sh.E + 1) if g not in (0, 3)]] = parts
    off = np.zeros(sh.E + 2, np.int64)
    off[1:] = np.cumsum(sizes)
    return off.astype(np.int32)


# T = 60: groups of up to two row tiles; T = 1000: groups of several row
# tiles (chunks of the tile order, partial last tiles)
@pytest.mark.parametrize("T", [60, 1000])
@pytest.mark.parametrize("which", [0, 1])
def test_grouped_gemm_exact_integers(which, T):
    layer, vals = _integer_layer()
    sh = layer.shape
    dev = tu.upload_layer(layer)
    rng = np.random.default_rng(3 + which)
    rows = T * (sh.K + 1)
    off = _group_offsets(sh, T, rng)
    Kdim = sh.H if which == 0 else sh.FB * 128
    a = vals[rng.integers(0, 9, (rows, Kdim))]
    nkb = Kdim // 128
    a_s = np.ones((nkb, rows), np.float32)
    ncols = 2 * sh.FB * 128 if which == 0 else sh.H
    out = torch.full((rows, ncols), float("nan"), device="cuda")
    fx.moe_test_grouped_gemm_f32(dev, which, tu.to_device(a), tu.to_device(a_s), tu.to_device(off), T, out)
    got = out.cpu().numpy().astype(np.float64)
    ints = moe.e4m3.decode(np.arange(256, dtype=np.uint8))
    A = ints[a].astype(np.int64)
    for g in range(sh.E + 1):
        r0, r1 = off[g], off[g + 1]
        if r0 == r1:
            continue
        if which == 0:
            Wg = ints[layer.w_gate[g]].astype(np.int64)
            Wu = ints[layer.w_up[g]].astype(np.int64)
            G, U = A[r0:r1] @ Wg.T, A[r0:r1] @ Wu.T
            for cb in range(sh.FB):
                assert np.array_equal(got[r0:r1, cb * 256:cb * 256 + 128], G[:, cb * 128:(cb + 1) * 128])
                assert np.array_equal(got[r0:r1, cb * 256 + 128:cb * 256 + 256], U[:, cb * 128:(cb + 1) * 128])
        else:
            Wd = ints[layer.w_down[g][:, :sh.F]].astype(np.int64)
            assert np.array_equal(got[r0:r1], A[r0:r1, :sh.F] @ Wd.T)


@pytest.mark.parametrize("T", [60, 1000])
@pytest.mark.parametrize("which", [0, 1])
def test_grouped_gemm_promotion_random_scales(which, T):
    """Non-uniform scales: a transposed or shifted scale index would show."""
    wl, layer0, _ = gen.workload_inputs("toy")
    sh = layer0.shape
    rng = np.random.default_rng(11 + which)
    layer = gen.Layer(sh, layer0.router_w, layer0.w_gate, layer0.s_gate * rng.uniform(0.25, 4, layer0.s_gate.shape)
                      .astype(np.float32), layer0.w_up, layer0.s_up, layer0.w_down,
                      layer0.s_down * rng.uniform(0.25, 4, layer0.s_down.shape).astype(np.float32))
    dev = tu.upload_layer(layer)
    rows = T * (sh.K + 1)
    off = _group_offsets(sh, T, rng)
    Kdim = sh.H if which == 0 else sh.FB * 128
    a = rng.integers(0, 256, (rows, Kdim)).astype(np.uint8)
    a[(a & 0x7F) == 0x7F] = 0x30     # no NaN codes
    nkb = Kdim // 128
    a_s = rng.uniform(0.001, 0.1, (nkb, rows)).astype(np.float32)
    ncols = 2 * sh.FB * 128 if which == 0 else sh.H
    out = torch.zeros((rows, ncols), device="cuda")
    fx.moe_test_grouped_gemm_f32(dev, which, tu.to_device(a), tu.to_device(a_s), tu.to_device(off), T, out)
    got = out.cpu().numpy().astype(np.float64)
    A = moe.dequant_rows(a, a_s.T.copy())
    for g in range(sh.E + 1):
        r0, r1 = off[g], off[g + 1]
        if r0 == r1:
            continue
        if which == 0:
            G = A[r0:r1] @ moe.dequant_block(layer.w_gate[g], layer.s_gate[g], sh.F, sh.H).T
            U = A[r0:r1] @ moe.dequant_block(layer.w_up[g], layer.s_up[g], sh.F, sh.H).T
            ref = np.concatenate([np.concatenate([G[:, cb * 128:(cb + 1) * 128], U[:, cb * 128:(cb + 1) * 128]], 1)
                                  for cb in range(sh.FB)], 1)
        else:
            ref = A[r0:r1, :sh.F] @ moe.dequant_block(layer.w_down[g], layer.s_down[g], sh.H, sh.F).T
        err = np.abs(got[r0:r1] - ref)
        assert err.max() <= 1e-5 * np.abs(ref).max() + 1e-30, (g, err.max(), np.abs(ref).max())


# ----------------------------------------------------------------------------- special inputs

def test_zero_input_exact_zero_output():
    wl, layer, _ = gen.workload_inputs("toy")
    x = np.zeros((17, layer.shape.H), np.uint16)
    c = gc.Case(layer, x)
    assert np.array_equal(c.np("idx"), np.tile(np.arange(layer.shape.K), (17, 1)))
    assert np.all(c.np("w") == np.float32(1.0 / layer.shape.K))
    assert not c.np("out").any()                  # +0 everywhere


def test_one_hot_router():
    wl, layer0, x = gen.workload_inputs("toy")
    sh = layer0.shape
    estar = 11
    router = np.zeros((sh.E, sh.H), np.float32)
    router[estar, 0] = 200.0
    layer = gen.Layer(sh, router, layer0.w_gate, layer0.s_gate, layer0.w_up, layer0.s_up, layer0.w_down,
                      layer0.s_down)
    xs = x.copy()
    xs[:, 0] = gen.f32_to_bf16_bits(np.float32([1.0]))[0]
    c = gc.Case(layer, xs)
    assert np.array_equal(c.np("idx"), np.tile([0, 1, 2, estar], (xs.shape[0], 1)))
    assert np.all(c.np("w") == np.float32([0, 0, 0, 1]))
    ref = moe.layer_forward(xs, layer)["out"]
    gc.assert_output_close(moe.bf16_to_f64(c.np("out")), ref, "one-hot router")
    c2 = gc.Case(layer, xs, c.dev)
    assert np.array_equal(c.np("out"), c2.np("out"))


def test_batch_invariance_ragged_tail():
    """The first 4096 tokens of the T=4099 run equal a T=4096 run bit for bit."""
    wl, layer, c = get_case("edge")
    c2 = gc.Case(layer, c.x_bits[:4096], c.dev)
    assert np.array_equal(c.np("out")[:4096], c2.np("out"))


def test_partial_blocks_equal_zero_padded_layer():
    """FFN 1500 (partial 128x128 blocks) equals the same layer zero-padded to 1536."""
    wl, layer, c = get_case("edge_f1500")
    sh = layer.shape
    sp = gen.LayerShape(H=sh.H, E=sh.E, K=sh.K, F=1536, ld_f=1536)
    pad = np.zeros((sh.E + 1, 36, sh.H), np.uint8)
    lp = gen.Layer(sp, layer.router_w, np.concatenate([layer.w_gate, pad], 1), layer.s_gate,
                   np.concatenate([layer.w_up, pad], 1), layer.s_up, layer.w_down, layer.s_down)
    assert not lp.w_down[:, :, 1500:].any()
    x = c.x_bits[:512]
    a = gc.Case(layer, x, c.dev)
    b = gc.Case(lp, x)
    assert np.array_equal(a.np("out"), b.np("out"))
    del b


# ----------------------------------------------------------------------------- errors

def test_bad_expert_ids_set_device_status():
    wl, layer, c = get_case("toy")
    sh, T = layer.shape, 8
    idx = torch.tensor(np.tile(np.arange(sh.K), (T, 1)), dtype=torch.int32, device="cuda")
    idx[2, 1] = sh.E            # out of range
    idx[5, 3] = idx[5, 0]       # repeated within a token
    rows = T * (sh.K + 1)
    off = torch.empty(sh.E + 2, dtype=torch.int32, device="cuda")
    perm = torch.full((rows,), -7, dtype=torch.int32, device="cuda")
    inv = torch.empty((T, sh.K), dtype=torch.int32, device="cuda")
    xq = torch.empty((rows, sh.H), dtype=torch.uint8, device="cuda")
    xs = torch.empty((sh.HB, rows), dtype=torch.float32, device="cuda")
    ws = tu.workspace(c.dev, T)
    fx.moe_permute(c.dev, c.x[:T], T, sh.H, idx, off, perm, inv, xq, xs, ws, ws.numel())
    code, bits = fx.moe_get_device_status(c.dev)
    assert code == fx.MOE_ERR_DEVICE and bits & 1 and bits & 2
    assert inv[2, 1].item() == -1 and inv[5, 3].item() == -1
    code, bits = fx.moe_get_device_status(c.dev)   # cleared by the read
    assert code == fx.MOE_OK and bits == 0


def test_host_validation():
    wl, layer, c = get_case("toy")
    sh = layer.shape
    T = 4
    ws = tu.workspace(c.dev, T)
    out = torch.empty((T, sh.H), dtype=torch.bfloat16, device="cuda")
    xmis = torch.empty(T * sh.H + 8, dtype=torch.bfloat16, device="cuda")[1:1 + T * sh.H]
    with pytest.raises(fx.MoeError) as e:
        fx.moe_layer_forward(c.dev, xmis, T, sh.H, out, sh.H, ws, ws.numel())
    assert e.value.code == fx.MOE_ERR_MISALIGNED
    with pytest.raises(fx.MoeError) as e:
        fx.moe_layer_forward(c.dev, c.x, T, sh.H, out, sh.H, ws, ws.numel() - 256)
    assert e.value.code == fx.MOE_ERR_WORKSPACE
    with pytest.raises(fx.MoeError) as e:
        fx.moe_layer_forward(c.dev, c.x, T, sh.H - 8, out, sh.H, ws, ws.numel())
    assert e.value.code == fx.MOE_ERR_INVALID_ARG
    fx.moe_layer_forward(c.dev, c.x, 0, sh.H, out, sh.H, ws, ws.numel())   # T = 0: no-op


def test_forward_is_deterministic():
    wl, layer, c = get_case("prefill")
    ws = tu.workspace(c.dev, c.T)
    outs = []
    for _ in range(2):
        o = torch.empty_like(c.out)
        fx.moe_layer_forward(c.dev, c.x, c.T, layer.shape.H, o, layer.shape.H, ws, ws.numel())
        outs.append(o)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))


def test_routed_scaling_factor():
    """routed_scaling_factor != 1 (Dots3NoteTextConfig field; the vision
    router's router_scaling_factor plays the same part): the K weights sum to
    the factor and the output follows the oracle with the same factor."""
    wl, layer0, x = gen.workload_inputs("toy")
    sh = layer0.shape
    layer = gen.Layer(sh, layer0.router_w, layer0.w_gate, layer0.s_gate, layer0.w_up, layer0.s_up, layer0.w_down,
                      layer0.s_down)
    layer.routed_scaling = 2.5
    dev = tu.upload_layer(layer, routed_scaling=2.5)
    c = gc.Case(layer, x, dev)
    assert np.allclose(c.np("w").sum(1), 2.5, atol=1e-5)
    ref = moe.layer_forward(x, layer)
    keep = ~ref["route"].near_tie
    gc.assert_output_close(moe.bf16_to_f64(c.np("out"))[keep], ref["out"][keep], "routed_scaling 2.5")


def test_dense_ffn_is_the_single_expert():
    """The dense FFN workload (one expert, top-1, no shared expert): every
    token is routed to expert 0 with weight exactly 1 and the output is that
    expert's FFN rounded once to bf16 (combine of a single row)."""
    wl, layer, c = get_case("dense")
    assert not c.np("idx").any() and np.all(c.np("w") == 1.0)
    assert np.array_equal(c.np("perm"), np.arange(c.T)) and np.array_equal(c.np("inv").ravel(), np.arange(c.T))
    assert np.array_equal(tu.bf16_bits(c.y), c.np("out"))


# ----------------------------------------------------------------------------- router variants

def _variant_layer(layer0, **opts):
    layer = gen.Layer(layer0.shape, layer0.router_w, layer0.w_gate, layer0.s_gate, layer0.w_up, layer0.s_up,
                      layer0.w_down, layer0.s_down)
    for k, v in opts.items():
        setattr(layer, k, v)
    return layer


_VARIANTS = {
    "groups": dict(n_group=4, topk_group=2),
    "bias": dict(router_bias="random"),
    "no_norm": dict(norm_topk=False, routed_scaling=1.5),
    "all": dict(n_group=8, topk_group=3, router_bias="random", norm_topk=False, routed_scaling=2.0),
}


def _opts(name, E):
    opts = dict(_VARIANTS[name])
    if opts.get("router_bias") == "random":
        # of the order of the probabilities (1/E), so that it changes choices
        opts["router_bias"] = np.random.default_rng(31).normal(0, 1.0 / E, E).astype(np.float32)
    return opts


@pytest.mark.parametrize("variant", list(_VARIANTS))
def test_router_variants_toy(variant):
    """Group-limited selection, a selection-only bias and norm_topk_prob off
    (Dots3NoteTextConfig n_group / topk_group / norm_topk_prob): routing
    bit-exact apart from flagged near-ties, and the whole layer within the
    output tolerance, on the toy layer at T = 512."""
    wl, layer0, _ = gen.workload_inputs("toy")
    sh = layer0.shape
    layer = _variant_layer(layer0, **_opts(variant, sh.E))
    x = gen.make_x(512, sh.H, 40 + len(variant))
    c = gc.Case(layer, x, tu.upload_layer(layer))
    ref = moe.layer_forward(x, layer)
    r = ref["route"]
    keep = ~r.near_tie
    assert keep.mean() > 0.95
    assert np.array_equal(c.np("idx")[keep], r.idx[keep])
    assert np.allclose(c.np("w")[keep], r.w[keep], rtol=2e-5, atol=1e-6)
    if variant == "bias":   # the bias changed the choice of some tokens
        assert (moe.route(x, layer.router_w, sh.K).idx != r.idx).any()
    gc.assert_output_close(moe.bf16_to_f64(c.np("out"))[keep], ref["out"][keep], f"router variant {variant}")


def test_router_variants_full_router():
    """The 256-expert router with 8 groups (4 eligible) and a bias: routing
    and weights against the oracle on the decode batch."""
    wl, layer0, c0 = get_case("decode")
    sh = layer0.shape
    layer = _variant_layer(layer0, n_group=8, topk_group=4, **{"router_bias": _opts("bias", sh.E)["router_bias"]})
    dev = tu.upload_layer(layer, share_experts=c0.dev)
    T = c0.T
    idx = torch.empty((T, sh.K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, sh.K), dtype=torch.float32, device="cuda")
    ws = tu.workspace(dev, T)
    fx.moe_route(dev, c0.x, T, sh.H, idx, w, None, ws, ws.numel())
    r = moe.route_layer(c0.x_bits, layer)
    keep = ~r.near_tie
    got = idx.cpu().numpy()
    assert np.array_equal(got[keep], r.idx[keep])
    assert np.allclose(w.cpu().numpy()[keep], r.w[keep], rtol=2e-5, atol=1e-6)
    gs = sh.E // 8
    assert all(len(set(int(e) // gs for e in row)) <= 4 for row in got)


# ----------------------------------------------------------------------------- degenerate batches

@pytest.mark.parametrize("T", [1, 2])
def test_single_token_batches(T):
    """T = 1 and 2 on the full layer (one row per touched group, K+1 groups
    per token): routing bit-exact and every output value within tolerance."""
    wl, layer, c0 = get_case("decode")
    x = c0.x_bits[:T]
    c = gc.Case(layer, x, c0.dev)
    r = moe.route(x, layer.router_w, layer.shape.K)
    keep = ~r.near_tie
    assert np.array_equal(c.np("idx")[keep], r.idx[keep])
    off = c.np("offsets")
    assert off[-1] == T * (layer.shape.K + 1) and (np.diff(off) >= 0).all()
    ref = moe.token_outputs(x, layer, np.arange(T)[keep])
    gc.assert_output_close(moe.bf16_to_f64(c.np("out"))[keep], ref, f"T={T}")


# ----------------------------------------------------------------------------- split-K down GEMM

def test_split_k_down_exact_integers():
    """A one-group layer at a small batch has fewer down-GEMM output tiles than
    SMs, so the down GEMM splits its K blocks over CTAs and a second kernel
    adds the FP32 partials. With integer codes and unit scales every partial
    and the total are exact, so y must be bf16(A Wd^T) bit for bit."""
    sh = gen.LayerShape(H=512, E=1, K=1, F=2048, ld_f=2048, S=0)
    rng = np.random.default_rng(41)
    vals = np.array([0x00, 0x38, 0x40, 0x44, 0x48, 0xB8, 0xC0, 0xC4, 0xC8], np.uint8)
    pick = lambda shape: vals[rng.integers(0, 9, shape)]
    layer = gen.Layer(sh, gen.make_router(sh, 0), pick((1, sh.F, sh.H)), np.ones((1, sh.FB, sh.HB), np.float32),
                      pick((1, sh.F, sh.H)), np.ones((1, sh.FB, sh.HB), np.float32),
                      pick((1, sh.H, sh.ld_f)), np.ones((1, sh.HB, sh.FB), np.float32))
    dev = tu.upload_layer(layer)
    T = 64
    hq = pick((T, sh.FB * 128))
    hs = np.ones((sh.FB, T), np.float32)
    off = np.array([0, T, T], np.int32)
    y = torch.full((T, sh.H), float("nan"), dtype=torch.bfloat16, device="cuda")
    fx.moe_down(dev, tu.to_device(hq), tu.to_device(hs), tu.to_device(off), T, y)
    code, bits = fx.moe_get_device_status(dev)
    assert code == fx.MOE_OK, f"{bits:#x}"
    ints = moe.e4m3.decode(np.arange(256, dtype=np.uint8))
    exact = ints[hq].astype(np.int64) @ ints[layer.w_down[0]].astype(np.int64).T
    want = tu.bf16_bits(torch.tensor(exact.astype(np.float32)).to(torch.bfloat16))
    assert np.array_equal(tu.bf16_bits(y), want)


def test_kernels_per_forward():
    """The launch count bench.py reports: route 2, permute 2 while the
    E x ceil(T/32)-word token bitmap fits one CTA (8192 words: T <= 1024 at
    E = 256) else 4, gate/up 1, down 1 (+1 when it splits its K blocks, as
    the dense FFN does at T = 64), combine 1."""
    _, _, c = get_case("decode")
    assert fx.moe_kernels_per_forward(c.dev, c.T) == 7
    assert fx.moe_kernels_per_forward(c.dev, 1024) == 7
    assert fx.moe_kernels_per_forward(c.dev, 1025) == 9
    assert fx.moe_kernels_per_forward(c.dev, 16384) == 9
    assert fx.moe_kernels_per_forward(c.dev, 0) == 0
    _, _, cd = get_case("dense")
    assert fx.moe_kernels_per_forward(cd.dev, cd.T) == 8


@pytest.mark.parametrize("T", [1, 31, 1024, 1025, 3000])
def test_permute_plan_paths_on_the_full_router(T):
    """Both plans of the permutation (one CTA while the 256-expert token
    bitmap fits 8192 words, T <= 1024; three kernels above) give the oracle's
    offsets, perm and inv bit-exactly on Zipf-skewed routing of the full
    layer, and both flag an out-of-range and a repeated expert id."""
    wl, layer, c = get_case("decode")
    sh = layer.shape
    rng = np.random.default_rng(T)
    pz = 1.0 / np.arange(1, sh.E + 1) ** 1.1
    pz /= pz.sum()
    idx_np = np.stack([rng.choice(sh.E, sh.K, replace=False, p=pz) for _ in range(T)]).astype(np.int32)
    x = tu.bf16_tensor(gen.make_x(T, sh.H, 77, outliers=2))
    rows = T * (sh.K + sh.S)

    def run(ix):
        off = torch.empty(sh.E + 2, dtype=torch.int32, device="cuda")
        perm = torch.full((rows,), -7, dtype=torch.int32, device="cuda")
        inv = torch.empty((T, sh.K), dtype=torch.int32, device="cuda")
        xq = torch.empty((rows, sh.H), dtype=torch.uint8, device="cuda")
        xs = torch.empty((sh.HB, rows), dtype=torch.float32, device="cuda")
        ws = tu.workspace(c.dev, T)
        fx.moe_permute(c.dev, x, T, sh.H, torch.from_numpy(ix).cuda(), off, perm, inv, xq, xs, ws, ws.numel())
        return off.cpu().numpy(), perm.cpu().numpy(), inv.cpu().numpy()

    off, perm, inv = run(idx_np)
    assert fx.moe_get_device_status(c.dev)[0] == fx.MOE_OK
    p = moe.permute(idx_np, sh.E, sh.S)
    assert np.array_equal(off, p.offsets) and np.array_equal(perm, p.perm) and np.array_equal(inv, p.inv)
    bad = idx_np.copy()
    bad[T - 1, 0] = sh.E                   # out of range
    if T > 1:
        bad[0, sh.K - 1] = bad[0, 0]       # repeated within token 0
    run(bad)
    code, bits = fx.moe_get_device_status(c.dev)
    assert code == fx.MOE_ERR_DEVICE and bits & 1
    assert T == 1 or bits & 2


def test_forward_is_cuda_graph_capturable():
    """The calls are asynchronous, allocate nothing and chain their kernels
    with programmatic dependent launch: a captured moe_layer_forward replays
    to the same bits as the eager call."""
    wl, layer, c = get_case("toy_t2048")
    sh = layer.shape
    ws = tu.workspace(c.dev, c.T)
    eager = torch.empty((c.T, sh.H), dtype=torch.bfloat16, device="cuda")
    fx.moe_layer_forward(c.dev, c.x, c.T, sh.H, eager, sh.H, ws, ws.numel())
    torch.cuda.synchronize()
    out = torch.zeros_like(eager)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            fx.moe_layer_forward(c.dev, c.x, c.T, sh.H, out, sh.H, ws, ws.numel())
    for _ in range(2):
        out.zero_()
        g.replay()
    torch.cuda.synchronize()
    code, bits = fx.moe_get_device_status(c.dev)
    assert code == fx.MOE_OK, f"{bits:#x}"
    assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
    del g


# ----------------------------------------------------------------------------- failure detection

def test_timed_out_wait_is_reported_and_the_handle_recovers():
    """A pipeline wait that runs out (a stage the producer withholds, with a
    1 ms limit) ends the GEMM launch with MOE_STATUS_WAIT_TIMEOUT instead of
    hanging; the next forward on the same handle is bit-identical to one
    before the fault."""
    wl, layer, c = get_case("toy")
    sh, T = layer.shape, c.T
    fx.moe_gate_up(c.dev, c.xq, c.xs, c.offsets, T, c.hq, c.hs)
    assert fx.moe_get_device_status(c.dev) == (fx.MOE_OK, 0)
    h_ref = c.hq.clone()
    for stage in ("gate_up", "down"):
        fx.moe_test_inject_stall(c.dev, 1_000_000)
        h = torch.zeros_like(c.hq)
        hs = torch.zeros_like(c.hs)
        y = torch.zeros_like(c.y)
        if stage == "gate_up":
            fx.moe_gate_up(c.dev, c.xq, c.xs, c.offsets, T, h, hs)
        else:
            fx.moe_down(c.dev, c.hq, c.hs, c.offsets, T, y)
        code, bits = fx.moe_get_device_status(c.dev)
        assert code == fx.MOE_ERR_DEVICE and bits & 0x4, (stage, code, hex(bits))
        # the handle is usable at once: the same launch again is complete and exact
        if stage == "gate_up":
            fx.moe_gate_up(c.dev, c.xq, c.xs, c.offsets, T, h, hs)
            assert fx.moe_get_device_status(c.dev) == (fx.MOE_OK, 0)
            assert torch.equal(h, h_ref)
        else:
            fx.moe_down(c.dev, c.hq, c.hs, c.offsets, T, y)
            assert fx.moe_get_device_status(c.dev) == (fx.MOE_OK, 0)
            assert torch.equal(y.view(torch.int16), c.y.view(torch.int16))
    ws = tu.workspace(c.dev, T)
    out = torch.empty_like(c.out)
    fx.moe_layer_forward(c.dev, c.x, T, sh.H, out, sh.H, ws, ws.numel())
    assert fx.moe_get_device_status(c.dev) == (fx.MOE_OK, 0)
    assert torch.equal(out.view(torch.int16), c.out.view(torch.int16))


def test_inconsistent_offsets_set_bad_plan_and_do_no_work():
    """Group offsets that decrease or run past the row count are caught by the
    GEMM's own check before any tile is planned: MOE_STATUS_BAD_PLAN, and the
    output buffers are left untouched."""
    wl, layer, c = get_case("toy")
    sh, T = layer.shape, c.T
    good = c.np("offsets")
    for bad in (np.concatenate([good[:5], good[4:5] - 1, good[6:]]),      # a decreasing step
                np.concatenate([good[:-1], [good[-1] + 128]])):          # past the last row
        off = torch.from_numpy(bad.astype(np.int32)).cuda()
        h = torch.full_like(c.hq, 0x5A)
        hs = torch.full_like(c.hs, 7.0)
        fx.moe_gate_up(c.dev, c.xq, c.xs, off, T, h, hs)
        code, bits = fx.moe_get_device_status(c.dev)
        assert code == fx.MOE_ERR_DEVICE and bits == 0x8, hex(bits)
        assert bool((h == 0x5A).all()) and bool((hs == 7.0).all())
    fx.moe_gate_up(c.dev, c.xq, c.xs, c.offsets, T, h, hs)
    assert fx.moe_get_device_status(c.dev) == (fx.MOE_OK, 0)


def test_strided_activations_outputs_and_weight_rows():
    """Row strides beyond the hidden size: x read from a [T][H+128] buffer,
    the output written into a [T][H+64] buffer (its pad left untouched), and
    gate/up weight rows stored with a padded stride ld_h = H + 128. The
    result equals the contiguous forward bit for bit."""
    wl, layer, c = get_case("toy")
    sh, T = layer.shape, c.T
    x_wide = torch.zeros((T, sh.H + 128), dtype=torch.bfloat16, device="cuda")
    x_wide[:, :sh.H] = c.x
    out_wide = torch.full((T, sh.H + 64), 7.0, dtype=torch.bfloat16, device="cuda")
    ws = tu.workspace(c.dev, T)
    fx.moe_layer_forward(c.dev, x_wide, T, sh.H + 128, out_wide, sh.H + 64, ws, ws.numel())
    assert torch.equal(out_wide[:, :sh.H].contiguous().view(torch.int16), c.out.view(torch.int16))
    assert bool((out_wide[:, sh.H:] == 7.0).all())
    # gate/up rows with a padded stride (pad bytes hold garbage that must not be read)
    w = c.dev.weights
    pad = lambda t: torch.cat([t, torch.full(t.shape[:2] + (128,), 0x7E, dtype=t.dtype, device=t.device)], 2)
    lw = fx.LayerWeights(pad(w.w_gate), pad(w.w_up), w.w_down, w.s_gate, w.s_up, w.s_down, w.router_w)
    wide = fx.MoeLayer(sh.H, sh.E, sh.K, sh.F, lw, ld_h=sh.H + 128, ld_f=sh.ld_f, n_shared=sh.S)
    o2 = torch.empty_like(c.out)
    ws2 = tu.workspace(wide, T)
    fx.moe_layer_forward(wide, c.x, T, sh.H, o2, sh.H, ws2, ws2.numel())
    assert fx.moe_get_device_status(wide)[0] == fx.MOE_OK
    assert torch.equal(o2.view(torch.int16), c.out.view(torch.int16))
