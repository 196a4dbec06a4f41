"""FP64 CPU oracle of the forward pass of one fine-grained-FP8 MoE layer.

TEST INFRASTRUCTURE: plain, slow, obviously correct. Only tests/,
__graft_entry__.smoke() and bench.py's CPU baseline may import this package;
the CUDA path never calls it and shares no code with it.

Layer (transformers docs page "Dots 3 Note Preview", Dots3NoteTextConfig:
hidden_size 5120, n_routed_experts 256, n_shared_experts 1,
num_experts_per_tok 8, n_group 1 / topk_group 1 (ungrouped), norm_topk_prob
True, routed_scaling_factor 1.0, hidden_act silu, mlp_bias False,
moe_intermediate_size 1536, shared_experts_intermediate_size 1536; model card
dots-studio/dots3-note-prev, "Model Overview": 256 routed + 1 shared, top-8).
Precision (transformers PR #47844, "What does this PR do?"): E4M3 weights with
one scale per 128 x 128 block and dynamically quantised activations.

Steps and the readings taken where the pages are silent:
  route    logits = x . Wr^T in FP64 (the kernel's are FP32); p = softmax over
           all E experts; the top-K by p, ties to the lower expert id; the K
           weights are p renormalised to sum 1, times routed_scaling_factor
           (1.0). Slots are listed in ascending expert id. A token is flagged
           as a near-tie when p_(K) - p_(K+1) < 1e-6.
           Router variants the config schema allows (n_group, topk_group,
           norm_topk_prob, and the selection bias of routers balanced by a
           bias instead of an auxiliary loss): the selection score is
           p + bias; with n_group > 1 the experts form n_group contiguous
           groups, each scored by its best member, and only the topk_group
           best groups (ties to the lower group) are eligible; the weights
           come from the unbiased p of the selected experts, renormalised
           only if norm_topk_prob. The near-tie gap is then taken on the
           selection score, and on the group scores when groups apply.
  permute  counting sort of the (token, slot) pairs by expert, stable in
           token order; offsets has E+2 entries, the shared expert is group E
           and holds one row per token, in token order.
  quantise per row, per 128-channel group: s = fp32(amax) / 448 in fp32,
           q = E4M3(fp32(v) / s) (fp32 division, RNE, saturating);
           an all-zero group gets s = 0 and q = 0.
  expert   G = A Wg^T, U = A Wu^T, h = silu(G) * U, all FP64 on dequantised
           operands (A = q * s per group, W = q * s per block); h is rounded
           to fp32 and quantised like the activations; y = dequant(h) Wd^T.
  combine  out[t] = sum_k w[t,k] y[row(t,k)] + y[shared row of t], FP64.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

from . import e4m3

GROUP = 128          # activation group / weight block edge
NEAR_TIE = 1e-6      # near-tie flag threshold on p_(K) - p_(K+1)
# Experts are independent, so the per-expert work runs on a thread pool
# (numpy releases the GIL in the table lookups and the matmuls).
WORKERS = max(1, min(32, os.cpu_count() or 1))


def _pool_map(fn, items):
    items = list(items)
    if WORKERS == 1 or len(items) < 2:
        return [fn(i) for i in items]
    with ThreadPoolExecutor(WORKERS) as ex:
        return list(ex.map(fn, items))


# ---------------------------------------------------------------------------
# bf16 helpers (inputs arrive as bf16 bit patterns)
# ---------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16_f64(v: np.ndarray) -> np.ndarray:
    """Round to bf16 (via fp32, nearest-even at each step) and return as f64."""
    f = np.asarray(v, dtype=np.float64).astype(np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    r = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint32) << 16
    return r.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# Quantisation (dynamic activations and dequantisation)
# ---------------------------------------------------------------------------

def quantize_rows(v: np.ndarray):
    """Per row, per 128-channel group: (codes uint8 [rows, C], scales f32 [rows, ceil(C/128)]).
    The last group may be partial; its amax covers the real channels only."""
    v32 = np.asarray(v, dtype=np.float32)
    rows, C = v32.shape
    ng = -(-C // GROUP)
    codes = np.zeros((rows, C), np.uint8)
    scales = np.zeros((rows, ng), np.float32)
    for g in range(ng):
        c0, c1 = g * GROUP, min(C, (g + 1) * GROUP)
        blk = v32[:, c0:c1]
        amax = np.max(np.abs(blk), axis=1).astype(np.float32)
        s = (amax / np.float32(448.0)).astype(np.float32)
        scales[:, g] = s
        nz = amax > 0
        if np.any(nz):
            q = e4m3.encode((blk[nz] / s[nz, None]).astype(np.float32))
            codes[np.nonzero(nz)[0][:, None], np.arange(c0, c1)[None, :]] = q
    return codes, scales


def dequant_rows(codes: np.ndarray, scales: np.ndarray, C: int = None) -> np.ndarray:
    """codes [rows, >=C], scales [rows, ceil(C/128)] -> f64 [rows, C]."""
    codes = np.asarray(codes)
    C = codes.shape[1] if C is None else C
    v = e4m3.decode(codes[:, :C])
    s = np.repeat(np.asarray(scales, np.float64), GROUP, axis=1)[:, :C]
    return v * s


def dequant_block(codes: np.ndarray, scales: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Weight matrix codes [rows, >=cols] with one scale per 128x128 block -> f64 [rows, cols].
    Element (n, k) is decode(codes[n, k]) * scales[n // 128, k // 128]."""
    rb, cb = -(-rows // GROUP), -(-cols // GROUP)
    padded = np.zeros((rb * GROUP, cb * GROUP), np.uint8)
    padded[:rows, :cols] = np.asarray(codes)[:rows, :cols]
    v = e4m3.decode(padded)
    v.reshape(rb, GROUP, cb, GROUP).__imul__(np.asarray(scales, np.float64)[:rb, None, :cb, None])
    return v[:rows, :cols]


# ---------------------------------------------------------------------------
# Routing
# ---------------------------------------------------------------------------

@dataclass
class Route:
    logits: np.ndarray   # f64 [T, E]
    probs: np.ndarray    # f64 [T, E] softmax over E
    idx: np.ndarray      # int32 [T, K], ascending expert id
    w: np.ndarray        # f64 [T, K], sums to routed_scaling_factor
    gap: np.ndarray      # f64 [T], p_(K) - p_(K+1)
    near_tie: np.ndarray  # bool [T]


def router_logits(x_bits: np.ndarray, router_w: np.ndarray) -> np.ndarray:
    return bf16_to_f64(x_bits) @ np.asarray(router_w, np.float64).T


def softmax(logits: np.ndarray) -> np.ndarray:
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    return e / e.sum(axis=1, keepdims=True)


def select_topk(probs: np.ndarray, K: int, routed_scaling: float = 1.0, n_group: int = 1, topk_group: int = 1,
                bias=None, norm_topk: bool = True):
    """Top-K by selection score s = p + bias among the eligible experts, ties
    to the lower expert id; slots in ascending id. Dots3NoteTextConfig:
    n_group partitions the routed experts for selection and topk_group is
    the number of groups a token may draw from (1 and 1: ungrouped)."""
    T, E = probs.shape
    ids = np.arange(E)
    b = np.zeros(E) if bias is None else np.asarray(bias, np.float64)
    gsize = E // n_group
    idx = np.empty((T, K), np.int32)
    w = np.empty((T, K), np.float64)
    gap = np.empty(T, np.float64)
    for t in range(T):
        s = probs[t] + b
        ggap = np.inf
        if n_group > 1:
            gscore = s.reshape(n_group, gsize).max(axis=1)          # a group's best member
            gorder = np.lexsort((np.arange(n_group), -gscore))
            keep = gorder[:topk_group]
            if topk_group < n_group:
                ggap = gscore[gorder[topk_group - 1]] - gscore[gorder[topk_group]]
            cand = np.sort(np.concatenate([ids[g * gsize:(g + 1) * gsize] for g in keep]))
        else:
            cand = ids
        order = cand[np.lexsort((cand, -s[cand]))]   # primary: s descending; secondary: id ascending
        sel = np.sort(order[:K])
        idx[t] = sel
        ps = probs[t, sel]
        w[t] = (ps / ps.sum() if norm_topk else ps) * routed_scaling
        egap = s[order[K - 1]] - s[order[K]] if K < len(cand) else np.inf
        gap[t] = min(egap, ggap)
    return idx, w, gap


def route(x_bits: np.ndarray, router_w: np.ndarray, K: int, routed_scaling: float = 1.0, n_group: int = 1,
          topk_group: int = 1, bias=None, norm_topk: bool = True) -> Route:
    logits = router_logits(x_bits, router_w)
    probs = softmax(logits)
    idx, w, gap = select_topk(probs, K, routed_scaling, n_group, topk_group, bias, norm_topk)
    return Route(logits, probs, idx, w, gap, gap < NEAR_TIE)


def router_options(layer) -> dict:
    """The layer's router settings (defaults: the text model's)."""
    return {"routed_scaling": getattr(layer, "routed_scaling", 1.0), "n_group": getattr(layer, "n_group", 1),
            "topk_group": getattr(layer, "topk_group", 1), "bias": getattr(layer, "router_bias", None),
            "norm_topk": getattr(layer, "norm_topk", True)}


def route_layer(x_bits: np.ndarray, layer) -> Route:
    return route(x_bits, layer.router_w, layer.shape.K, **router_options(layer))


# ---------------------------------------------------------------------------
# Permutation
# ---------------------------------------------------------------------------

@dataclass
class Perm:
    offsets: np.ndarray  # int32 [E+2]; group E (shared) is rows [R, R+T)
    perm: np.ndarray     # int32 [R+T]; row -> token
    inv: np.ndarray      # int32 [T, K]; (token, slot) -> row


def permute(idx: np.ndarray, E: int, S: int = 1) -> Perm:
    """Counting sort of (token, slot) pairs by expert, stable in token order;
    with S = 1 the shared expert's group E holds one row per token."""
    idx = np.asarray(idx)
    T, K = idx.shape
    R = T * K
    counts = np.bincount(idx.reshape(-1), minlength=E)[:E]
    offsets = np.zeros(E + 2, np.int64)
    offsets[1:E + 1] = np.cumsum(counts)
    offsets[E + 1] = offsets[E] + T * S
    flat = idx.reshape(-1)
    order = np.argsort(flat, kind="stable")     # (t, k) pairs grouped by expert, token order kept
    rows = np.empty(R, np.int64)
    rows[order] = np.arange(R)
    inv = rows.reshape(T, K)
    perm = np.empty(R + T * S, np.int64)
    perm[rows] = np.arange(R) // K
    perm[R:] = np.arange(T * S) % max(T, 1)
    return Perm(offsets.astype(np.int32), perm.astype(np.int32), inv.astype(np.int32))


# ---------------------------------------------------------------------------
# Expert FFN and combine
# ---------------------------------------------------------------------------

def silu(g: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def expert_gate_up(a: np.ndarray, w_gate, s_gate, w_up, s_up, F: int, H: int) -> np.ndarray:
    """a: f64 [n, H] dequantised activations -> h f64 [n, F] = silu(a Wg^T) * (a Wu^T)."""
    Wg = dequant_block(w_gate, s_gate, F, H)
    Wu = dequant_block(w_up, s_up, F, H)
    return silu(a @ Wg.T) * (a @ Wu.T)


def expert_down(b: np.ndarray, w_down, s_down, H: int, F: int) -> np.ndarray:
    """b: f64 [n, F] dequantised h -> y f64 [n, H]."""
    return b @ dequant_block(w_down, s_down, H, F).T


def expert_ffn_rows(xq, xs, offsets, layer, groups=None):
    """Grouped expert FFN over permuted rows. Returns dict with
    h (f64 [rows, F]), hq (u8), hs (f32), y (f64 [rows, H]) for the groups given."""
    sh = layer.shape
    H, F = sh.H, sh.F
    rows = int(offsets[-1])
    h = np.zeros((rows, F), np.float64)
    hq = np.zeros((rows, F), np.uint8)
    hs = np.zeros((rows, sh.FB), np.float32)
    y = np.zeros((rows, H), np.float64)
    groups = range(sh.E + 1) if groups is None else groups

    def one(g):
        r0, r1 = int(offsets[g]), int(offsets[g + 1])
        if r1 == r0:
            return None
        a = dequant_rows(xq[r0:r1], xs[r0:r1], H)
        hg = expert_gate_up(a, layer.w_gate[g], layer.s_gate[g], layer.w_up[g], layer.s_up[g], F, H)
        q, s = quantize_rows(hg.astype(np.float32))
        yg = expert_down(dequant_rows(q, s, F), layer.w_down[g], layer.s_down[g], H, F)
        return r0, r1, hg, q, s, yg

    for res in _pool_map(one, groups):
        if res is not None:
            r0, r1, hg, q, s, yg = res
            h[r0:r1], hq[r0:r1], hs[r0:r1], y[r0:r1] = hg, q, s, yg
    return {"h": h, "hq": hq, "hs": hs, "y": y}


def expert_down_rows(hq, hs, offsets, layer, groups=None):
    """Down projection alone over permuted rows (h given as codes + scales)."""
    sh = layer.shape
    rows = int(offsets[-1])
    y = np.zeros((rows, sh.H), np.float64)
    groups = range(sh.E + 1) if groups is None else groups

    def one(g):
        r0, r1 = int(offsets[g]), int(offsets[g + 1])
        if r1 == r0:
            return None
        return r0, r1, expert_down(dequant_rows(hq[r0:r1], hs[r0:r1], sh.F), layer.w_down[g], layer.s_down[g],
                                   sh.H, sh.F)

    for res in _pool_map(one, groups):
        if res is not None:
            y[res[0]:res[1]] = res[2]
    return y


def combine(y: np.ndarray, inv: np.ndarray, w: np.ndarray, S: int = 1) -> np.ndarray:
    """out[t] = sum_k w[t,k] * y[inv[t,k]] + y[R + t] (shared expert, weight 1, when S = 1)."""
    inv = np.asarray(inv)
    T, K = inv.shape
    R = T * K
    out = np.zeros((T, y.shape[1]), np.float64)
    for k in range(K):
        out += np.asarray(w, np.float64)[:, k:k + 1] * y[inv[:, k]]
    return out + y[R:R + T] if S else out


def quantize_tokens(x_bits: np.ndarray):
    """Dynamic activation quantisation of every token (the rows the permute gathers)."""
    return quantize_rows(bf16_to_f64(x_bits).astype(np.float32))


def gather_rows(tok_codes, tok_scales, perm):
    return tok_codes[perm], tok_scales[perm]


def layer_forward(x_bits: np.ndarray, layer) -> dict:
    """Whole layer: route -> permute -> quantise/gather -> expert FFNs -> combine."""
    sh = layer.shape
    r = route_layer(x_bits, layer)
    p = permute(r.idx, sh.E, sh.S)
    tq, ts = quantize_tokens(x_bits)
    xq, xs = gather_rows(tq, ts, p.perm)
    f = expert_ffn_rows(xq, xs, p.offsets, layer)
    out = combine(f["y"], p.inv, r.w, sh.S)
    return {"route": r, "perm": p, "xq": xq, "xs": xs, **f, "out": out}


def token_outputs(x_bits: np.ndarray, layer, tokens, idx=None, w=None, y_bf16: bool = False) -> np.ndarray:
    """Direct per-token evaluation (no permutation) for a subset of tokens:
    out[t] = sum_k w_k FFN_{e_k}(x_t) + FFN_shared(x_t). Routing is the
    oracle's unless idx/w (full [T, K] tables) are given. Each expert is
    dequantised once for all the sampled tokens that use it. With y_bf16,
    each expert's output row is rounded to bf16 before it is weighted: the
    layer keeps the down projection's output y as a bf16 tensor (the model's
    activation dtype) and the combine sums those rows; everything else
    stays FP64."""
    sh = layer.shape
    tokens = np.asarray(tokens)
    xb = np.asarray(x_bits)[tokens]
    if idx is None:
        r = route_layer(xb, layer)
        idx_s, w_s = r.idx, r.w
    else:
        idx_s, w_s = np.asarray(idx)[tokens], np.asarray(w, np.float64)[tokens]
    tq, ts = quantize_tokens(xb)
    a = dequant_rows(tq, ts, sh.H)
    n = len(tokens)
    out = np.zeros((n, sh.H), np.float64)
    users = {}
    for i in range(n):
        for k in range(sh.K):
            users.setdefault(int(idx_s[i, k]), []).append((i, float(w_s[i, k])))
    if sh.S:
        users[sh.E] = [(i, 1.0) for i in range(n)]
    def one(item):
        g, lst = item
        rows = np.array([i for i, _ in lst])
        wt = np.array([c for _, c in lst])
        hg = expert_gate_up(a[rows], layer.w_gate[g], layer.s_gate[g], layer.w_up[g], layer.s_up[g], sh.F, sh.H)
        q, s = quantize_rows(hg.astype(np.float32))
        yg = expert_down(dequant_rows(q, s, sh.F), layer.w_down[g], layer.s_down[g], sh.H, sh.F)
        if y_bf16:
            yg = f64_to_bf16_f64(yg)
        return rows, wt[:, None] * yg

    for rows, contrib in _pool_map(one, sorted(users.items())):
        np.add.at(out, rows, contrib)
    return out


def layer_forward_bf16(x_bits: np.ndarray, layer, tokens=None, idx=None, w=None) -> np.ndarray:
    """BF16-checkpoint cross-check path: weights W = bf16(q * s), no
    activation or h quantisation, FP64 arithmetic otherwise (transformers
    PR #47844, "What does this PR do?": BF16 and FP8 checkpoints)."""
    sh = layer.shape
    T = np.asarray(x_bits).shape[0]
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    xb = np.asarray(x_bits)[tokens]
    if idx is None:
        r = route_layer(xb, layer)
        idx_s, w_s = r.idx, r.w
    else:
        idx_s, w_s = np.asarray(idx)[tokens], np.asarray(w, np.float64)[tokens]
    a = bf16_to_f64(xb)
    out = np.zeros((len(tokens), sh.H), np.float64)
    users = {}
    for i in range(len(tokens)):
        for k in range(sh.K):
            users.setdefault(int(idx_s[i, k]), []).append((i, float(w_s[i, k])))
    if sh.S:
        users[sh.E] = [(i, 1.0) for i in range(len(tokens))]
    def one(item):
        g, lst = item
        rows = np.array([i for i, _ in lst])
        wt = np.array([c for _, c in lst])
        Wg = f64_to_bf16_f64(dequant_block(layer.w_gate[g], layer.s_gate[g], sh.F, sh.H))
        Wu = f64_to_bf16_f64(dequant_block(layer.w_up[g], layer.s_up[g], sh.F, sh.H))
        Wd = f64_to_bf16_f64(dequant_block(layer.w_down[g], layer.s_down[g], sh.H, sh.F))
        hg = silu(a[rows] @ Wg.T) * (a[rows] @ Wu.T)
        return rows, wt[:, None] * (hg @ Wd.T)

    for rows, contrib in _pool_map(one, sorted(users.items())):
        np.add.at(out, rows, contrib)
    return out
