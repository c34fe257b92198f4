"""Float64 CPU oracle of the routed MoE block.  TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this module.  It shares no code with the CUDA path; its inputs come
from ``sigmoid_top_routing_b200.inputs`` (a generator with none of the
block's arithmetic), widened exactly to float64.

What it computes, and where each step is stated:

  route      TileGym PR #187 ("[E2E Model Support] Add TileGym kernel
             integration for LFM2 MoE"), section "Weight layout and routing":
             sigmoid (not softmax) scores; the expert bias only chooses the
             top-k experts and the gathered weights stay unbiased;
             norm_topk_prob divides by sum + 1e-6, then routed_scaling_factor
             multiplies.  TensorFold pull #1492 (lfm2_moe on CUDA), section
             "What": fp32 router weights, expert bias, normalised top-k,
             eps 1e-6; section "Verification": an all-NaN router row must not
             pick the same expert twice.
  experts    TileGym PR #187, "Weight layout and routing": gate_up is
             (E, 2I, H) gate rows first, down is (E, H, I).  vllm.cpp PR #684
             ("W2 (MODEL-NEMOTRON-H): the non-gated relu^2 MoE expert"),
             section "The seam decision": h = up(x); h = relu(h)^2;
             y = down(h), no gate half.  bloomery PR #235 ("the common pieces
             a Nemotron-H card body attaches to"), section "What": relu_sqr
             is max(x, 0)^2 and a non-finite input stays non-finite.
  combine    vllm.cpp PR #684, "The finding that justifies the row": the
             routed scale multiplies the finished routed sum once; folding it
             into each expert weight is a different rounded value.
  plan       TensorFold issue #548 ("Zig CUDA ports: shared layers below
             lanes.Backend, and one place to coordinate them"): the grouped
             expert plan (per-expert grouping of the routed pairs).  Written
             here as counts, exclusive offsets and a stable permutation.
  affine-4   TensorFold pull #1492, "What": MLX affine 4-bit experts,
             dequantised exactly in float64 as in its "Verification" section
             (the float64 reference dequantises the MLX weights exactly).
  nvfp4      TensorFold issue #548: NVFP4 experts read as stored in the
             ModelOpt layout, "weight uint8 [N, K/2], weight_scale e4m3
             [N, K/16], weight_scale_2 as the global scale", W4A16; its
             skip/down_scale rows name the down projection's own global scale.
             Dequantised exactly in float64: w = e2m1(code) * e4m3(scale) * g.

Readings where the pages are silent:
  * the bias is added to the sigmoid score, c = s + b, for selection only;
  * selection order: descending c, ties to the lower expert index, NaN below
    every number, -0.0 == +0.0; the k picks are returned in rank order;
  * an all-NaN row picks experts 0..k-1; its weights, and so its output row,
    are NaN;
  * relu^2 keeps NaN (u > 0 ? u : (NaN ? u : 0)) and then squares;
  * NVFP4: the low nibble of a code byte is the lower k; e2m1 is 1 sign,
    2 exponent (bias 1) and 1 mantissa bit with no inf/NaN; the block scale is
    e4m3 "fn" (bias 7, no infinities, 0x7F/0xFF NaN); each expert has one
    fp32 global scale for W1 (gate and up together) and one for W2.

Router and activation variants (TensorFold issue #548: the table of pieces
each model family builds lists "routers (softmax, sigmoid + bias)"; its
section "Paths your experts test does not reach" runs swiglu_limit 10, where
gate and up pre-activations clamp and limit 0 is the control):
  * score "softmax": s = exp(L - max_e L) / sum_e exp(L - max_e L) over the
    token's E logits; the bias, if any, still only selects; a row with a NaN
    logit scores NaN throughout;
  * norm_topk off: w_j = s[idx_j] * scale, no division;
  * swiglu_limit L > 0: g <- min(g, L), u <- clamp(u, -L, L) before
    silu(g) * u, NaN kept (0 turns the clamp off).

Skip slot (TensorFold issue #548, "Paths your experts test does not reach",
the "skip a slot" row: the block's 9-slot plan is top-8 plus the shared
expert's id 288, over 289 plan experts, with expert 288 skipped; the result
equals the 8-slot form and the skipped slot's rows are left untouched):
  * the plan is built over the plan experts as usual (the skip id is an
    ordinary expert there);
  * the expert stage computes nothing for pairs routed to the skip id, and
    the combine leaves them out: acc = sum over the kept slots, in slot order.

Shared expert (vllm.cpp PR #684, "The finding that justifies the row": the
combine multiplies the routed sum by the routed scale BEFORE the shared
expert's output is added; the shared output itself is not scaled):
    y = out_scale * sum_j w_j * o_j  +  down_s(act(up_s(x)))
with the shared expert's own width I_s, the block's activation, weight 1.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "bf16_to_f64", "router_logits", "sigmoid", "select_topk", "select_topk_bruteforce",
    "route", "tie_margins", "plan", "dequant_affine4", "e2m1_value", "e4m3_value", "dequant_nvfp4", "silu", "swiglu", "relu2", "softmax",
    "clamp_swiglu_inputs",
    "expert_outputs", "combine", "moe_block", "moe_block_all_experts", "shared_expert", "experts_block",
    "BM",
]

BM = 128  # rows of one GEMM M-tile; the plan's tile table counts ceil(count / BM) per expert


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact: a bf16 value is an fp32 value with
    the low 16 mantissa bits zero)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------- route

def router_logits(x_bits: np.ndarray, w_router: np.ndarray) -> np.ndarray:
    """L[t, e] = sum_h x[t, h] * Wr[e, h] in float64 (fp32 router weights;
    TensorFold pull #1492, "What")."""
    x = bf16_to_f64(x_bits)
    wr = np.asarray(w_router, dtype=np.float32).astype(np.float64)
    return x @ wr.T


def sigmoid(L: np.ndarray) -> np.ndarray:
    """s = 1 / (1 + exp(-L)); NaN in gives NaN out, -inf gives 0, +inf gives 1."""
    L = np.asarray(L, dtype=np.float64)
    with np.errstate(over="ignore", invalid="ignore"):
        return 1.0 / (1.0 + np.exp(-L))


def softmax(L: np.ndarray) -> np.ndarray:
    """Row-wise exp(L - max) / sum(exp(L - max)); a NaN anywhere in a row
    makes the whole row NaN."""
    L = np.asarray(L, dtype=np.float64)
    with np.errstate(over="ignore", invalid="ignore"):
        z = np.exp(L - L.max(axis=-1, keepdims=True))
        return z / z.sum(axis=-1, keepdims=True)


def select_topk(c: np.ndarray, k: int) -> np.ndarray:
    """Distinct top-k expert ids per row, in rank order.

    Rank order: c descending; equal c -> lower index first; NaN after every
    number (then lower index first).  -0.0 and +0.0 compare equal.  Written
    as a sort of all E experts by that key, keeping the first k."""
    c = np.asarray(c, dtype=np.float64)
    T, E = c.shape
    assert 1 <= k <= E
    isnan = np.isnan(c)
    neg = np.where(isnan, 0.0, -c)            # ascending -c  ==  descending c
    neg = np.where(neg == 0.0, 0.0, neg)      # fold -0.0 onto +0.0
    ids = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((ids, neg, isnan), axis=-1)   # last key is primary
    return order[:, :k].astype(np.int64)


def select_topk_bruteforce(c_row, k: int):
    """Pure-Python k-round argmax over one row (tiny inputs only): each round
    takes the unpicked expert maximising (c, -e), NaN below every number."""
    E = len(c_row)
    picked = []
    for _ in range(k):
        best = None
        for e in range(E):
            if e in picked:
                continue
            if best is None:
                best = e
                continue
            ce, cb = float(c_row[e]), float(c_row[best])
            if np.isnan(cb) and not np.isnan(ce):
                best = e
            elif not np.isnan(ce) and not np.isnan(cb) and ce > cb:
                best = e
        picked.append(best)
    return picked


def route(*, k: int, eps: float, scale: float, expert_bias, x_bits=None, w_router=None,
          logits=None, score: str = "sigmoid", norm_topk: bool = True):
    """Sigmoid (or softmax) routing with a selection-only expert bias.

    Exactly one of (x_bits with w_router) or logits (fp32, widened) is given.
    Returns a dict with L, s, c, idx (T, k) and w (T, k):
        s = sigmoid(L) (or softmax(L));  c = s + bias (selection only);
        idx = top-k of c;
        w_j = s[idx_j] / (sum_j s[idx_j] + eps) * scale   (sum in slot order),
        or s[idx_j] * scale with norm_topk off.
    """
    if (x_bits is None) == (logits is None):
        raise ValueError("give exactly one of x_bits or logits")
    if logits is None:
        L = router_logits(x_bits, w_router)
    else:
        L = np.asarray(logits, dtype=np.float32).astype(np.float64)
    if score == "sigmoid":
        s = sigmoid(L)
    elif score == "softmax":
        s = softmax(L)
    else:
        raise ValueError(score)
    b = np.asarray(expert_bias, dtype=np.float32).astype(np.float64)
    c = s + b[None, :]
    idx = select_topk(c, k)
    sel = np.take_along_axis(s, idx, axis=1)
    tot = np.zeros(sel.shape[0])
    for j in range(k):
        tot = tot + sel[:, j]
    w = sel / (tot + eps)[:, None] * scale if norm_topk else sel * scale
    return {"L": L, "s": s, "c": c, "idx": idx, "w": w}


def tie_margins(c: np.ndarray, k: int) -> np.ndarray:
    """Smallest gap between adjacent ranks among the first min(k+1, E) ranks
    of each row (numbers only; a gap next to a NaN counts as infinite).  A row
    whose margin is below 1e-6 is a near-tie: its picks may legitimately
    differ under fp32 arithmetic."""
    c = np.asarray(c, dtype=np.float64)
    T, E = c.shape
    m = min(k + 1, E)
    order = select_topk(c, m)
    v = np.take_along_axis(c, order, axis=1)
    if m < 2:
        return np.full(T, np.inf)
    gaps = v[:, :-1] - v[:, 1:]
    gaps = np.where(np.isnan(gaps), np.inf, gaps)
    return gaps.min(axis=1)


# --------------------------------------------------------------------------- plan

def plan(idx: np.ndarray, E: int, bm: int = BM):
    """Grouped expert plan of the (T, k) picks.

    Pair p = t * k + j.  counts[e] = #pairs routed to e; offsets = exclusive
    scan (E + 1 entries); perm lists the pairs sorted stably by (e, p);
    inv[p] is the sorted position of pair p; tiles = exclusive scan of
    ceil(counts / bm) (E + 1 entries), the M-tile table."""
    flat = np.asarray(idx, dtype=np.int64).ravel()
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    perm = np.argsort(flat, kind="stable")
    inv = np.empty_like(perm)
    inv[perm] = np.arange(flat.size)
    mt = (counts + bm - 1) // bm
    tiles = np.concatenate([[0], np.cumsum(mt)])
    return {"counts": counts, "offsets": offsets, "perm": perm, "inv": inv, "tiles": tiles}


# --------------------------------------------------------------------------- experts

def dequant_affine4(q_words: np.ndarray, scale_bits: np.ndarray, bias_bits: np.ndarray) -> np.ndarray:
    """MLX-style affine 4-bit, group 64 along K, to float64: w = scale * q + bias.

    q_words (..., N, K/8) uint32 with 8 codes each, low nibble = lowest k;
    scale/bias (..., N, K/64) bf16 bits."""
    p = np.asarray(q_words, dtype=np.uint32)
    codes = np.stack([(p >> np.uint32(4 * i)) & np.uint32(0xF) for i in range(8)], axis=-1)
    codes = codes.reshape(*p.shape[:-1], p.shape[-1] * 8).astype(np.float64)
    s = np.repeat(bf16_to_f64(scale_bits), 64, axis=-1)
    b = np.repeat(bf16_to_f64(bias_bits), 64, axis=-1)
    return s * codes + b


def e2m1_value(code) -> np.ndarray:
    """Value of 4-bit e2m1 codes: bit 3 sign, bits 2-1 exponent e, bit 0
    mantissa m; e == 0 is subnormal (m * 0.5), else 2^(e - 1) * (1 + m / 2)."""
    c = np.asarray(code).astype(np.int64) & 0xF
    e = (c >> 1) & 3
    m = (c & 1).astype(np.float64)
    mag = np.where(e == 0, m * 0.5, np.ldexp(1.0 + m / 2.0, e - 1))
    return np.where(c & 8, -mag, mag)


def e4m3_value(byte) -> np.ndarray:
    """Value of e4m3 ("fn") bytes: bit 7 sign, bits 6-3 exponent e (bias 7),
    bits 2-0 mantissa m; e == 0 is subnormal (m / 8 * 2^-6); exponent 15 with
    mantissa 7 is NaN (no infinities)."""
    b = np.asarray(byte).astype(np.int64) & 0xFF
    e = (b >> 3) & 0xF
    m = (b & 7).astype(np.float64)
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    mag = np.where((e == 15) & (b & 7 == 7), np.nan, mag)
    return np.where(b & 0x80, -mag, mag)


def dequant_nvfp4(codes: np.ndarray, scales: np.ndarray, global_scale: float) -> np.ndarray:
    """NVFP4 (ModelOpt layout) to float64: w[n, k] = e2m1(q[n, k]) *
    e4m3(scale[n, k // 16]) * global_scale.

    codes (..., N, K/2) uint8 with the lower k in the low nibble; scales
    (..., N, K/16) uint8 e4m3 bytes; global_scale the fp32 weight_scale_2."""
    p = np.asarray(codes, dtype=np.uint8)
    q = np.stack([p & 0xF, p >> 4], axis=-1).reshape(*p.shape[:-1], p.shape[-1] * 2)
    s = np.repeat(e4m3_value(scales), 16, axis=-1)
    return e2m1_value(q) * s * float(np.float32(global_scale))


def silu(g):
    with np.errstate(over="ignore", invalid="ignore"):
        return g / (1.0 + np.exp(-g))


def swiglu(g, u):
    """SwiGLU activation: silu(gate) * up."""
    return silu(g) * u


def relu2(u):
    """relu(u)^2 with NaN kept: (u > 0 ? u : (isnan(u) ? u : 0))^2."""
    r = np.where(u > 0, u, np.where(np.isnan(u), u, 0.0))
    return r * r


def _expert_w(inp, which: str, e: int) -> np.ndarray:
    """float64 (N, K) weight of expert e (which = 'w1' or 'w2')."""
    if inp.wl.fmt == "bf16":
        return bf16_to_f64(getattr(inp, which + "_bits")[e])
    if inp.wl.fmt == "nvfp4":
        return dequant_nvfp4(getattr(inp, which + "_q")[e], getattr(inp, which + "_scale")[e],
                             getattr(inp, which + "_global")[e])
    return dequant_affine4(getattr(inp, which + "_q")[e], getattr(inp, which + "_scale")[e],
                           getattr(inp, which + "_bias")[e])


def clamp_swiglu_inputs(g, u, limit: float):
    """g <- min(g, limit), u <- clamp(u, -limit, limit), NaN kept; limit 0
    leaves both as they are."""
    if not limit:
        return g, u
    g = np.where(g > limit, limit, g)
    u = np.where(u > limit, limit, np.where(u < -limit, -limit, u))
    return g, u


def _act(h1: np.ndarray, act: str, I: int, limit: float = 0.0) -> np.ndarray:
    if act == "swiglu":
        return swiglu(*clamp_swiglu_inputs(h1[:, :I], h1[:, I:2 * I], limit))
    if act == "relu2":
        return relu2(h1)
    raise ValueError(act)


def expert_outputs(inp, idx: np.ndarray, tokens: np.ndarray, skip=None) -> np.ndarray:
    """o[r, j, :] = down_e(act(up_e(x_t))) for t = tokens[r], e = idx[r, j].

    For each expert, the rows routed to it are stacked and multiplied by its
    weights (a matmul per expert); nothing else is reordered.  Pairs routed to
    the expert id ``skip`` are not computed (their o stays 0; the skipped
    expert has no weights)."""
    wl = inp.wl
    x = bf16_to_f64(inp.x_bits[tokens])
    R, k = idx.shape
    o = np.zeros((R, k, wl.H))
    for e in np.unique(idx):
        if skip is not None and e == skip:
            continue
        rr, jj = np.nonzero(idx == e)
        W1 = _expert_w(inp, "w1", int(e))
        W2 = _expert_w(inp, "w2", int(e))
        with np.errstate(invalid="ignore", over="ignore"):
            a = _act(x[rr] @ W1.T, wl.act, wl.I, wl.swiglu_limit)
            o[rr, jj] = a @ W2.T
    return o


def _shared_w(inp, which: str) -> np.ndarray:
    """float64 (N, K) weight of the shared expert."""
    sh = inp.shared
    if inp.wl.fmt == "bf16":
        return bf16_to_f64(sh[which + "_bits"][0])
    if inp.wl.fmt == "nvfp4":
        return dequant_nvfp4(sh[which + "_q"][0], sh[which + "_scale"][0], sh[which + "_global"][0])
    return dequant_affine4(sh[which + "_q"][0], sh[which + "_scale"][0], sh[which + "_bias"][0])


def shared_expert(inp, tokens: np.ndarray) -> np.ndarray:
    """sh[r] = down_s(act(up_s(x_t))) for t = tokens[r]: the shared expert,
    on every token, with weight 1."""
    wl = inp.wl
    x = bf16_to_f64(inp.x_bits[tokens])
    with np.errstate(invalid="ignore", over="ignore"):
        a = _act(x @ _shared_w(inp, "w1").T, wl.act, wl.shared_I, wl.swiglu_limit)
        return a @ _shared_w(inp, "w2").T


def combine(o: np.ndarray, w: np.ndarray, out_scale: float, dtype=np.float64, keep=None):
    """acc = sum_j w_j * o_j in slot order, then y = out_scale * acc: one
    multiply on the finished sum (vllm.cpp PR #684).  ``dtype`` float32 gives
    the fp32 mirror used to pin the order of operations.  ``keep`` (R, k)
    bool leaves the unkept slots out of the sum (skip slots)."""
    o = np.asarray(o).astype(dtype)
    w = np.asarray(w).astype(dtype)
    acc = np.zeros(o.shape[0:1] + o.shape[2:], dtype=dtype)
    for j in range(o.shape[1]):
        term = w[:, j, None] * o[:, j]
        if keep is not None:
            term = np.where(np.asarray(keep)[:, j, None], term, dtype(0))
        acc = acc + term
    return acc, dtype(out_scale) * acc


def moe_block(inp, tokens=None, *, use_logits=None, idx=None):
    """Whole block for the chosen token rows (default: all).

    Returns route dict plus 'acc' (unscaled routed sum) and 'y'.  ``idx``
    overrides the picks (to evaluate the expert stage on another routing);
    weights are then recomputed from the oracle's s for those picks."""
    wl = inp.wl
    T = wl.T
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    if use_logits is not None:
        r = route(k=wl.k, eps=wl.eps, scale=wl.router_scale, expert_bias=inp.expert_bias,
                  logits=np.asarray(use_logits)[tokens], score=wl.score, norm_topk=wl.norm_topk)
    else:
        r = route(k=wl.k, eps=wl.eps, scale=wl.router_scale, expert_bias=inp.expert_bias,
                  x_bits=inp.x_bits[tokens], w_router=inp.w_router, score=wl.score,
                  norm_topk=wl.norm_topk)
    if idx is not None:
        idx = np.asarray(idx, dtype=np.int64)
        sel = np.take_along_axis(r["s"], idx, axis=1)
        tot = np.zeros(sel.shape[0])
        for j in range(wl.k):
            tot = tot + sel[:, j]
        r["idx"] = idx
        r["w"] = sel / (tot + wl.eps)[:, None] * wl.router_scale if wl.norm_topk else sel * wl.router_scale
    o = expert_outputs(inp, r["idx"], tokens)
    acc, y = combine(o, r["w"], wl.out_scale)
    if wl.shared_I:
        sh = shared_expert(inp, tokens)
        y = y + sh                                   # after the routed scale, unscaled
        r["shared"] = sh
    r.update({"tokens": tokens, "acc": acc, "y": y})
    return r


def experts_block(inp, idx, w, tokens=None, skip=None):
    """The expert stage and combine on given picks and weights: for token rows
    ``tokens`` (default all), idx (R, k) plan-expert ids and w (R, k) weights,
    returns (acc, y) with the pairs routed to ``skip`` computed nowhere and left
    out of the sum (the 9-slot plan of TensorFold issue #548: top-8 plus the
    shared id, that id skipped)."""
    tokens = np.arange(inp.wl.T) if tokens is None else np.asarray(tokens)
    idx = np.asarray(idx, dtype=np.int64)
    o = expert_outputs(inp, idx, tokens, skip=skip)
    keep = None if skip is None else idx != skip
    return combine(o, w, inp.wl.out_scale, keep=keep)


def moe_block_all_experts(inp):
    """Brute force: run every token through all E experts and weight each
    expert's output by the token's routing weight for it (zero if unpicked).
    Tiny inputs only."""
    wl = inp.wl
    r = route(k=wl.k, eps=wl.eps, scale=wl.router_scale, expert_bias=inp.expert_bias,
              x_bits=inp.x_bits, w_router=inp.w_router, score=wl.score, norm_topk=wl.norm_topk)
    x = bf16_to_f64(inp.x_bits)
    dense_w = np.zeros((wl.T, wl.E))
    for j in range(wl.k):
        dense_w[np.arange(wl.T), r["idx"][:, j]] += r["w"][:, j]
    acc = np.zeros((wl.T, wl.H))
    for e in range(wl.E):
        with np.errstate(invalid="ignore", over="ignore"):
            a = _act(x @ _expert_w(inp, "w1", e).T, wl.act, wl.I, wl.swiglu_limit)
            acc += dense_w[:, e, None] * (a @ _expert_w(inp, "w2", e).T)
    return acc, wl.out_scale * acc
