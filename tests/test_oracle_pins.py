"""Pins of the float64 oracle to facts other than itself.

Each test checks the oracle against something it does not compute with:
a brute-force loop, a closed form, a library routine (scipy's expit), an
invariant the pages state, or hand-decoded codes.  Every test is chosen so a
plausible slip in the oracle (a dropped term, the bias in the weights, a
swapped gate/up half, a transposed weight, a folded scale) fails it.
"""
import dataclasses
import math

import numpy as np
import pytest
import scipy.special

import oracle as O
from sigmoid_top_routing_b200 import inputs as G


def _rng(seed=1):
    return np.random.default_rng(seed)


# ------------------------------------------------------------------ selection

def _nasty_scores(rng, T, E):
    c = rng.uniform(-0.2, 1.2, size=(T, E))
    c[rng.random((T, E)) < 0.1] = np.nan
    c[0] = np.nan                                      # an all-NaN row
    c[1, :] = 0.25                                     # all tied
    c[2, : E // 2] = -0.0
    c[2, E // 2:] = 0.0                                # signed zeros tie
    c[3, ::3] = -np.inf
    c[4] = np.round(c[4], 1)                           # coarse grid, many ties
    return c


@pytest.mark.parametrize("E,k", [(8, 2), (8, 8), (32, 4), (64, 6), (5, 1)])
def test_select_matches_bruteforce(E, k):
    c = _nasty_scores(_rng(E * 31 + k), 40, E)
    got = O.select_topk(c, k)
    for t in range(c.shape[0]):
        assert list(got[t]) == O.select_topk_bruteforce(c[t], k), t


def test_select_invariants():
    rng = _rng(7)
    E, k = 64, 6
    c = _nasty_scores(rng, 200, E)
    idx = O.select_topk(c, k)
    for t in range(c.shape[0]):
        row = idx[t]
        assert len(set(row.tolist())) == k                       # k distinct
        assert row.min() >= 0 and row.max() < E
        vals = c[t, row]
        fin = vals[~np.isnan(vals)]
        assert np.all(np.diff(fin) <= 0)                        # non-increasing along slots
        nan_pos = np.nonzero(np.isnan(vals))[0]
        if len(nan_pos):                                        # NaN picks only after numbers
            assert np.all(np.isnan(vals[nan_pos[0]:]))
        rest = np.setdiff1d(np.arange(E), row)
        rest_fin = c[t, rest][~np.isnan(c[t, rest])]
        if len(fin) == k and len(rest_fin):
            assert rest_fin.max() <= fin.min()                  # nothing unpicked is larger


def test_all_nan_row_picks_distinct_low_ids_and_nan_weights():
    """TensorFold pull #1492, "Verification": an all-NaN router row once
    picked expert 0 twice; picks must be distinct."""
    E, k = 32, 4
    L = np.full((3, E), np.nan, dtype=np.float32)
    L[1] = np.linspace(-1, 1, E)
    r = O.route(k=k, eps=1e-6, scale=1.0, expert_bias=np.zeros(E, np.float32), logits=L)
    assert r["idx"][0].tolist() == [0, 1, 2, 3]
    assert r["idx"][2].tolist() == [0, 1, 2, 3]
    assert np.isnan(r["w"][0]).all()
    assert np.isfinite(r["w"][1]).all()


# ------------------------------------------------------------------ sigmoid

def test_sigmoid_against_library_and_special_values():
    x = np.concatenate([np.linspace(-40, 40, 1001), [0.0, -0.0, np.inf, -np.inf, np.log(3.0)]])
    s = O.sigmoid(x)
    np.testing.assert_allclose(s, scipy.special.expit(x), rtol=1e-15, atol=0)
    assert s[-5] == 0.5 and s[-4] == 0.5 and s[-3] == 1.0 and s[-2] == 0.0
    assert O.sigmoid(np.array([0.0]))[0] == 0.5
    assert abs(O.sigmoid(np.array([math.log(3.0)]))[0] - 0.75) < 1e-15
    assert np.isnan(O.sigmoid(np.array([np.nan]))[0])


# ------------------------------------------------------------------ weights

def _route_case(seed=3, T=64, E=32, H=64, k=4, scale=1.0, eps=1e-6):
    rng = _rng(seed)
    x = G.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    wr = (rng.standard_normal((E, H)) * 0.3).astype(np.float32)
    b = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    return x, wr, b, O.route(k=k, eps=eps, scale=scale, expert_bias=b, x_bits=x, w_router=wr)


def test_weights_are_bias_free_ratios():
    """TileGym PR #187, "Weight layout and routing": the gathered weights stay
    unbiased, so w_i / w_j = s_i / s_j for every pair of slots."""
    _, _, b, r = _route_case()
    s_sel = np.take_along_axis(r["s"], r["idx"], axis=1)
    c_sel = np.take_along_axis(r["c"], r["idx"], axis=1)
    ratio_w = r["w"][:, 1:] / r["w"][:, :1]
    np.testing.assert_allclose(ratio_w, s_sel[:, 1:] / s_sel[:, :1], rtol=1e-14)
    # the mutant that gathers c (score + bias) instead of s must not pass
    assert not np.allclose(ratio_w, c_sel[:, 1:] / c_sel[:, :1], rtol=1e-6)


@pytest.mark.parametrize("scale,eps", [(1.0, 1e-6), (2.5, 1e-6), (0.7, 1e-20)])
def test_weight_sum_closed_form(scale, eps):
    """sum_j w_j = scale * S / (S + eps) with S the sum of the picked scores."""
    _, _, _, r = _route_case(scale=scale, eps=eps)
    S = np.take_along_axis(r["s"], r["idx"], axis=1).sum(axis=1)
    np.testing.assert_allclose(r["w"].sum(axis=1), scale * S / (S + eps), rtol=1e-14)


def test_bias_only_moves_selection():
    """Nudging the bias without changing the picks leaves the weights bit-identical."""
    x, wr, b, r = _route_case()
    r2 = O.route(k=4, eps=1e-6, scale=1.0, expert_bias=b + np.float32(1e-9), x_bits=x, w_router=wr)
    same = (r2["idx"] == r["idx"]).all(axis=1)
    assert same.sum() > 50
    assert np.array_equal(r2["w"][same], r["w"][same])


def test_zero_router_closed_form():
    """W_router = 0: every score is 1/2, the picks are the top-k of the bias,
    and every weight is scale * 0.5 / (0.5 k + eps)."""
    E, k, T, H, scale, eps = 16, 4, 5, 32, 2.0, 1e-6
    rng = _rng(11)
    x = G.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    b = rng.permutation(np.linspace(-0.1, 0.1, E)).astype(np.float32)
    r = O.route(k=k, eps=eps, scale=scale, expert_bias=b, x_bits=x, w_router=np.zeros((E, H), np.float32))
    want = np.argsort(-b)[:k]
    assert all(r["idx"][t].tolist() == want.tolist() for t in range(T))
    np.testing.assert_allclose(r["w"], scale * 0.5 / (0.5 * k + eps), rtol=1e-15)


def test_router_logits_bruteforce():
    rng = _rng(5)
    x = G.f32_to_bf16_bits(rng.standard_normal((3, 16)).astype(np.float32))
    wr = rng.standard_normal((4, 16)).astype(np.float32)
    L = O.router_logits(x, wr)
    xf = G.bf16_bits_to_f32(x)
    for t in range(3):
        for e in range(4):
            acc = math.fsum(float(xf[t, h]) * float(wr[e, h]) for h in range(16))
            assert abs(L[t, e] - acc) <= 1e-12 * max(1.0, abs(acc))


def test_tie_margin_definition():
    c = np.array([[0.9, 0.5, 0.5 + 5e-7, 0.1, 0.0],      # in-set near tie
                  [0.9, 0.8, 0.7, 0.6, 0.6 - 3e-7],      # ranks 4 and 5 nearly tie
                  [0.9, 0.7, 0.5, 0.3, 0.1]])
    m = O.tie_margins(c, 3)
    assert m[0] < 1e-6
    assert m[1] == pytest.approx(0.1)                      # ranks 1..4 only: 0.6 vs 0.6-3e-7 is rank 5
    assert m[2] == pytest.approx(0.2)
    m4 = O.tie_margins(c, 4)
    assert m4[1] < 1e-6                                    # now the boundary is ranks 4/5


# ------------------------------------------------------------------ plan

def test_plan_bruteforce():
    rng = _rng(9)
    T, k, E = 77, 3, 10
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    p = O.plan(idx, E, bm=8)
    flat = idx.ravel().tolist()
    want_perm = sorted(range(T * k), key=lambda q: (flat[q], q))
    assert p["perm"].tolist() == want_perm
    for q in range(T * k):
        assert p["perm"][p["inv"][q]] == q
    for e in range(E):
        n = flat.count(e)
        assert p["counts"][e] == n
        assert p["offsets"][e + 1] - p["offsets"][e] == n
        assert p["tiles"][e + 1] - p["tiles"][e] == -(-n // 8)
    assert p["offsets"][0] == 0 and p["offsets"][-1] == T * k


# ------------------------------------------------------------------ experts

def _small(name, **over):
    base = dict(seed=0)
    base.update(over)
    return G.Workload(name, **base)


SMALL = [
    _small("tiny_like", T=16, H=256, E=8, k=2, I=128),
    _small("lfm2_small", T=12, H=128, E=32, k=4, I=64),
    _small("relu2_small", T=20, H=128, E=16, k=6, I=64, act="relu2", out_scale=2.5),
    _small("affine4_small", T=9, H=128, E=8, k=4, I=64, fmt="affine4"),
]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_sparse_oracle_equals_all_expert_bruteforce(wl):
    inp = G.make_inputs(wl)
    r = O.moe_block(inp)
    acc_b, y_b = O.moe_block_all_experts(inp)
    np.testing.assert_allclose(r["y"], y_b, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(r["acc"], acc_b, rtol=1e-12, atol=1e-14)


def test_zero_input_gives_zero_output():
    for wl in SMALL:
        inp = G.make_inputs(wl)
        inp.x_bits[:] = 0
        r = O.moe_block(inp)
        assert np.all(r["y"] == 0.0), wl.name


def _one_hot_inputs(act):
    """x = e_{h0}; expert e's up rows hold g_i / u_i at column h0 only; down
    sends activation i to output (i + 1) mod I (a cyclic shift, so a
    transposed down matrix is visible).  Then o_e[(i + 1) % I] = act(g_i, u_i)."""
    T, H, E, k, I = 4, 64, 4, 2, 8
    wl = G.Workload("onehot", T=T, H=H, E=E, k=k, I=I, act=act)
    n1 = 2 * I if act == "swiglu" else I
    h0 = 5
    x = np.zeros((T, H), np.float32)
    x[:, h0] = 1.0
    g = np.array([0.0, 1.0, -1.0, 2.0, -4.0, 0.5, 3.0, -0.25], np.float32)
    u = np.array([1.0, 2.0, -3.0, 0.5, 1.0, -2.0, 4.0, 8.0], np.float32)
    w1 = np.zeros((E, n1, H), np.float32)
    w2 = np.zeros((E, H, I), np.float32)
    for e in range(E):
        if act == "swiglu":
            w1[e, :I, h0] = g * (e + 1)
            w1[e, I:, h0] = u
        else:
            w1[e, :, h0] = u * (e + 1) * np.where(np.arange(I) % 2 == 0, 1, -1)
        w2[e, :I, :] = np.roll(np.eye(I, dtype=np.float32), 1, axis=0)
    inp = G.MoEInputs(wl=wl, x_bits=G.f32_to_bf16_bits(x),
                      w_router=_rng(2).standard_normal((E, H)).astype(np.float32),
                      expert_bias=np.zeros(E, np.float32),
                      w1_bits=G.f32_to_bf16_bits(w1), w2_bits=G.f32_to_bf16_bits(w2))
    return inp, g, u


def test_one_hot_swiglu_closed_form():
    """Gate rows first, then up (TileGym PR #187): o[n] = silu(g_n) * u_n with
    silu(z) = z * expit(z) from scipy; a gate/up swap or a transposed weight fails."""
    inp, g, u = _one_hot_inputs("swiglu")
    r = O.moe_block(inp)
    for t in range(inp.wl.T):
        want = np.zeros(inp.wl.H)
        for j in range(inp.wl.k):
            e = r["idx"][t, j]
            z = g.astype(np.float64) * (e + 1)
            o = np.zeros(inp.wl.H)
            o[:8] = np.roll(z * scipy.special.expit(z) * u, 1)
            want += r["w"][t, j] * o
        np.testing.assert_allclose(r["y"][t], want, rtol=1e-13, atol=1e-15)


def test_one_hot_relu2_closed_form():
    """relu^2 = max(u, 0)^2 (bloomery PR #235 "What"; vllm.cpp PR #684)."""
    inp, _, u = _one_hot_inputs("relu2")
    r = O.moe_block(inp)
    for t in range(inp.wl.T):
        want = np.zeros(inp.wl.H)
        for j in range(inp.wl.k):
            e = r["idx"][t, j]
            z = u.astype(np.float64) * (e + 1) * np.where(np.arange(8) % 2 == 0, 1, -1)
            o = np.zeros(inp.wl.H)
            o[:8] = np.roll(np.maximum(z, 0.0) ** 2, 1)
            want += r["w"][t, j] * o
        np.testing.assert_allclose(r["y"][t], want, rtol=1e-13, atol=1e-15)


def test_relu2_special_values():
    u = np.array([3.0, -2.0, 0.0, -0.0, np.nan, np.inf, -np.inf])
    v = O.relu2(u)
    assert v[0] == 9.0 and v[1] == 0.0 and v[2] == 0.0 and v[3] == 0.0
    assert np.isnan(v[4])                    # NaN stays NaN (not fmax's 0)
    assert v[5] == np.inf and v[6] == 0.0
    # mutant: relu instead of relu^2
    assert not np.array_equal(v[:1], np.maximum(u[:1], 0))


def test_swiglu_special_values():
    assert O.swiglu(np.array([0.0]), np.array([5.0]))[0] == 0.0
    v = O.swiglu(np.array([math.log(3.0)]), np.array([2.0]))[0]
    assert abs(v - 2.0 * 0.75 * math.log(3.0)) < 1e-15        # sigmoid(ln 3) = 3/4


def test_out_scale_is_linear():
    wl = SMALL[2]
    inp = G.make_inputs(wl)
    y25 = O.moe_block(inp)["y"]
    inp1 = dataclasses.replace(inp, wl=dataclasses.replace(wl, out_scale=1.0))
    y1 = O.moe_block(inp1)["y"]
    np.testing.assert_allclose(y25, 2.5 * y1, rtol=1e-15)


def test_routed_scale_applied_after_the_sum_not_folded():
    """vllm.cpp PR #684, "The finding that justifies the row": scaling the
    finished sum and folding the scale into each weight are equal in exact
    arithmetic but differ after fp32 rounding.  On decimal-grid data the two
    orders must separate (checked first, so the test cannot pass vacuously),
    and the oracle's fp32 mirror must give the scale-after-sum value."""
    rng = _rng(21)
    R, k, H, scale = 2000, 6, 8, np.float32(2.5)
    o = (rng.integers(-999, 1000, size=(R, k, H)) / 997.0).astype(np.float32)
    w = (rng.integers(1, 1000, size=(R, k)) / 1009.0).astype(np.float32)
    fold = np.zeros((R, H), np.float32)
    for j in range(k):
        fold = fold + (scale * w[:, j, None]) * o[:, j]
    acc, y = O.combine(o, w, float(scale), dtype=np.float32)
    differ = np.any(fold != y, axis=1)
    assert differ.sum() > R // 10                # the data separates the orders
    assert np.array_equal(y, scale * acc)        # one multiply on the finished sum
    assert not np.array_equal(y, fold)


# ------------------------------------------------------------------ affine-4

def test_affine4_hand_decoded_codes():
    q = np.array([[0x76543210, 0xFEDCBA98] * 4], dtype=np.uint32)       # one row, K = 64
    scale = G.f32_to_bf16_bits(np.array([[2.0]], np.float32))
    bias = G.f32_to_bf16_bits(np.array([[-1.0]], np.float32))
    w = O.dequant_affine4(q, scale, bias)
    codes = np.tile(np.arange(16), 4)
    np.testing.assert_array_equal(w[0], 2.0 * codes - 1.0)


def test_affine4_quantizer_round_trip_bound():
    """Generator check: dequantised weights lie within half a step (plus bf16
    rounding of scale/bias) of the drawn fp32 weights."""
    rng = _rng(4)
    w = (rng.standard_normal((3, 8, 128)) * 0.02).astype(np.float32)
    q, s, b = G.quantize_affine4_g64(w)
    back = O.dequant_affine4(q, s, b)
    step = np.repeat(G.bf16_bits_to_f32(s), 64, axis=-1).astype(np.float64)
    assert np.all(np.abs(back - w) <= 0.5 * step + 0.02 * np.abs(w) + 1e-3 * step + 4e-4)
    assert np.array_equal(G.unpack_affine4(q).max() <= 15, True)
