"""Pins of the oracle's router and activation variants (softmax scores,
norm_topk off, the SwiGLU input clamp) to facts other than the oracle itself:
scipy's softmax and expit, closed forms on one-hot experts written out
scalar by scalar, and the brute-force top-k.  The FAIL-first mutants at the
end plant one mistake each and require its pin to go red.

TensorFold issue #548 names the pieces: its table of what each model family
builds lists "routers (softmax, sigmoid + bias)"; its section "Paths your
experts test does not reach" runs swiglu_limit 10 (gate and up
pre-activations clamp; limit 0 is the control)."""
import dataclasses

import numpy as np
import pytest
import scipy.special

import oracle
import oracle.moe_oracle as OM
from tests import test_oracle_pins as pins


def _rng(seed):
    return np.random.default_rng(seed)


# ------------------------------------------------------------------ softmax

def test_softmax_matches_scipy_including_huge_logits():
    L = _rng(1).normal(0, 3, size=(20, 32))
    L[3] *= 400.0                                   # |L| up to ~4000: a naive exp overflows
    L[4] -= 900.0
    np.testing.assert_allclose(oracle.softmax(L), scipy.special.softmax(L, axis=-1), rtol=1e-12, atol=0)
    np.testing.assert_allclose(oracle.softmax(L).sum(axis=-1), 1.0, rtol=1e-14)


def test_softmax_row_with_a_nan_is_all_nan():
    L = _rng(2).normal(size=(3, 8))
    L[1, 5] = np.nan
    s = oracle.softmax(L)
    assert np.isnan(s[1]).all() and not np.isnan(s[[0, 2]]).any()


def test_softmax_route_closed_form():
    """Picks = brute-force top-k of p + bias; w_j = p_j / (sum_j p_j + eps) * scale,
    p = scipy's softmax of the fp32 logits."""
    T, E, k, eps, scale = 24, 16, 3, 1e-6, 1.7
    rng = _rng(3)
    L = rng.normal(0, 2, size=(T, E)).astype(np.float32)
    b = rng.uniform(-0.1, 0.1, size=E).astype(np.float32)
    r = oracle.route(k=k, eps=eps, scale=scale, expert_bias=b, logits=L, score="softmax")
    p = scipy.special.softmax(L.astype(np.float64), axis=-1)
    for t in range(T):
        picks = oracle.select_topk_bruteforce(p[t] + b.astype(np.float64), k)
        assert list(r["idx"][t]) == picks
        sel = p[t, picks]
        np.testing.assert_allclose(r["w"][t], sel / (sel.sum() + eps) * scale, rtol=1e-14)


# ------------------------------------------------------------------ norm_topk off

@pytest.mark.parametrize("score", ["sigmoid", "softmax"])
def test_norm_topk_off_keeps_the_raw_scores(score):
    """w_j = s[idx_j] * scale exactly: no division by the picked sum."""
    T, E, k, scale = 16, 8, 2, 2.5
    L = _rng(4).normal(size=(T, E)).astype(np.float32)
    r = oracle.route(k=k, eps=1e-6, scale=scale, expert_bias=np.zeros(E, np.float32), logits=L,
                     score=score, norm_topk=False)
    Ld = L.astype(np.float64)
    s = scipy.special.expit(Ld) if score == "sigmoid" else scipy.special.softmax(Ld, axis=-1)
    np.testing.assert_allclose(r["w"], np.take_along_axis(s, r["idx"], axis=1) * scale, rtol=1e-14)
    assert not np.allclose(r["w"].sum(axis=1), scale)        # would hold if it normalised


# ------------------------------------------------------------------ swiglu_limit

def _clamped_swiglu_scalar(g, u, lim):
    g = lim if g > lim else g                       # gate: clamped from above only
    u = lim if u > lim else (-lim if u < -lim else u)
    return g * scipy.special.expit(g) * u


@pytest.mark.parametrize("lim", [1.5, 3.0])
def test_swiglu_limit_one_hot_closed_form(lim):
    """One-hot experts (gate g_i (e + 1), up u_i, down a cyclic shift): with the
    clamp o[(i + 1) % I] = silu(min(g, L)) * clamp(u, -L, L), scalar by scalar."""
    inp, g, u = pins._one_hot_inputs("swiglu")
    inp = dataclasses.replace(inp, wl=dataclasses.replace(inp.wl, swiglu_limit=lim))
    r = oracle.moe_block(inp)
    fired = 0
    for t in range(inp.wl.T):
        want = np.zeros(inp.wl.H)
        for j in range(inp.wl.k):
            e = r["idx"][t, j]
            act = np.zeros(8)
            for i in range(8):
                z = float(g[i]) * (e + 1)
                act[i] = _clamped_swiglu_scalar(z, float(u[i]), lim)
                fired += z > lim or abs(float(u[i])) > lim
            o = np.zeros(inp.wl.H)
            o[:8] = np.roll(act, 1)
            want += r["w"][t, j] * o
        np.testing.assert_allclose(r["y"][t], want, rtol=1e-13, atol=1e-15)
    assert fired > 0                                 # the clamp did fire on these inputs


def test_swiglu_limit_zero_is_off_and_nan_stays():
    g = np.array([5.0, -7.0, np.nan, 0.5])
    u = np.array([-9.0, 9.0, 1.0, np.nan])
    g0, u0 = oracle.clamp_swiglu_inputs(g, u, 0.0)
    assert np.array_equal(g0, g, equal_nan=True) and np.array_equal(u0, u, equal_nan=True)
    g1, u1 = oracle.clamp_swiglu_inputs(g, u, 2.0)
    assert list(g1[:2]) == [2.0, -7.0] and list(u1[:3]) == [-2.0, 2.0, 1.0]
    assert np.isnan(g1[2]) and np.isnan(u1[3])


# ------------------------------------------------------------------ FAIL-first mutants

def _expect_red(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_mutant_gate_clamped_from_below_too(monkeypatch):
    def bad(g, u, limit):
        if not limit:
            return g, u
        return np.clip(g, -limit, limit), np.clip(u, -limit, limit)
    monkeypatch.setattr(OM, "clamp_swiglu_inputs", bad)
    _expect_red(test_swiglu_limit_one_hot_closed_form, 1.5)


def test_mutant_softmax_without_max_shift(monkeypatch):
    def bad(L):
        with np.errstate(over="ignore", invalid="ignore"):
            z = np.exp(np.asarray(L, dtype=np.float64))
            return z / z.sum(axis=-1, keepdims=True)
    monkeypatch.setattr(OM, "softmax", bad)
    monkeypatch.setattr(oracle, "softmax", bad)
    _expect_red(test_softmax_matches_scipy_including_huge_logits)


def test_mutant_norm_flag_ignored(monkeypatch):
    real = OM.route

    def bad(**kw):
        kw = dict(kw)
        kw["norm_topk"] = True
        return real(**kw)
    monkeypatch.setattr(oracle, "route", bad)
    _expect_red(test_norm_topk_off_keeps_the_raw_scores, "sigmoid")


# ------------------------------------------------------------------ shared expert

def _with_shared(inp, sw1, sw2, shared_I, **wl_over):
    wl = dataclasses.replace(inp.wl, shared_I=shared_I, **wl_over)
    import sigmoid_top_routing_b200.inputs as G
    return dataclasses.replace(inp, wl=wl, shared={"w1_bits": G.f32_to_bf16_bits(sw1[None]),
                                                   "w2_bits": G.f32_to_bf16_bits(sw2[None])})


def test_shared_expert_one_hot_closed_form():
    """Routed experts zeroed (their outputs are exactly 0); the shared expert of
    width 12 holds g / u at column h0 and shifts activation i to output i + 1:
    y[t, (i + 1) % 12] = silu(g_i) * u_i, whatever the routing."""
    inp, _, _ = pins._one_hot_inputs("swiglu")
    inp = dataclasses.replace(inp, w1_bits=np.zeros_like(inp.w1_bits))
    Is, H = 12, inp.wl.H
    g = np.arange(-3.0, 3.0, 0.5).astype(np.float32)          # exact in bf16
    u = np.arange(2.0, -1.0, -0.25).astype(np.float32)
    sw1 = np.zeros((2 * Is, H), np.float32)
    sw1[:Is, 5] = g                                   # x = e_5 in the one-hot inputs
    sw1[Is:, 5] = u
    sw2 = np.zeros((H, Is), np.float32)
    sw2[:Is, :] = np.roll(np.eye(Is, dtype=np.float32), 1, axis=0)
    inp = _with_shared(inp, sw1, sw2, Is, out_scale=2.5)
    r = oracle.moe_block(inp)
    gd = g.astype(np.float64)
    want = np.zeros(H)
    want[:Is] = np.roll(gd * scipy.special.expit(gd) * u, 1)
    for t in range(inp.wl.T):
        np.testing.assert_allclose(r["y"][t], want, rtol=1e-13, atol=1e-15)


def test_shared_term_is_added_after_the_routed_scale():
    """y = out_scale * acc + sh with sh computed here by an explicit loop over
    rows (relu^2, width 40); the shared term itself is not scaled."""
    import sigmoid_top_routing_b200.inputs as G
    wl = G.Workload("sh", T=6, H=64, E=4, k=2, I=32, act="relu2", out_scale=2.5)
    inp = G.make_inputs(wl)
    rng = _rng(9)
    Is = 40
    sw1 = (rng.standard_normal((Is, 64)) * 0.1).astype(np.float32)
    sw2 = (rng.standard_normal((64, Is)) * 0.1).astype(np.float32)
    inp = _with_shared(inp, sw1, sw2, Is)
    r = oracle.moe_block(inp)
    x = oracle.bf16_to_f64(inp.x_bits)
    W1 = oracle.bf16_to_f64(inp.shared["w1_bits"][0])
    W2 = oracle.bf16_to_f64(inp.shared["w2_bits"][0])
    for t in range(wl.T):
        hmid = [sum(W1[i, h] * x[t, h] for h in range(64)) for i in range(Is)]
        a = [max(v, 0.0) ** 2 for v in hmid]
        sh = np.array([sum(W2[n, i] * a[i] for i in range(Is)) for n in range(64)])
        np.testing.assert_allclose(r["y"][t], 2.5 * r["acc"][t] + sh, rtol=1e-12, atol=1e-14)
        assert not np.allclose(r["y"][t], 2.5 * (r["acc"][t] + sh), rtol=1e-6)


def test_mutant_shared_term_scaled_too(monkeypatch):
    real = OM.shared_expert
    monkeypatch.setattr(OM, "shared_expert", lambda inp, tokens: inp.wl.out_scale * real(inp, tokens))
    _expect_red(test_shared_term_is_added_after_the_routed_scale)
