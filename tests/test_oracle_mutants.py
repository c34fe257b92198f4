"""FAIL-first check of the pins: plant one plausible mistake at a time in the
oracle (on the CPU, through monkeypatch) and require the pin aimed at it to
go red.  bloomery PR #235 ("FAIL-first") and vllm.cpp PR #684 (mutations
M1-M10) run their tests the same way."""
import numpy as np
import pytest

import oracle
import oracle.moe_oracle as OM
from tests import test_oracle_pins as pins


def _patch(monkeypatch, name, fn):
    monkeypatch.setattr(OM, name, fn)
    monkeypatch.setattr(oracle, name, fn)


def _expect_red(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_mutant_bias_in_weights(monkeypatch):
    real = OM.route

    def bad(**kw):
        r = real(**kw)
        sel = np.take_along_axis(r["c"], r["idx"], axis=1)
        r["w"] = sel / (sel.sum(axis=1) + kw["eps"])[:, None] * kw["scale"]
        return r
    _patch(monkeypatch, "route", bad)
    _expect_red(pins.test_weights_are_bias_free_ratios)


def test_mutant_eps_dropped(monkeypatch):
    real = OM.route

    def bad(**kw):
        kw = dict(kw)
        kw["eps"] = 0.0
        return real(**kw)
    monkeypatch.setattr(oracle, "route", bad)
    _expect_red(pins.test_weight_sum_closed_form, 1.0, 1e-6)


def test_mutant_nan_ranks_first(monkeypatch):
    def bad(c, k):
        c = np.where(np.isnan(c), np.inf, c)
        order = np.lexsort((np.broadcast_to(np.arange(c.shape[1]), c.shape), -c), axis=-1)
        return order[:, :k]
    _patch(monkeypatch, "select_topk", bad)
    _expect_red(pins.test_select_matches_bruteforce, 32, 4)


def test_mutant_ties_to_higher_index(monkeypatch):
    def bad(c, k):
        E = c.shape[1]
        neg = np.where(np.isnan(c), 0.0, -c)
        order = np.lexsort((-np.broadcast_to(np.arange(E), c.shape), neg, np.isnan(c)), axis=-1)
        return order[:, :k]
    _patch(monkeypatch, "select_topk", bad)
    _expect_red(pins.test_select_matches_bruteforce, 8, 2)


def test_mutant_relu_not_squared(monkeypatch):
    _patch(monkeypatch, "relu2", lambda u: np.where(u > 0, u, np.where(np.isnan(u), u, 0.0)))
    _expect_red(pins.test_one_hot_relu2_closed_form)


def test_mutant_relu2_drops_nan(monkeypatch):
    _patch(monkeypatch, "relu2", lambda u: np.fmax(u, 0.0) * np.fmax(u, 0.0))
    _expect_red(pins.test_relu2_special_values)


def test_mutant_gate_up_swapped(monkeypatch):
    real = OM._act

    def bad(h1, act, I, limit=0.0):
        if act == "swiglu":
            return OM.swiglu(h1[:, I:2 * I], h1[:, :I])
        return real(h1, act, I, limit)
    monkeypatch.setattr(OM, "_act", bad)
    _expect_red(pins.test_one_hot_swiglu_closed_form)


def test_mutant_scale_folded_into_weights(monkeypatch):
    def bad(o, w, out_scale, dtype=np.float64):
        o = np.asarray(o).astype(dtype)
        w = np.asarray(w).astype(dtype)
        acc = np.zeros(o.shape[0:1] + o.shape[2:], dtype=dtype)
        for j in range(o.shape[1]):
            acc = acc + (dtype(out_scale) * w[:, j, None]) * o[:, j]
        return acc / dtype(out_scale), acc
    _patch(monkeypatch, "combine", bad)
    _expect_red(pins.test_routed_scale_applied_after_the_sum_not_folded)


def test_mutant_plan_unstable(monkeypatch):
    real = OM.plan

    def bad(idx, E, bm=OM.BM):
        p = real(idx, E, bm)
        perm = p["perm"].copy()
        for e in range(E):
            a, b = p["offsets"][e], p["offsets"][e + 1]
            perm[a:b] = perm[a:b][::-1]
        p["perm"] = perm
        return p
    _patch(monkeypatch, "plan", bad)
    _expect_red(pins.test_plan_bruteforce)


def test_mutant_affine_nibbles_reversed(monkeypatch):
    real = OM.dequant_affine4

    def bad(q, s, b):
        q = np.asarray(q, dtype=np.uint32)
        rev = np.zeros_like(q)
        for i in range(8):
            rev |= ((q >> np.uint32(4 * i)) & np.uint32(0xF)) << np.uint32(4 * (7 - i))
        return real(rev, s, b)
    _patch(monkeypatch, "dequant_affine4", bad)
    _expect_red(pins.test_affine4_hand_decoded_codes)


def test_mutant_transposed_down(monkeypatch):
    real = OM._expert_w

    def bad(inp, which, e):
        w = real(inp, which, e)
        if which == "w2":
            n = w.shape[1]
            w = w.copy()
            w[:n, :] = w[:n, :].T
        return w
    monkeypatch.setattr(OM, "_expert_w", bad)
    _expect_red(pins.test_one_hot_swiglu_closed_form)
