"""Pins of the oracle's skip-slot form (TensorFold issue #548, "Paths your
experts test does not reach", the "skip a slot" row: the block's 9-slot plan
is top-8 plus the shared expert's id, over one more plan expert than there
are routed experts, with that id skipped; the result is byte-equal to the
8-slot form and the skipped slot's rows stay untouched).

What pins it, other than the oracle itself: the routed block computed the
ordinary way (the skip form must reproduce it exactly, whatever slot the skip
id sits in), and the plan over E + 1 experts written out by hand.  A planted
mutant (drop the last slot instead of the skip id's) must go red."""
import dataclasses

import numpy as np
import pytest

import oracle
import oracle.moe_oracle as OM
from sigmoid_top_routing_b200 import inputs as G


def _small(name, T=None, **kw):
    wl = G.WORKLOADS[name]
    wl = dataclasses.replace(wl, **kw) if kw else wl
    if T is not None:
        wl = wl.with_T(T)
    return G.make_inputs(wl)


def _with_skip_slot(idx, w, E, pos):
    """Insert the skip id E with weight 1 at slot pos[t] of each row."""
    T, k = idx.shape
    idx2 = np.empty((T, k + 1), dtype=np.int64)
    w2 = np.empty((T, k + 1))
    for t in range(T):
        p = pos[t]
        idx2[t] = np.concatenate([idx[t, :p], [E], idx[t, p:]])
        w2[t] = np.concatenate([w[t, :p], [1.0], w[t, p:]])
    return idx2, w2


@pytest.mark.parametrize("name,T,kw", [
    ("tiny", None, {}),
    ("lfm2_decode_t8", None, {"H": 256, "I": 128}),
    ("nemotron_relu2_t2048", 24, {"H": 128, "I": 64, "E": 16}),
])
def test_skip_slot_last_equals_routed_block(name, T, kw):
    """The pages' form: top-k plus the shared id in the last slot; the expert
    stage with that id skipped gives exactly the routed block's sum."""
    inp = _small(name, T, **kw)
    wl = inp.wl
    r = oracle.moe_block(inp)
    idx2, w2 = _with_skip_slot(r["idx"], r["w"], wl.E, np.full(wl.T, wl.k))
    acc, y = oracle.experts_block(inp, idx2, w2, skip=wl.E)
    assert np.array_equal(acc, r["acc"]) and np.array_equal(y, r["y"])


def test_skip_slot_anywhere_equals_routed_block():
    """The skip id sits in a different slot on each row; the kept slots keep
    their order, so the sum is still the routed block's, bit for bit."""
    inp = _small("tiny")
    wl = inp.wl
    r = oracle.moe_block(inp)
    pos = np.arange(wl.T) % (wl.k + 1)
    assert set(pos.tolist()) == set(range(wl.k + 1))
    idx2, w2 = _with_skip_slot(r["idx"], r["w"], wl.E, pos)
    acc, _ = oracle.experts_block(inp, idx2, w2, skip=wl.E)
    assert np.array_equal(acc, r["acc"])


def test_skip_slot_weight_is_left_out():
    """Whatever weight the skipped slot carries, it does not enter the sum."""
    inp = _small("tiny")
    wl = inp.wl
    r = oracle.moe_block(inp)
    idx2, w2 = _with_skip_slot(r["idx"], r["w"], wl.E, np.full(wl.T, wl.k))
    w2[:, -1] = 1e30
    acc, _ = oracle.experts_block(inp, idx2, w2, skip=wl.E)
    assert np.array_equal(acc, r["acc"])


def test_plan_over_one_more_expert():
    """The 9-slot plan written out: the skip id is plan expert E, it gets every
    token once, and its block is the last T positions, pairs ascending."""
    T, k, E = 6, 2, 4
    idx = np.array([[0, 3], [3, 1], [2, 0], [1, 3], [0, 2], [3, 2]])
    idx2, _ = _with_skip_slot(idx, np.ones((T, k)), E, np.full(T, k))
    p = oracle.plan(idx2, E + 1)
    assert p["counts"].tolist() == [3, 2, 3, 4, 6]
    assert p["offsets"].tolist() == [0, 3, 5, 8, 12, 18]
    assert p["perm"][12:].tolist() == [t * (k + 1) + k for t in range(T)]


def test_mutant_skip_by_position_goes_red(monkeypatch):
    """Plant 'drop the last slot' in place of 'drop the skip id': the pin with
    the skip id in varying slots must fail."""
    real = OM.combine

    def bad(o, w, out_scale, dtype=np.float64, keep=None):
        if keep is not None:
            keep = np.ones_like(keep)
            keep[:, -1] = False
        return real(o, w, out_scale, dtype=dtype, keep=keep)
    monkeypatch.setattr(OM, "combine", bad)
    with pytest.raises(AssertionError):
        test_skip_slot_anywhere_equals_routed_block()
