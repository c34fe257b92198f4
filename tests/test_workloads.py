"""The seeded workloads match their recipe, and the stored golden values are
still what the oracle gives."""
import json
import os

import numpy as np

import oracle as O
from sigmoid_top_routing_b200 import inputs as G

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_hot_delta_recorded_and_share_in_band():
    with open(os.path.join(GOLDEN, "nemotron_hot_delta.json")) as f:
        gold = json.load(f)
    wl = G.WORKLOADS["nemotron_relu2_t2048"]
    assert wl.hot_delta == gold["hot_delta"]
    inp = G.make_inputs(wl, with_experts=False)
    assert inp.hot.tolist() == gold["hot_experts"]
    r = O.route(k=wl.k, eps=wl.eps, scale=wl.router_scale, expert_bias=inp.expert_bias,
                x_bits=inp.x_bits, w_router=inp.w_router)
    share = np.isin(r["idx"], inp.hot).mean()
    assert 0.38 <= share <= 0.42


def test_tiny_golden_reproduced():
    with open(os.path.join(GOLDEN, "tiny_oracle.json")) as f:
        gold = json.load(f)
    r = O.moe_block(G.make_inputs(G.WORKLOADS["tiny"]))
    assert r["idx"].tolist() == gold["idx"]
    np.testing.assert_array_equal(r["w"], np.array(gold["w"]))
    np.testing.assert_allclose(r["y"][:, :32], np.array(gold["y_first32"]), rtol=1e-13, atol=1e-16)
    np.testing.assert_allclose(r["y"].sum(axis=1), np.array(gold["y_row_sum"]), rtol=1e-12, atol=1e-15)


def test_prefill_nan_rows():
    wl = G.WORKLOADS["lfm2_prefill_t4096"]
    inp = G.make_inputs(wl, with_experts=False)
    assert len(inp.nan_rows) == 41 == wl.nan_rows
    x = G.bf16_bits_to_f32(inp.x_bits)
    assert np.isnan(x[inp.nan_rows]).all()
    assert np.isfinite(np.delete(x, inp.nan_rows, axis=0)).all()
    L = O.router_logits(inp.x_bits[inp.nan_rows[:3]], inp.w_router)
    assert np.isnan(L).all()


def test_bf16_rounding_nearest_even():
    a = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0, np.inf], np.float32)
    b = G.f32_to_bf16_bits(a)
    back = G.bf16_bits_to_f32(b)
    np.testing.assert_array_equal(back, np.array([1.0, 1.0, 1.0 + 2 ** -6, -2.5, 0.0, np.inf], np.float32))


def test_affine4_shapes():
    wl = G.Workload("a4", T=2, H=128, E=3, k=2, I=64, fmt="affine4")
    inp = G.make_inputs(wl)
    assert inp.w1_q.shape == (3, 128, 16) and inp.w1_q.dtype == np.uint32
    assert inp.w1_scale.shape == (3, 128, 2) and inp.w1_bias.shape == (3, 128, 2)
    assert inp.w2_q.shape == (3, 128, 8) and inp.w2_scale.shape == (3, 128, 1)
    w = O.dequant_affine4(inp.w1_q, inp.w1_scale, inp.w1_bias)
    assert abs(w.std() - 0.02) < 0.003
