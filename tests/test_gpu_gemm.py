"""Parity of the tcgen05 grouped-GEMM expert path with the float64 oracle,
from tiny shapes with ragged token tiles up to the full prefill and relu^2
workloads (the sizes the benchmark runs)."""
import dataclasses

import numpy as np
import pytest

from sigmoid_top_routing_b200 import inputs as G
from tests.test_gpu_parity import _check_all, _small, inputs_of, run_forward

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def api():
    from sigmoid_top_routing_b200 import build
    build.build(quiet=True)
    from sigmoid_top_routing_b200 import api as A
    A.load()
    return A


def _gemm(api, inp, **kw):
    from sigmoid_top_routing_b200 import abi
    return run_forward(api, inp, dispatch=abi.MOE_DISPATCH_GEMM, **kw)


def test_gemm_tiny(api):
    inp = inputs_of(G.WORKLOADS["tiny"])
    _check_all(inp, _gemm(api, inp))


@pytest.mark.parametrize("T", [1, 8, 13, 16, 17, 33])
def test_gemm_decode_shapes(api, T):
    """Token tiles of width 32 (N = 16 or 32 per expert).  At T <= 16 the up
    GEMM multiplies x itself (every token, N = T rounded up to 16) and keeps
    the routed tokens' columns; above, it reads the rows gathered in plan
    order."""
    inp = inputs_of(_small("lfm2_decode_t8", T))
    _check_all(inp, _gemm(api, inp))


@pytest.mark.parametrize("T", [5, 16])
def test_gemm_relu2_x_operand(api, T):
    """relu^2 up at T <= 16 (the x operand with its routed columns), E = 64, k = 6."""
    inp = inputs_of(_small("nemotron_relu2_t2048", T))
    _check_all(inp, _gemm(api, inp))


def test_gemm_mid_tiles(api):
    """T = 300: token tiles of width 128, ragged per expert, 3 NaN token rows."""
    inp = inputs_of(_small("lfm2_prefill_t4096", 300))
    rep = _check_all(inp, _gemm(api, inp))
    assert rep.nan_rows == 3


def test_gemm_relu2_small(api):
    inp = inputs_of(_small("nemotron_relu2_t2048", 96))
    _check_all(inp, _gemm(api, inp))


def test_gemm_tiny_dims_ragged(api):
    """I = 64 (one SwiGLU tile), H = 192 (three k-blocks), E = 5, k = 3."""
    wl = G.Workload("ragged", T=57, H=192, E=5, k=3, I=64)
    inp = inputs_of(wl)
    _check_all(inp, _gemm(api, inp))
    wl2 = dataclasses.replace(wl, name="ragged_relu2", act="relu2", I=192, out_scale=2.5)
    inp2 = inputs_of(wl2)
    _check_all(inp2, _gemm(api, inp2))


def test_lfm2_prefill_t4096_full(api):
    """The prefill workload at full size (41 all-NaN token rows), every row
    against the oracle."""
    inp = inputs_of(G.WORKLOADS["lfm2_prefill_t4096"])
    rep = _check_all(inp, run_forward(api, inp))
    assert rep.nan_rows == 41


def test_nemotron_relu2_t2048_full(api):
    inp = inputs_of(G.WORKLOADS["nemotron_relu2_t2048"])
    out = run_forward(api, inp)
    _check_all(inp, out)
    counts = out["plan"]["counts"]
    hot = inp.hot
    assert 0.38 <= counts[hot].sum() / counts.sum() <= 0.42


def test_gemm_equals_gemv_on_decode(api):
    """Both expert paths on the same decode batch: identical picks and plan,
    outputs within bf16 rounding of each other."""
    from sigmoid_top_routing_b200 import abi
    inp = inputs_of(G.WORKLOADS["lfm2_decode_t8"])
    a = run_forward(api, inp, dispatch=abi.MOE_DISPATCH_GEMV)
    b = run_forward(api, inp, dispatch=abi.MOE_DISPATCH_GEMM)
    assert np.array_equal(a["idx"], b["idx"])
    ya = a["y_bits"].astype(np.uint32) << 16
    yb = b["y_bits"].astype(np.uint32) << 16
    fa, fb = ya.view(np.float32), yb.view(np.float32)
    assert np.abs(fa - fb).max() <= 2e-2
