"""The slot-ordered combine (MOE_COMBINE_ORDERED): parity with the float64
oracle on every expert path, bitwise reproducibility, and batch invariance of
a token's output for bf16 experts."""
import dataclasses

import numpy as np
import pytest

from sigmoid_top_routing_b200 import inputs as G
from tests.test_gpu_parity import _check_all, _small, inputs_of, run_forward

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def api():
    from sigmoid_top_routing_b200 import abi, build
    build.build(quiet=True)
    from sigmoid_top_routing_b200 import api as A
    A.load()
    old = A.moe_set_combine(abi.MOE_COMBINE_ORDERED)
    yield A
    A.moe_set_combine(old)


def test_decode_gemm(api):
    inp = inputs_of(G.WORKLOADS["lfm2_decode_t8"])
    _check_all(inp, run_forward(api, inp))


def test_prefill_shape_with_nan_rows(api):
    inp = inputs_of(_small("lfm2_prefill_t4096", 500))
    rep = _check_all(inp, run_forward(api, inp))
    assert rep.nan_rows == 5


def test_relu2_out_scale(api):
    inp = inputs_of(_small("nemotron_relu2_t2048", 700))
    _check_all(inp, run_forward(api, inp))


def test_bf16_gemv(api):
    from sigmoid_top_routing_b200 import abi
    inp = inputs_of(_small("lfm2_decode_t8", 17))
    _check_all(inp, run_forward(api, inp, dispatch=abi.MOE_DISPATCH_GEMV))


@pytest.mark.parametrize("T", [8, 512])
def test_affine4(api, T):
    """T = 8 runs the TMA-fed 4-bit GEMV, T = 512 the tcgen05 GEMM."""
    inp = inputs_of(G.WORKLOADS[f"affine4_t{T}"])
    _check_all(inp, run_forward(api, inp))


def test_reproducible_bits(api):
    inp = inputs_of(_small("nemotron_relu2_t2048", 700))
    a = run_forward(api, inp)["y_bits"]
    b = run_forward(api, inp)["y_bits"]
    assert np.array_equal(a, b)


@pytest.mark.parametrize("T", [8, 64, 512, 4096])
def test_token_output_does_not_depend_on_the_batch(api, T):
    """The first 8 tokens' y bits are the same whether the batch holds 8 or
    T tokens (token tiles of 32, 128 or 256 columns)."""
    wl = dataclasses.replace(G.WORKLOADS["lfm2_prefill_t4096"], nan_rows=0)
    inp_T = G.make_inputs(wl.with_T(T))
    inp_8 = G.make_inputs(wl.with_T(8))
    assert np.array_equal(inp_T.x_bits[:8], inp_8.x_bits)
    y_T = run_forward(api, inp_T)["y_bits"][:8]
    y_8 = run_forward(api, inp_8)["y_bits"]
    assert np.array_equal(y_T, y_8)
