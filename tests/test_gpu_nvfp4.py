"""Parity of the NVFP4 expert paths (ModelOpt layout, TensorFold issue #548)
with the float64 oracle, which dequantises the same codes exactly
(e2m1 * e4m3 * global scale).  The decode GEMV dequantises e2m1 * e4m3 exactly
into f16 and stages the token rows in f16 after an exact per-token power-of-two
scale; the global scale multiplies the fp32 sum.  Gate: rel-L2 <= 3e-2 (the
4-bit tolerance), plus the NaN-row, plan and pick checks of every parity test."""
import dataclasses

import numpy as np
import pytest

from sigmoid_top_routing_b200 import inputs as G
from tests.test_gpu_parity import _check_all, inputs_of, run_forward

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def api():
    from sigmoid_top_routing_b200 import build
    build.build(quiet=True)
    from sigmoid_top_routing_b200 import api as A
    A.load()
    return A


def test_nvfp4_small_ragged(api):
    wl = G.Workload("n4_small", T=33, H=128, E=8, k=4, I=64, fmt="nvfp4")
    inp = inputs_of(wl)
    _check_all(inp, run_forward(api, inp))


def test_nvfp4_relu2_small(api):
    wl = G.Workload("n4_relu2", T=40, H=256, E=16, k=6, I=192, act="relu2", fmt="nvfp4", out_scale=2.5)
    inp = inputs_of(wl)
    _check_all(inp, run_forward(api, inp))


@pytest.mark.parametrize("T", [1, 8, 64])
def test_nvfp4_decode_sizes(api, T):
    inp = inputs_of(G.WORKLOADS[f"nvfp4_t{T}"])
    _check_all(inp, run_forward(api, inp))


@pytest.mark.parametrize("path", ["auto", "gemv"])
def test_nvfp4_t512(api, path):
    """AUTO: the tcgen05 path; forced: the TMA GEMV over many 8-token chunks."""
    from sigmoid_top_routing_b200 import abi
    d = {"auto": abi.MOE_DISPATCH_AUTO, "gemv": abi.MOE_DISPATCH_GEMV}[path]
    inp = inputs_of(G.WORKLOADS["nvfp4_t512"])
    _check_all(inp, run_forward(api, inp, dispatch=d))


@pytest.mark.parametrize("act", ["swiglu", "relu2"])
def test_nvfp4_tma_gemv_many_chunks(api, act):
    """The TMA GEMV (forced) at 48 pairs per expert: six 8-token chunks per
    expert, H = 1024, I = 512 (K of the down projection: one stage), 2 all-NaN
    token rows."""
    from sigmoid_top_routing_b200 import abi
    wl = G.Workload("n4_mid", T=96, H=1024, E=8, k=4, I=512, act=act, fmt="nvfp4", nan_rows=2)
    inp = inputs_of(wl)
    rep = _check_all(inp, run_forward(api, inp, dispatch=abi.MOE_DISPATCH_GEMV))
    assert rep.nan_rows == 2


def test_nvfp4_t8192_full(api):
    """The full 8192-token workload as the benchmark runs it, every row."""
    inp = inputs_of(G.WORKLOADS["nvfp4_t8192"])
    _check_all(inp, run_forward(api, inp))


def test_nvfp4_nan_and_huge_token_rows(api):
    """A NaN token row stays NaN; a row of huge (but finite) activations is
    staged after its power-of-two scale, so nothing overflows f16."""
    wl = dataclasses.replace(G.WORKLOADS["nvfp4_t8"], name="n4_big")
    inp = G.make_inputs(wl)
    x = inp.x_bits.copy()
    f = G.bf16_bits_to_f32(x[3]) * np.float32(2.0 ** 40)
    x[3] = G.f32_to_bf16_bits(f)                       # |x| up to ~4e12, far beyond f16
    x[5] = G.f32_to_bf16_bits(G.bf16_bits_to_f32(x[5]) * np.float32(2.0 ** -60))   # tiny row
    inp = dataclasses.replace(inp, x_bits=x)
    _check_all(inp, run_forward(api, inp))


def test_nvfp4_shared_expert_and_skip(api):
    """The shared expert in NVFP4 added after the routed scale."""
    wl = dataclasses.replace(G.WORKLOADS["nvfp4_t64"], shared_I=512, out_scale=1.5, name="n4_shared")
    inp = G.make_inputs(wl)
    _check_all(inp, run_forward(api, inp))
