"""Parity of the MLX-style affine 4-bit expert paths with the float64 oracle,
which dequantises the same codes exactly.  Two paths: the tcgen05 GEMM (codes
dequantised on chip into its shared-memory operand, weights rounded once to
bf16) and the decode GEMV (codes dequantised in registers, scale and bias
applied in fp32 per group).  Gate: rel-L2 <= 3e-2."""
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


def test_affine4_small_ragged(api):
    """Decode-width tiles (token tiles of 32), I = 64 (one SwiGLU tile), E = 8."""
    wl = G.Workload("a4_small", T=33, H=128, E=8, k=4, I=64, fmt="affine4")
    inp = inputs_of(wl)
    _check_all(inp, run_forward(api, inp))


def test_affine4_relu2_small(api):
    wl = G.Workload("a4_relu2", T=40, H=256, E=16, k=6, I=192, act="relu2", fmt="affine4", out_scale=2.5)
    inp = inputs_of(wl)
    _check_all(inp, run_forward(api, inp))


@pytest.mark.parametrize("path", ["auto", "gemm", "gemv"])
@pytest.mark.parametrize("T", [1, 8, 64])
def test_affine4_decode_sizes(api, T, path):
    from sigmoid_top_routing_b200 import abi
    d = {"auto": abi.MOE_DISPATCH_AUTO, "gemm": abi.MOE_DISPATCH_GEMM, "gemv": abi.MOE_DISPATCH_GEMV}[path]
    inp = inputs_of(G.WORKLOADS[f"affine4_t{T}"])
    _check_all(inp, run_forward(api, inp, dispatch=d))


def test_affine4_gemv_token_chunks_and_short_k(api):
    """GEMV with more than 8 tokens per expert (several token chunks per row
    block) and H = 128 (two groups of 64: most warps get no K slice)."""
    from sigmoid_top_routing_b200 import abi
    wl = G.Workload("a4_small", T=33, H=128, E=8, k=4, I=64, fmt="affine4")
    inp = inputs_of(wl)
    _check_all(inp, run_forward(api, inp, dispatch=abi.MOE_DISPATCH_GEMV))


def test_affine4_gemv_relu2(api):
    from sigmoid_top_routing_b200 import abi
    wl = G.Workload("a4_relu2", T=40, H=256, E=16, k=6, I=192, act="relu2", fmt="affine4", out_scale=2.5)
    inp = inputs_of(wl)
    _check_all(inp, run_forward(api, inp, dispatch=abi.MOE_DISPATCH_GEMV))


@pytest.mark.parametrize("path", ["auto", "gemv"])
def test_affine4_t512(api, path):
    """32 pairs per expert: AUTO runs the tcgen05 path (token tiles of 128,
    interleaved SwiGLU tiles); the TMA GEMV is forced (four 8-token chunks per
    expert on average, the hot experts' many more)."""
    from sigmoid_top_routing_b200 import abi
    d = {"auto": abi.MOE_DISPATCH_AUTO, "gemv": abi.MOE_DISPATCH_GEMV}[path]
    inp = inputs_of(G.WORKLOADS["affine4_t512"])
    _check_all(inp, run_forward(api, inp, dispatch=d))


@pytest.mark.parametrize("act", ["swiglu", "relu2"])
def test_affine4_tma_gemv_many_chunks(api, act):
    """The TMA GEMV (forced) at 48 pairs per expert on average: six 8-token
    chunks per expert, ragged, H = 1024 (two stages of K), I = 512, 2 all-NaN
    token rows."""
    from sigmoid_top_routing_b200 import abi
    wl = G.Workload("a4_mid", T=96, H=1024, E=8, k=4, I=512, act=act, fmt="affine4", nan_rows=2)
    inp = inputs_of(wl)
    rep = _check_all(inp, run_forward(api, inp, dispatch=abi.MOE_DISPATCH_GEMV))
    assert rep.nan_rows == 2


def test_affine4_t8192_full(api):
    """The full 8192-token workload as the benchmark runs it: every row
    against the oracle, plus the whole plan."""
    inp = inputs_of(G.WORKLOADS["affine4_t8192"])
    out = run_forward(api, inp)
    _check_all(inp, out)


def test_affine4_relu2_wide_tiles(api):
    """relu^2 with token tiles of 256 (mean pairs per expert > 96)."""
    wl = G.Workload("a4_relu2_wide", T=1024, H=256, E=8, k=2, I=320, act="relu2", fmt="affine4")
    inp = inputs_of(wl)
    _check_all(inp, run_forward(api, inp))
