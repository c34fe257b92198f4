"""Router and activation variants on the GPU (through moe_forward_ex) against
the float64 oracle: softmax scores, norm_topk off, Nemotron's eps 1e-20 and
the SwiGLU input clamp, on each expert path (tcgen05 GEMM at 32- and
128-wide token tiles, bf16 GEMV, affine 4-bit GEMV and GEMM)."""
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


def _wl(base, T, **over):
    return dataclasses.replace(_small(base, T), **over)


@pytest.mark.parametrize("base,T", [("lfm2_decode_t8", 8), ("lfm2_prefill_t4096", 500),
                                    ("nemotron_relu2_t2048", 300)])
@pytest.mark.parametrize("norm", [True, False])
def test_softmax_router(api, base, T, norm):
    """T <= 32 selects in one CTA with the plan; larger T in the per-token
    warps of the partial-logit path; NaN rows score NaN throughout."""
    inp = inputs_of(_wl(base, T, score="softmax", norm_topk=norm))
    _check_all(inp, run_forward(api, inp))


def test_sigmoid_without_normalisation(api):
    """Without the division the six weights sum to ~3 instead of ~1, so y is
    ~3x larger; out_scale 1 (instead of 2.5) keeps y, and so the bf16 rounding
    the absolute max-abs gate sees, at the size of the other workloads."""
    inp = inputs_of(_wl("nemotron_relu2_t2048", 700, norm_topk=False, out_scale=1.0))
    _check_all(inp, run_forward(api, inp))


def test_nemotron_eps(api):
    """Nemotron's engine keeps + 1e-20 on the weights' sum (TensorFold issue
    #548, its router top-k status comment)."""
    inp = inputs_of(_wl("nemotron_relu2_t2048", 300, eps=1e-20))
    _check_all(inp, run_forward(api, inp))


@pytest.mark.parametrize("base,T,dispatch", [
    ("lfm2_decode_t8", 8, None),          # tcgen05 GEMM, 32-wide tiles (gate and up halves in one tile)
    ("lfm2_prefill_t4096", 600, None),    # 128-wide tiles, two accumulators
    ("lfm2_decode_t8", 17, "gemv"),       # bf16 CUDA-core GEMV
    ("affine4_t8", 8, None),              # affine 4-bit TMA-fed GEMV
    ("affine4_t512", 512, None),          # affine 4-bit tcgen05 GEMM
])
def test_swiglu_limit(api, base, T, dispatch):
    """With limit 1.0 about a quarter of the gate and up values clamp; the
    output follows the oracle and differs from the unclamped one."""
    from sigmoid_top_routing_b200 import abi
    d = None if dispatch is None else abi.MOE_DISPATCH_GEMV
    inp = inputs_of(_wl(base, T, swiglu_limit=1.0))
    out = run_forward(api, inp, dispatch=d)
    _check_all(inp, out)
    free = inputs_of(_wl(base, T))
    y_free = run_forward(api, free, dispatch=d)["y_bits"]
    assert np.mean(out["y_bits"] != y_free) > 0.05          # the clamp fired


@pytest.mark.parametrize("base,T", [("lfm2_decode_t8", 8), ("lfm2_prefill_t4096", 4096)])
def test_softmax_forward_router_matches_standalone_bitwise(api, base, T):
    wl = _wl(base, T, nan_rows=0, score="softmax")
    inp = G.make_inputs(wl, with_experts=False)
    from sigmoid_top_routing_b200.device_inputs import bf16_tensor
    x = bf16_tensor(inp.x_bits, "cuda")
    wr = torch.from_numpy(inp.w_router).cuda()
    b = torch.from_numpy(inp.expert_bias).cuda()
    i_ref, w_ref = api.moe_route(x, None, wr, b, E=wl.E, k=wl.k, score="softmax")
    W = api.ExpertWeights(act=0, fmt=0, w1=torch.zeros((wl.E, 2 * wl.I, wl.H), dtype=torch.bfloat16, device="cuda"),
                          w2=torch.zeros((wl.E, wl.H, wl.I), dtype=torch.bfloat16, device="cuda"))
    _, i_fwd, w_fwd, _ = api.moe_forward(x, W, wr, b, E=wl.E, k=wl.k, I=wl.I, score="softmax")
    torch.cuda.synchronize()
    assert torch.equal(i_fwd, i_ref)
    assert torch.equal(w_fwd.view(torch.int32), w_ref.view(torch.int32))
