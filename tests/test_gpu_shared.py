"""The shared expert on the GPU: moe_shared_expert (one expert over every
token, same kernels as the routed experts) against the oracle's shared term,
and the whole block with y = bf16(out_scale * routed sum + shared) against
the oracle (vllm.cpp PR #684: the routed scale multiplies the routed sum
before the shared output is added)."""
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


def _wl(base, T, shared_I, **over):
    return dataclasses.replace(_small(base, T), shared_I=shared_I, **over)


@pytest.mark.parametrize("base,T,shared_I,dispatch", [
    ("nemotron_relu2_t2048", 300, 1536, None),   # tcgen05 GEMM, one expert, 300 tokens
    ("lfm2_decode_t8", 8, 1792, None),           # 32-wide token tiles, the x operand (T <= 16)
    ("nemotron_relu2_t2048", 12, 1536, None),    # relu^2, the x operand
    ("lfm2_decode_t8", 8, 1792, "gemv"),         # bf16 GEMV
    ("affine4_t8", 8, 1536, None),               # affine 4-bit TMA-fed GEMV
])
def test_shared_expert_alone(api, base, T, shared_I, dispatch):
    import oracle as O
    from sigmoid_top_routing_b200 import abi
    from sigmoid_top_routing_b200.device_inputs import shared_to_device, to_device
    inp = inputs_of(_wl(base, T, shared_I))
    D = to_device(inp)
    old = api.moe_set_dispatch(abi.MOE_DISPATCH_GEMV if dispatch == "gemv" else abi.MOE_DISPATCH_AUTO)
    try:
        y_sh = api.moe_shared_expert(D.x, shared_to_device(inp), I=shared_I)
        torch.cuda.synchronize()
    finally:
        api.moe_set_dispatch(old)
    got = y_sh.cpu().numpy().astype(np.float64)
    want = O.shared_expert(inp, np.arange(inp.wl.T))
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert rel < (3e-2 if inp.wl.fmt != "bf16" else 1e-2), rel


@pytest.mark.parametrize("base,T,shared_I", [("nemotron_relu2_t2048", 300, 1536),
                                              ("lfm2_decode_t8", 8, 1792), ("affine4_t64", 64, 1536)])
def test_block_with_shared_expert(api, base, T, shared_I):
    inp = inputs_of(_wl(base, T, shared_I))
    _check_all(inp, run_forward(api, inp))


def test_block_with_shared_expert_ordered_combine(api):
    from sigmoid_top_routing_b200 import abi
    old = api.moe_set_combine(abi.MOE_COMBINE_ORDERED)
    try:
        inp = inputs_of(_wl("nemotron_relu2_t2048", 300, 1536))
        _check_all(inp, run_forward(api, inp))
    finally:
        api.moe_set_combine(old)
