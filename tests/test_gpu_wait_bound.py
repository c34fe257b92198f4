"""Failure detection on the GPU without a fault: the tcgen05 pipelines'
bounded mbarrier wait is made to run out on purpose (a barrier nothing
arrives on, a short poll limit, in a one-warp kernel with no TMA and no TMEM),
and the host reads the error code it leaves; the context stays usable, which
a normal forward right after shows by passing oracle parity."""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def api():
    from sigmoid_top_routing_b200 import build
    build.build(quiet=True)
    from sigmoid_top_routing_b200 import api as A
    A.load()
    return A


def test_expired_wait_reports_code_2_and_context_survives(api):
    from sigmoid_top_routing_b200 import abi, inputs
    from sigmoid_top_routing_b200.device_inputs import to_device
    lib = api.load()
    assert api.moe_device_error() == 0                      # start clean
    assert lib.moe_wait_bound_check(4096, None) == abi.MOE_OK
    assert api.moe_device_error() == 2                      # the wait ran out and said so
    assert api.moe_device_error() == 0                      # read-and-clear
    assert lib.moe_wait_bound_check(0, None) == abi.MOE_ERR_SHAPE
    assert lib.moe_wait_bound_check((1 << 20) + 1, None) == abi.MOE_ERR_SHAPE

    wl = inputs.WORKLOADS["lfm2_decode_t8"]
    inp = inputs.make_inputs(wl)
    D = to_device(inp)
    y, idx, w, _ = api.moe_forward(D.x, D.W, D.w_router, D.expert_bias, E=wl.E, k=wl.k, I=wl.I, eps=wl.eps,
                                   dispatch=abi.MOE_DISPATCH_GEMM)
    torch.cuda.synchronize()
    assert api.moe_device_error() == 0
    ref = oracle.moe_block(inp)
    assert np.array_equal(idx.cpu().numpy(), ref["idx"])
    yg = y.float().cpu().numpy().astype(np.float64)
    assert np.linalg.norm(yg - ref["y"]) / np.linalg.norm(ref["y"]) < 1e-2
