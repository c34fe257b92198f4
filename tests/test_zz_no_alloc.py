"""moe_forward_static, the forward pass for callers that cannot allocate
device memory (a plugin host that only hands over input and output tensors,
a serving loop that must not wait on an allocator).  It keeps its scratch in a fixed array inside the
library instead of a caller workspace.

Called here through the C ABI, twice in a row (the array keeps the previous
call's contents, so the second call checks that it starts clean), and
compared with moe_forward given an ordinary workspace, within the parity
tolerances of the other GPU tests.  Collected last on purpose."""
import ctypes

import numpy as np
import pytest

from tests import parity

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def lib():
    from sigmoid_top_routing_b200 import abi, build
    build.build(quiet=True)
    return abi.load()


def _case(name, T=None):
    from sigmoid_top_routing_b200 import inputs as G
    wl = G.WORKLOADS[name]
    if T is not None:
        wl = wl.with_T(T)
    return G.make_inputs(wl)


@pytest.mark.parametrize("name,T", [("lfm2_decode_t8", None), ("nemotron_relu2_t2048", 40)])
def test_static_forward_matches_workspace_forward(lib, name, T):
    from sigmoid_top_routing_b200 import abi, api
    from sigmoid_top_routing_b200.device_inputs import to_device
    inp = _case(name, T)
    wl = inp.wl
    D = to_device(inp)
    y_ref, idx_ref, w_ref, _ = api.moe_forward(D.x, D.W, D.w_router, D.expert_bias, E=wl.E, k=wl.k, I=wl.I,
                                               eps=wl.eps, router_scale=wl.router_scale,
                                               out_scale=wl.out_scale)
    torch.cuda.synchronize()
    ref = y_ref.float().cpu().numpy().astype(np.float64)

    d = abi.moe_dims(wl.T, wl.H, wl.E, wl.k, wl.I)
    cw = D.W.c_struct()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        plan = api.new_plan(wl.T, wl.E, wl.k)
        y = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
        idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
        w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
        for t in (y, idx, w):
            t.view(torch.uint8).fill_(0xFF)
        cp = plan.c_struct()
        st = lib.moe_forward_static(D.x.data_ptr(), None, D.w_router.data_ptr(), D.expert_bias.data_ptr(),
                                    ctypes.byref(d), wl.eps, wl.router_scale, wl.out_scale, ctypes.byref(cw),
                                    idx.data_ptr(), w.data_ptr(), ctypes.byref(cp), y.data_ptr(), stream)
        assert st == abi.MOE_OK, lib.moe_last_error().decode()
        torch.cuda.synchronize()
        assert api.moe_device_error() == 0
        assert torch.equal(idx, idx_ref), f"call {call}: picks"
        assert torch.equal(w.view(torch.int32), w_ref.view(torch.int32)), f"call {call}: weights"
        got = y.float().cpu().numpy().astype(np.float64)
        rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert rel <= parity.BF16_REL_L2, f"call {call}: rel-L2 {rel}"
        assert np.abs(got - ref).max() <= parity.BF16_MAX_ABS, f"call {call}: max-abs"


def test_static_forward_refuses_sizes_beyond_its_scratch(lib):
    from sigmoid_top_routing_b200 import abi
    d = abi.moe_dims(4096, 2048, 32, 4, 1792)
    W = abi.moe_experts_w(0, 0, 0x100000, None, None, 0x200000, None, None)
    p = abi.moe_plan_t(0x1000, 0x2000, 0x3000, 0x4000, 0x5000)
    st = lib.moe_forward_static(0x10000, None, 0x20000, None, ctypes.byref(d), 1e-6, 1.0, 1.0,
                                ctypes.byref(W), 0x30000, 0x40000, ctypes.byref(p), 0x50000, None)
    assert st == abi.MOE_ERR_WORKSPACE
    assert "use moe_forward with a workspace" in lib.moe_last_error().decode()
