"""The block through its separate C-ABI calls -- moe_route, then moe_plan,
then moe_experts -- and through moe_forward_host (host buffers in and out),
against the float64 oracle with the same gates as the fused moe_forward."""
import dataclasses

import numpy as np
import pytest

from sigmoid_top_routing_b200 import inputs as G
from tests import parity
from tests.test_gpu_parity import _small, inputs_of

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def api():
    from sigmoid_top_routing_b200 import build
    build.build(quiet=True)
    from sigmoid_top_routing_b200 import api as A
    A.load()
    return A


def _plan_dict(idx, plan, P):
    return {"idx": idx.cpu().numpy(), "counts": plan.counts.cpu().numpy(), "offsets": plan.offsets.cpu().numpy(),
            "perm": plan.perm.cpu().numpy()[:P], "inv": plan.inv.cpu().numpy()[:P],
            "tiles": plan.tiles.cpu().numpy()}


def _check(inp, idx, w, y, plan):
    wl = inp.wl
    rep = parity.check(inp, np.arange(wl.T), idx.cpu().numpy().astype(np.int64), w.cpu().numpy(),
                       y.view(torch.int16).cpu().numpy().view(np.uint16), gpu_plan=_plan_dict(idx, plan, wl.P))
    print(wl.name, rep.as_dict())


@pytest.mark.parametrize("base,T", [("lfm2_decode_t8", 8), ("lfm2_prefill_t4096", 600),
                                    ("nemotron_relu2_t2048", 300), ("affine4_t8", 8)])
@pytest.mark.parametrize("combine", ["atomic", "ordered"])
def test_route_then_plan_then_experts(api, base, T, combine):
    from sigmoid_top_routing_b200 import abi
    from sigmoid_top_routing_b200.device_inputs import to_device
    inp = inputs_of(_small(base, T))
    wl = inp.wl
    D = to_device(inp)
    old = api.moe_set_combine(abi.MOE_COMBINE_ORDERED if combine == "ordered" else abi.MOE_COMBINE_ATOMIC)
    try:
        idx, w = api.moe_route(D.x, None, D.w_router, D.expert_bias, E=wl.E, k=wl.k, eps=wl.eps,
                               scale=wl.router_scale)
        plan = api.moe_plan(idx, E=wl.E, H=wl.H, I=wl.I)
        y = api.moe_experts(D.x, plan, w, D.W, E=wl.E, I=wl.I, out_scale=wl.out_scale)
        torch.cuda.synchronize()
        assert api.moe_device_error() == 0
    finally:
        api.moe_set_combine(old)
    _check(inp, idx, w, y, plan)


@pytest.mark.parametrize("base,T", [("lfm2_decode_t8", 8), ("nemotron_relu2_t2048", 300)])
def test_forward_host_buffers(api, base, T):
    from sigmoid_top_routing_b200.device_inputs import to_device
    inp = inputs_of(_small(base, T))
    wl = inp.wl
    D = to_device(inp)
    x_host = D.x.cpu().pin_memory()
    x_dev = torch.empty_like(D.x)
    y_dev = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    y_host = torch.empty((wl.T, wl.H), dtype=torch.bfloat16).pin_memory()
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    plan = api.new_plan(wl.T, wl.E, wl.k)
    ws = api.new_workspace(api.dims(wl.T, wl.H, wl.E, wl.k, wl.I), D.W.fmt)
    api.moe_forward_host(x_host, x_dev, D.W, D.w_router, D.expert_bias, E=wl.E, k=wl.k, I=wl.I, y_dev=y_dev,
                         y_host=y_host, topk_idx=idx, topk_w=w, plan=plan, ws=ws, eps=wl.eps,
                         router_scale=wl.router_scale, out_scale=wl.out_scale)
    assert api.moe_device_error() == 0
    assert torch.equal(y_host.view(torch.int16), y_dev.cpu().view(torch.int16))
    _check(inp, idx, w, y_host, plan)
