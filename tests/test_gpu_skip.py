"""The skip-slot plan on the GPU (TensorFold issue #548, "Paths your experts
test does not reach", the skip-a-slot row): the block's picks plus the shared
expert's id E in one more slot, planned over E + 1 plan experts, run through
moe_experts_ex with plan expert E skipped.  The pages' checks, here through
the C ABI with the workspace filled with 0xFF before the launches:

  * the skipped slot's rows stay untouched (its h rows, and its per-slot
    output rows under the ordered combine, are still 0xFF);
  * the result has the bytes of the plain k-slot form (ordered combine: bit
    for bit; atomic combine: the same up to the order of fp32 additions);
  * the plan is the oracle's plan over E + 1 experts, bit for bit;
  * y matches the oracle's skip form (experts_block) on the GPU's picks.
A skip of the most-routed expert, with weights for every plan expert, is
checked against the oracle too."""
import numpy as np
import pytest

import oracle
from sigmoid_top_routing_b200 import inputs as G
from tests import parity

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def api():
    from sigmoid_top_routing_b200 import build
    build.build(quiet=True)
    from sigmoid_top_routing_b200 import api as A
    A.load()
    return A


_CACHE = {}


def _inputs(name, T):
    key = (name, T)
    if key not in _CACHE:
        _CACHE.clear()
        wl = G.WORKLOADS[name]
        _CACHE[key] = G.make_inputs(wl if T is None else wl.with_T(T))
    return _CACHE[key]


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _oracle_gate(inp, idx, w, y_bits, skip):
    _, y_ref = oracle.experts_block(inp, idx, w, skip=skip)
    y = oracle.bf16_to_f64(y_bits)
    rn = np.isnan(y_ref).any(axis=1)
    assert np.array_equal(np.isnan(y).any(axis=1), rn)
    err = y[~rn] - y_ref[~rn]
    rel = np.linalg.norm(err) / np.linalg.norm(y_ref[~rn])
    if inp.wl.fmt == "bf16":
        assert rel <= parity.BF16_REL_L2 and np.abs(err).max() <= parity.BF16_MAX_ABS, rel
    else:
        assert rel <= parity.AFFINE4_REL_L2, rel
    return rel


CASES = [("lfm2_decode_t8", None, "gemm"), ("lfm2_decode_t8", None, "gemv"),
         ("lfm2_prefill_t4096", 300, "auto"), ("nemotron_relu2_t2048", 200, "auto"),
         ("affine4_t64", None, "auto"), ("affine4_t512", None, "gemm"), ("nvfp4_t64", None, "auto")]


@pytest.mark.parametrize("combine", ["ordered", "atomic"])
@pytest.mark.parametrize("name,T,dispatch", CASES)
def test_shared_id_slot_skipped(api, name, T, dispatch, combine):
    from sigmoid_top_routing_b200 import abi
    from sigmoid_top_routing_b200.device_inputs import to_device
    inp = _inputs(name, T)
    wl = inp.wl
    D = to_device(inp)
    disp = {"auto": abi.MOE_DISPATCH_AUTO, "gemv": abi.MOE_DISPATCH_GEMV, "gemm": abi.MOE_DISPATCH_GEMM}[dispatch]
    comb = abi.MOE_COMBINE_ORDERED if combine == "ordered" else abi.MOE_COMBINE_ATOMIC
    idx, w = api.moe_route(D.x, None, D.w_router, D.expert_bias, E=wl.E, k=wl.k, eps=wl.eps, scale=wl.router_scale)
    # the k-slot form
    plan_k = api.moe_plan(idx, E=wl.E, H=wl.H, I=wl.I)
    y_k = api.moe_experts(D.x, plan_k, w, D.W, E=wl.E, I=wl.I, out_scale=wl.out_scale, dispatch=disp,
                          combine=comb)
    # the (k + 1)-slot form: the shared id E with weight 1 in the last slot, E + 1 plan experts
    E1, k1 = wl.E + 1, wl.k + 1
    idx1 = torch.cat([idx, torch.full((wl.T, 1), wl.E, dtype=torch.int32, device="cuda")], dim=1).contiguous()
    w1 = torch.cat([w, torch.ones((wl.T, 1), dtype=torch.float32, device="cuda")], dim=1).contiguous()
    d1 = api.dims(wl.T, wl.H, E1, k1, wl.I)
    ws1 = api.new_workspace(d1, D.W.fmt, dispatch=disp, combine=comb)
    plan1 = api.new_plan(wl.T, E1, k1)
    y1 = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    for t in (ws1, y1, plan1.counts, plan1.offsets, plan1.perm, plan1.inv, plan1.tiles):
        t.view(torch.uint8).fill_(0xFF)
    api.moe_plan(idx1, E=E1, H=wl.H, I=wl.I, plan=plan1, ws=ws1)
    ws1.fill_(0xFF)                                  # the expert stage starts from 0xFF everywhere
    api.moe_experts(D.x, plan1, w1, D.W, E=E1, I=wl.I, out_scale=wl.out_scale, y=y1, ws=ws1, skip=wl.E,
                    dispatch=disp, combine=comb)
    torch.cuda.synchronize()
    assert api.moe_device_error() == 0

    idx1_np = idx1.cpu().numpy().astype(np.int64)
    want = oracle.plan(idx1_np, E1)
    got = {"counts": plan1.counts, "offsets": plan1.offsets, "perm": plan1.perm, "inv": plan1.inv,
           "tiles": plan1.tiles}
    for key, t in got.items():
        assert np.array_equal(t.cpu().numpy().astype(np.int64), want[key]), f"plan.{key}"
    lo, hi = int(want["offsets"][wl.E]), int(want["offsets"][wl.E + 1])
    assert hi - lo == wl.T

    # the skipped slot's rows are untouched
    L = api.moe_workspace_layout(d1, D.W.fmt, dispatch=disp, combine=comb)
    wsb = ws1.cpu().numpy()
    h_rows = wsb[L.h: L.h + wl.T * k1 * wl.I * 2].reshape(wl.T * k1, wl.I * 2)
    assert (h_rows[lo:hi] == 0xFF).all(), "h rows of the skipped slot were written"
    assert not (h_rows[:lo] == 0xFF).all(axis=1).any(), "an h row of a computed slot was not written"
    if combine == "ordered":
        s_rows = wsb[L.y_acc: L.y_acc + wl.T * k1 * wl.H * 4].reshape(wl.T * k1, wl.H * 4)
        assert (s_rows[lo:hi] == 0xFF).all(), "slot rows of the skipped slot were written"
        assert np.array_equal(_bits(y1), _bits(y_k)), "the skip form differs from the k-slot form"
    else:
        a = oracle.bf16_to_f64(_bits(y1))
        b = oracle.bf16_to_f64(_bits(y_k))
        ok = ~np.isnan(b).any(axis=1)
        assert np.array_equal(np.isnan(a).any(axis=1), ~ok)
        assert np.linalg.norm(a[ok] - b[ok]) <= 2e-3 * np.linalg.norm(b[ok])

    rel = _oracle_gate(inp, idx1_np, w1.cpu().numpy().astype(np.float64), _bits(y1), wl.E)
    print(name, T, dispatch, combine, "rel-L2", rel)


@pytest.mark.parametrize("name,T,dispatch", [("lfm2_decode_t8", None, "gemm"), ("lfm2_prefill_t4096", 200, "gemv"),
                                             ("affine4_t64", None, "auto")])
def test_skip_below_the_last_expert(api, name, T, dispatch):
    """Skip the most-routed plan expert (weights for all E): its pairs are left out."""
    from sigmoid_top_routing_b200 import abi
    from sigmoid_top_routing_b200.device_inputs import to_device
    inp = _inputs(name, T)
    wl = inp.wl
    D = to_device(inp)
    disp = {"auto": abi.MOE_DISPATCH_AUTO, "gemv": abi.MOE_DISPATCH_GEMV, "gemm": abi.MOE_DISPATCH_GEMM}[dispatch]
    idx, w = api.moe_route(D.x, None, D.w_router, D.expert_bias, E=wl.E, k=wl.k, eps=wl.eps, scale=wl.router_scale)
    idx_np = idx.cpu().numpy().astype(np.int64)
    skip = int(np.bincount(idx_np.ravel(), minlength=wl.E).argmax())
    plan = api.moe_plan(idx, E=wl.E, H=wl.H, I=wl.I)
    y = api.moe_experts(D.x, plan, w, D.W, E=wl.E, I=wl.I, out_scale=wl.out_scale, skip=skip, dispatch=disp)
    torch.cuda.synchronize()
    assert api.moe_device_error() == 0
    _oracle_gate(inp, idx_np, w.cpu().numpy().astype(np.float64), _bits(y), skip)
