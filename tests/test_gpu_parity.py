"""Parity of the CUDA path (through the C ABI) with the float64 oracle."""
import dataclasses

import numpy as np
import pytest

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


def inputs_of(wl):
    if wl not in _CACHE:
        _CACHE.clear()
        _CACHE[wl] = G.make_inputs(wl)
    return _CACHE[wl]


def run_forward(api, inp, *, dispatch=None, logits=None, poison=True):
    from sigmoid_top_routing_b200 import abi
    from sigmoid_top_routing_b200.device_inputs import to_device
    wl = inp.wl
    D = to_device(inp)
    old = api.moe_set_dispatch(dispatch if dispatch is not None else abi.MOE_DISPATCH_AUTO)
    try:
        d = api.dims(wl.T, wl.H, wl.E, wl.k, wl.I)
        ws = api.new_workspace(d, D.W.fmt)
        plan = api.new_plan(wl.T, wl.E, wl.k)
        y = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
        idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
        w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
        if poison:                              # outputs prefilled with 0xFF: unwritten rows show
            for t in (ws, y.view(torch.uint8), idx, w, plan.counts, plan.offsets, plan.perm, plan.inv,
                      plan.tiles):
                t.view(torch.uint8).fill_(0xFF)
        lg = None if logits is None else torch.from_numpy(logits).cuda()
        y_sh = None
        if wl.shared_I:
            from sigmoid_top_routing_b200.device_inputs import shared_to_device
            y_sh = api.moe_shared_expert(D.x, shared_to_device(inp), I=wl.shared_I)
        api.moe_forward(D.x, D.W, D.w_router, D.expert_bias, E=wl.E, k=wl.k, I=wl.I, logits=lg,
                        eps=wl.eps, router_scale=wl.router_scale, out_scale=wl.out_scale, topk_idx=idx,
                        topk_w=w, plan=plan, y=y, ws=ws, score=wl.score, norm_topk=wl.norm_topk, y_shared=y_sh)
        torch.cuda.synchronize()
        assert api.moe_device_error() == 0
    finally:
        api.moe_set_dispatch(old)
    out = {
        "idx": idx.cpu().numpy().astype(np.int64), "w": w.cpu().numpy(),
        "y_bits": y.view(torch.int16).cpu().numpy().view(np.uint16),
        "plan": {"idx": idx.cpu().numpy(), "counts": plan.counts.cpu().numpy(),
                 "offsets": plan.offsets.cpu().numpy(), "perm": plan.perm.cpu().numpy()[: wl.P],
                 "inv": plan.inv.cpu().numpy()[: wl.P], "tiles": plan.tiles.cpu().numpy()},
        "ws": ws, "d": d,
    }
    return out


def _check_all(inp, out, logits=None, tokens=None):
    wl = inp.wl
    tokens = np.arange(wl.T) if tokens is None else tokens
    rep = parity.check(inp, tokens, out["idx"][tokens], out["w"][tokens], out["y_bits"][tokens],
                       logits=logits, gpu_plan=out["plan"])
    print(wl.name, rep.as_dict())
    return rep


def _small(base, T, **over):
    return dataclasses.replace(G.WORKLOADS[base].with_T(T), **over)


# ---------------------------------------------------------------- decode path

def test_tiny(api):
    inp = inputs_of(G.WORKLOADS["tiny"])
    _check_all(inp, run_forward(api, inp))


def test_lfm2_decode_t8(api):
    inp = inputs_of(G.WORKLOADS["lfm2_decode_t8"])
    _check_all(inp, run_forward(api, inp))


@pytest.mark.parametrize("T", [1, 3, 17, 33])
def test_gemv_ragged_token_counts(api, T):
    from sigmoid_top_routing_b200 import abi
    inp = inputs_of(_small("lfm2_decode_t8", T))
    _check_all(inp, run_forward(api, inp, dispatch=abi.MOE_DISPATCH_GEMV))


def test_relu2_gemv(api):
    from sigmoid_top_routing_b200 import abi
    inp = inputs_of(_small("nemotron_relu2_t2048", 40))
    _check_all(inp, run_forward(api, inp, dispatch=abi.MOE_DISPATCH_GEMV))


def test_nan_logit_rows_via_logits_argument(api):
    """1 % of router-logit rows all-NaN, passed through the logits argument:
    picks stay distinct (0..k-1), weights and output rows are NaN."""
    from sigmoid_top_routing_b200 import abi
    import oracle as O
    wl = _small("lfm2_prefill_t4096", 200)
    inp = inputs_of(dataclasses.replace(wl, nan_rows=0))
    L = O.router_logits(inp.x_bits, inp.w_router).astype(np.float32)
    rows = np.random.default_rng(3).choice(wl.T, 2, replace=False)
    L[rows] = np.nan
    out = run_forward(api, inp, dispatch=abi.MOE_DISPATCH_GEMV, logits=L)
    assert np.all(out["idx"][rows] == np.arange(wl.k))
    rep = _check_all(inp, out, logits=L)
    assert rep.nan_rows == 2


def test_nan_logit_rows_via_logits_argument_tcgen05_prefill(api):
    """The prefill workload at full size with 1 % of router-logit rows all-NaN
    passed through the logits argument, on the library's own choice of expert
    kernels (the tcgen05 grouped GEMM at this size)."""
    import oracle as O
    wl = dataclasses.replace(G.WORKLOADS["lfm2_prefill_t4096"], nan_rows=0)
    inp = inputs_of(wl)
    L = O.router_logits(inp.x_bits, inp.w_router).astype(np.float32)
    rows = np.sort(np.random.default_rng(5).choice(wl.T, 41, replace=False))
    L[rows] = np.nan
    out = run_forward(api, inp, logits=L)
    assert np.all(out["idx"][rows] == np.arange(wl.k))
    rep = _check_all(inp, out, logits=L)
    assert rep.nan_rows == 41


def test_nan_token_rows_prefill_shape(api):
    from sigmoid_top_routing_b200 import abi
    inp = inputs_of(_small("lfm2_prefill_t4096", 300))
    assert inp.nan_rows is not None and len(inp.nan_rows) == 3
    out = run_forward(api, inp, dispatch=abi.MOE_DISPATCH_GEMV)
    rep = _check_all(inp, out)
    assert rep.nan_rows == 3


# ---------------------------------------------------------------- properties

def test_route_is_batch_invariant(api):
    """A token's picks and weights are the same bits whether it is routed
    alone, among 8, or among 4096 (one fixed fp32 summation order)."""
    wl = G.WORKLOADS["lfm2_prefill_t4096"]
    inp = G.make_inputs(dataclasses.replace(wl, nan_rows=0), with_experts=False)
    from sigmoid_top_routing_b200.device_inputs import bf16_tensor
    x = bf16_tensor(inp.x_bits, "cuda")
    wr = torch.from_numpy(inp.w_router).cuda()
    b = torch.from_numpy(inp.expert_bias).cuda()
    big_i, big_w = api.moe_route(x, None, wr, b, E=wl.E, k=wl.k)
    for T in (1, 8, 32):
        i, w = api.moe_route(x[:T].contiguous(), None, wr, b, E=wl.E, k=wl.k)
        assert torch.equal(i, big_i[:T])
        assert torch.equal(w.view(torch.int32), big_w[:T].view(torch.int32))


def test_out_scale_applied_once_to_finished_sum(api):
    """vllm.cpp PR #684: y = bf16_rn(2.5 * y_acc) bitwise, and y_acc is the
    unscaled routed sum (not a sum of pre-scaled terms)."""
    from sigmoid_top_routing_b200 import abi
    import oracle as O
    inp = inputs_of(_small("nemotron_relu2_t2048", 24))
    out = run_forward(api, inp, dispatch=abi.MOE_DISPATCH_GEMV)
    L = api.moe_workspace_layout(out["d"], 0)
    wl = inp.wl
    yacc = out["ws"][L.y_acc: L.y_acc + wl.T * wl.H * 4].view(torch.float32).view(wl.T, wl.H)
    want = (yacc * 2.5).to(torch.bfloat16)
    assert torch.equal(want.view(torch.int16).cpu(), torch.from_numpy(out["y_bits"].view(np.int16)))
    ref = O.moe_block(inp)
    acc = yacc.cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(acc - ref["acc"]) / np.linalg.norm(ref["acc"])
    assert rel < 5e-3
    assert np.linalg.norm(acc - ref["y"]) / np.linalg.norm(ref["y"]) > 0.3    # not the scaled sum


def test_plan_standalone_matches_oracle(api):
    import oracle as O
    rng = np.random.default_rng(0)
    for T, E, k in [(1, 8, 2), (5, 32, 4), (777, 64, 6), (4096, 32, 4), (9000, 256, 8)]:
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
        ti = torch.from_numpy(idx).cuda()
        plan = api.moe_plan(ti, E=E)
        torch.cuda.synchronize()
        want = O.plan(idx, E)
        P = T * k
        assert np.array_equal(plan.counts.cpu().numpy(), want["counts"])
        assert np.array_equal(plan.offsets.cpu().numpy(), want["offsets"])
        assert np.array_equal(plan.perm.cpu().numpy()[:P], want["perm"])
        assert np.array_equal(plan.inv.cpu().numpy()[:P], want["inv"])
        assert np.array_equal(plan.tiles.cpu().numpy(), want["tiles"])


def test_plan_reports_bad_expert_id(api):
    idx = torch.tensor([[0, 1], [2, 9]], dtype=torch.int32, device="cuda")
    plan = api.moe_plan(idx, E=8)
    assert api.moe_device_error() == 1
    assert api.moe_device_error() == 0          # read clears
    assert plan.counts.sum().item() == 3


def test_empty_batch_is_a_no_op(api):
    from sigmoid_top_routing_b200.device_inputs import to_device
    inp = inputs_of(G.WORKLOADS["tiny"])
    D = to_device(inp)
    wl = inp.wl
    x = D.x[:0]
    y = torch.empty((0, wl.H), dtype=torch.bfloat16, device="cuda")
    api.moe_forward(x, D.W, D.w_router, D.expert_bias, E=wl.E, k=wl.k, I=wl.I, y=y)
    torch.cuda.synchronize()


@pytest.mark.parametrize("base,T", [("lfm2_decode_t8", 8), ("lfm2_prefill_t4096", 4096),
                                    ("nemotron_relu2_t2048", 2048), ("nemotron_relu2_t2048", 19)])
def test_forward_router_matches_standalone_router_bitwise(api, base, T):
    """moe_forward routes through per-segment partial logits (8x the CTAs);
    moe_route uses one CTA per token block.  Both follow the same fp32 order,
    so picks and weights must be the same bits."""
    wl = dataclasses.replace(G.WORKLOADS[base].with_T(T), nan_rows=0)
    inp = G.make_inputs(wl, with_experts=False)
    from sigmoid_top_routing_b200.device_inputs import bf16_tensor
    x = bf16_tensor(inp.x_bits, "cuda")
    wr = torch.from_numpy(inp.w_router).cuda()
    b = torch.from_numpy(inp.expert_bias).cuda()
    i_ref, w_ref = api.moe_route(x, None, wr, b, E=wl.E, k=wl.k, eps=wl.eps, scale=wl.router_scale)
    # forward with dummy experts: only the router outputs are compared
    W = api.ExpertWeights(act=0 if wl.act == "swiglu" else 1, fmt=0,
                          w1=torch.zeros((wl.E, (2 if wl.act == "swiglu" else 1) * wl.I, wl.H),
                                         dtype=torch.bfloat16, device="cuda"),
                          w2=torch.zeros((wl.E, wl.H, wl.I), dtype=torch.bfloat16, device="cuda"))
    _, i_fwd, w_fwd, _ = api.moe_forward(x, W, wr, b, E=wl.E, k=wl.k, I=wl.I, eps=wl.eps,
                                         router_scale=wl.router_scale, out_scale=wl.out_scale)
    torch.cuda.synchronize()
    assert torch.equal(i_fwd, i_ref)
    assert torch.equal(w_fwd.view(torch.int32), w_ref.view(torch.int32))
