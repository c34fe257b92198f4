"""The C-ABI library loads without a GPU, exports every call include/moe.h
declares, and refuses bad arguments on the host before anything launches
(bloomery PR #235 and vllm.cpp PR #684 refuse mis-shaped or mis-placed
tensors before dispatch; these tests need no GPU because validation runs
first and returns a status).  Fake pointer values below are never
dereferenced: every call fails validation before it touches them."""
import ctypes
import os
import re

import pytest

from sigmoid_top_routing_b200 import abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def _declared():
    src = open(HEADER).read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)


@pytest.fixture(scope="module")
def lib():
    from sigmoid_top_routing_b200 import build
    build.build(quiet=True)
    return abi.load()


def test_header_declares_the_documented_calls():
    names = set(_declared())
    for n in ["moe_route", "moe_plan", "moe_experts", "moe_forward", "moe_workspace_bytes",
              "moe_last_error", "moe_device_error", "moe_forward_host"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name
        assert name in abi.PROTOTYPES, name
    assert lib.moe_version().decode().startswith("moe-b200")


def _d(T=16, H=256, E=8, k=2, I=128):
    return abi.moe_dims(T, H, E, k, I)


def test_workspace_bytes_and_layout(lib):
    d = _d(T=4096, H=2048, E=32, k=4, I=1792)
    n = lib.moe_workspace_bytes(ctypes.byref(d), 0)
    L = abi.moe_ws_layout()
    assert lib.moe_workspace_layout(ctypes.byref(d), 0, ctypes.byref(L)) == abi.MOE_OK
    assert L.total == n
    assert L.y_acc == 0 and L.h >= 4096 * 2048 * 4 and L.xs >= L.h + 16384 * 1792 * 2
    assert all(v % 256 == 0 for v in (L.y_acc, L.h, L.xs, L.scratch, L.total))
    assert lib.moe_workspace_bytes(ctypes.byref(_d(H=100)), 0) == 0
    assert lib.moe_workspace_bytes(ctypes.byref(d), 7) == 0


def test_ordered_combine_sizes_the_slot_outputs(lib):
    """Under the ordered combine the y_acc region holds (P, H) fp32 slot rows."""
    d = _d(T=4096, H=2048, E=32, k=4, I=1792)
    old = lib.moe_set_combine(abi.MOE_COMBINE_ORDERED)
    try:
        assert lib.moe_set_combine(abi.MOE_COMBINE_ORDERED) == abi.MOE_COMBINE_ORDERED
        L = abi.moe_ws_layout()
        assert lib.moe_workspace_layout(ctypes.byref(d), 0, ctypes.byref(L)) == abi.MOE_OK
        assert L.h >= 4096 * 4 * 2048 * 4
        ordered_total = L.total
    finally:
        lib.moe_set_combine(old)
    assert lib.moe_set_combine(99) == old                     # invalid value ignored
    assert lib.moe_workspace_bytes(ctypes.byref(d), 0) < ordered_total


@pytest.mark.parametrize("bad,status", [
    (dict(T=-1), abi.MOE_ERR_SHAPE), (dict(H=100), abi.MOE_ERR_SHAPE), (dict(H=32), abi.MOE_ERR_SHAPE),
    (dict(I=96), abi.MOE_ERR_SHAPE), (dict(E=0), abi.MOE_ERR_SHAPE), (dict(E=257), abi.MOE_ERR_SHAPE),
    (dict(k=0), abi.MOE_ERR_SHAPE), (dict(k=9), abi.MOE_ERR_SHAPE), (dict(E=64, k=33), abi.MOE_ERR_SHAPE),
])
def test_route_refuses_bad_sizes(lib, bad, status):
    d = _d(**bad)
    st = lib.moe_route(0x10000, None, 0x20000, None, ctypes.byref(d), 1e-6, 1.0, 0x30000, 0x40000, None)
    assert st == status
    assert lib.moe_last_error()


def test_route_refuses_bad_pointers(lib):
    d = _d()
    D = ctypes.byref(d)
    assert lib.moe_route(None, None, 0x20000, None, D, 1e-6, 1.0, 0x30000, 0x40000, None) == abi.MOE_ERR_NULL
    assert lib.moe_route(0x10000, 0x50000, 0x20000, None, D, 1e-6, 1.0, 0x30000, 0x40000, None) == abi.MOE_ERR_NULL
    assert lib.moe_route(0x10000, None, None, None, D, 1e-6, 1.0, 0x30000, 0x40000, None) == abi.MOE_ERR_NULL
    assert lib.moe_route(0x10000, None, 0x20000, None, D, 1e-6, 1.0, None, 0x40000, None) == abi.MOE_ERR_NULL
    assert lib.moe_route(0x10008, None, 0x20000, None, D, 1e-6, 1.0, 0x30000, 0x40000, None) == abi.MOE_ERR_ALIGN


def _plan():
    return abi.moe_plan_t(0x1000, 0x2000, 0x3000, 0x4000, 0x5000)


def _weights(**over):
    w = dict(fmt=0, act=0, w1=0x100000, w1_scale=None, w1_bias=None, w2=0x200000, w2_scale=None, w2_bias=None)
    w.update(over)
    return abi.moe_experts_w(**w)


def test_plan_refuses_small_workspace(lib):
    d = _d()
    n = lib.moe_workspace_bytes(ctypes.byref(d), 0)
    p = _plan()
    st = lib.moe_plan(0x10000, ctypes.byref(d), ctypes.byref(p), 0x100000, n - 1, None)
    assert st == abi.MOE_ERR_WORKSPACE
    st = lib.moe_plan(0x10000, ctypes.byref(d), ctypes.byref(p), None, n, None)
    assert st == abi.MOE_ERR_WORKSPACE
    st = lib.moe_plan(0x10000, ctypes.byref(d), ctypes.byref(p), 0x100080, n, None)
    assert st == abi.MOE_ERR_ALIGN
    bad = abi.moe_plan_t(0x1000, None, 0x3000, 0x4000, 0x5000)
    st = lib.moe_plan(0x10000, ctypes.byref(d), ctypes.byref(bad), 0x100000, n, None)
    assert st == abi.MOE_ERR_NULL


def test_experts_refuses_bad_weights(lib):
    d = _d()
    n = lib.moe_workspace_bytes(ctypes.byref(d), 0)
    p = _plan()

    def call(W, x=0x10000, y=0x20000):
        return lib.moe_experts(x, ctypes.byref(p), 0x30000, ctypes.byref(d), ctypes.byref(W), 1.0, y,
                               0x1000000, n, None)
    assert call(_weights(act=5)) == abi.MOE_ERR_UNSUPPORTED
    assert call(_weights(fmt=9)) == abi.MOE_ERR_UNSUPPORTED
    assert call(_weights(w1=None)) == abi.MOE_ERR_NULL
    assert call(_weights(w2=0x200004)) == abi.MOE_ERR_ALIGN
    assert call(_weights(fmt=1)) == abi.MOE_ERR_NULL                 # affine-4 without scales
    assert call(_weights(), x=0x10002) == abi.MOE_ERR_ALIGN
    assert call(_weights(), y=None) == abi.MOE_ERR_NULL


def test_swiglu_limit_must_be_finite_and_non_negative(lib):
    d = _d()
    n = lib.moe_workspace_bytes(ctypes.byref(d), 0)
    p = _plan()
    for bad in (-1.0, float("nan"), float("inf")):
        W = _weights()
        W.swiglu_limit = bad
        assert lib.moe_experts(0x10000, ctypes.byref(p), 0x30000, ctypes.byref(d), ctypes.byref(W), 1.0,
                               0x20000, 0x1000000, n, None) == abi.MOE_ERR_SHAPE


def test_router_cfg_refuses_unknown_modes(lib):
    d = _d()
    for cfg in (abi.moe_router_cfg(7, 1), abi.moe_router_cfg(0, 2)):
        assert lib.moe_route_ex(0x10000, None, 0x20000, None, ctypes.byref(d), 1e-6, 1.0, ctypes.byref(cfg),
                                0x30000, 0x40000, None) == abi.MOE_ERR_UNSUPPORTED
        assert lib.moe_forward_ex(0x10000, None, 0x20000, None, ctypes.byref(d), 1e-6, 1.0, 1.0,
                                  ctypes.byref(cfg), None, None, ctypes.byref(_weights()), 0x30000, 0x40000,
                                  ctypes.byref(_plan()), 0x50000, 0x1000000, 1 << 30, None) == abi.MOE_ERR_UNSUPPORTED


def test_shared_expert_refuses_bad_shapes(lib):
    W = _weights()
    for d in (_d(E=2, k=1), _d(E=4, k=2)):
        assert lib.moe_shared_expert(0x10000, ctypes.byref(W), ctypes.byref(d), 0x20000, 0x1000000, 1 << 30,
                                     None) == abi.MOE_ERR_SHAPE
    d = _d(E=1, k=1)
    assert lib.moe_shared_expert(0x10000, ctypes.byref(W), ctypes.byref(d), None, 0x1000000, 1 << 30,
                                 None) == abi.MOE_ERR_NULL
    assert lib.moe_shared_expert(0x10000, ctypes.byref(W), ctypes.byref(d), 0x20004, 0x1000000, 1 << 30,
                                 None) == abi.MOE_ERR_ALIGN


def test_forward_refuses_missing_router(lib):
    d = _d()
    n = lib.moe_workspace_bytes(ctypes.byref(d), 0)
    p, W = _plan(), _weights()
    st = lib.moe_forward(0x10000, None, None, None, ctypes.byref(d), 1e-6, 1.0, 1.0, ctypes.byref(W),
                         0x30000, 0x40000, ctypes.byref(p), 0x50000, 0x1000000, n, None)
    assert st == abi.MOE_ERR_NULL
    assert "w_router" in lib.moe_last_error().decode()


def test_dispatch_switch(lib):
    old = lib.moe_set_dispatch(abi.MOE_DISPATCH_GEMV)
    assert lib.moe_set_dispatch(99) == abi.MOE_DISPATCH_GEMV      # invalid value ignored
    assert lib.moe_set_dispatch(old) == abi.MOE_DISPATCH_GEMV


def test_exec_cfg_is_per_call_and_validated(lib):
    """The combine mode passed per call sizes the workspace whatever the
    process-wide default is; values outside the enums are refused."""
    d = _d()
    atomic, ordered = abi.moe_exec_cfg(0, abi.MOE_COMBINE_ATOMIC), abi.moe_exec_cfg(0, abi.MOE_COMBINE_ORDERED)
    n_a = lib.moe_workspace_bytes_ex(ctypes.byref(d), 0, ctypes.byref(atomic))
    n_o = lib.moe_workspace_bytes_ex(ctypes.byref(d), 0, ctypes.byref(ordered))
    assert n_o > n_a > 0
    old = lib.moe_set_combine(abi.MOE_COMBINE_ORDERED)
    try:
        assert lib.moe_workspace_bytes_ex(ctypes.byref(d), 0, ctypes.byref(atomic)) == n_a
        assert lib.moe_workspace_bytes_ex(ctypes.byref(d), 0, None) == n_o      # NULL: the process default
    finally:
        lib.moe_set_combine(old)
    for bad in (abi.moe_exec_cfg(7, 0), abi.moe_exec_cfg(0, 5)):
        assert lib.moe_workspace_bytes_ex(ctypes.byref(d), 0, ctypes.byref(bad)) == 0
        assert lib.moe_experts_ex(0x10000, ctypes.byref(_plan()), 0x30000, ctypes.byref(d),
                                  ctypes.byref(_weights()), ctypes.byref(bad), -1, None, 1.0, 0x20000,
                                  0x1000000, n_o, None) == abi.MOE_ERR_UNSUPPORTED
        assert lib.moe_forward_ex(0x10000, None, 0x20000, None, ctypes.byref(d), 1e-6, 1.0, 1.0, None,
                                  ctypes.byref(bad), None, ctypes.byref(_weights()), 0x30000, 0x40000,
                                  ctypes.byref(_plan()), 0x50000, 0x1000000, 1 << 30, None) == abi.MOE_ERR_UNSUPPORTED


def test_experts_ex_refuses_bad_skip(lib):
    d = _d()
    n = lib.moe_workspace_bytes(ctypes.byref(d), 0)

    def call(skip, dd=d):
        return lib.moe_experts_ex(0x10000, ctypes.byref(_plan()), 0x30000, ctypes.byref(dd),
                                  ctypes.byref(_weights()), None, skip, None, 1.0, 0x20000, 0x1000000, n, None)
    assert call(-2) == abi.MOE_ERR_SHAPE
    assert call(d.E) == abi.MOE_ERR_SHAPE
    assert "skip_expert" in lib.moe_last_error().decode()
    assert call(0, _d(E=1, k=1)) == abi.MOE_ERR_SHAPE
    assert lib.moe_experts_ex(0x10000, ctypes.byref(_plan()), 0x30000, ctypes.byref(d), ctypes.byref(_weights()),
                              None, -1, 0x40004, 1.0, 0x20000, 0x1000000, n, None) == abi.MOE_ERR_ALIGN
