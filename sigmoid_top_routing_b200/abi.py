"""ctypes view of the C ABI in include/moe.h (argument marshalling only).

The shared library is built in-tree by ``python -m sigmoid_top_routing_b200.build``
(or ``__graft_entry__.build()``).  Loading fails loudly when it is missing:
there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int32, c_size_t, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libmoe_b200.so")

# moe_status
MOE_OK, MOE_ERR_NULL, MOE_ERR_SHAPE, MOE_ERR_ALIGN, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, \
    MOE_ERR_CUDA, MOE_ERR_DEVICE = range(8)
STATUS_NAMES = ["MOE_OK", "MOE_ERR_NULL", "MOE_ERR_SHAPE", "MOE_ERR_ALIGN", "MOE_ERR_UNSUPPORTED",
                "MOE_ERR_WORKSPACE", "MOE_ERR_CUDA", "MOE_ERR_DEVICE"]
MOE_ACT_SWIGLU, MOE_ACT_RELU2 = 0, 1
MOE_W_BF16, MOE_W_AFFINE4_G64, MOE_W_NVFP4 = 0, 1, 2
MOE_DISPATCH_AUTO, MOE_DISPATCH_GEMV, MOE_DISPATCH_GEMM = 0, 1, 2
MOE_COMBINE_ATOMIC, MOE_COMBINE_ORDERED = 0, 1
MOE_SCORE_SIGMOID, MOE_SCORE_SOFTMAX = 0, 1
MOE_STAGE_ROUTE, MOE_STAGE_PLAN, MOE_STAGE_UP, MOE_STAGE_DOWN, MOE_STAGE_FINAL, MOE_STAGE_GATHER = range(6)
MOE_TILE_M = 128


class moe_dims(ctypes.Structure):
    _fields_ = [("T", c_int32), ("H", c_int32), ("E", c_int32), ("k", c_int32), ("I", c_int32)]


class moe_experts_w(ctypes.Structure):
    _fields_ = [("fmt", c_int32), ("act", c_int32),
                ("w1", c_void_p), ("w1_scale", c_void_p), ("w1_bias", c_void_p),
                ("w2", c_void_p), ("w2_scale", c_void_p), ("w2_bias", c_void_p),
                ("swiglu_limit", c_float), ("w1_global", c_void_p), ("w2_global", c_void_p)]


class moe_router_cfg(ctypes.Structure):
    _fields_ = [("score", c_int32), ("norm_topk", c_int32)]


class moe_exec_cfg(ctypes.Structure):
    _fields_ = [("dispatch", c_int32), ("combine", c_int32)]


class moe_plan_t(ctypes.Structure):
    _fields_ = [("counts", c_void_p), ("offsets", c_void_p), ("perm", c_void_p), ("inv", c_void_p),
                ("tiles", c_void_p)]


class moe_ws_layout(ctypes.Structure):
    _fields_ = [("y_acc", c_size_t), ("h", c_size_t), ("xs", c_size_t), ("scratch", c_size_t),
                ("total", c_size_t)]


# name -> (restype, argtypes), exactly the declarations of include/moe.h
PROTOTYPES = {
    "moe_workspace_bytes": (c_size_t, [POINTER(moe_dims), c_int32]),
    "moe_workspace_layout": (c_int32, [POINTER(moe_dims), c_int32, POINTER(moe_ws_layout)]),
    "moe_workspace_bytes_ex": (c_size_t, [POINTER(moe_dims), c_int32, POINTER(moe_exec_cfg)]),
    "moe_workspace_layout_ex": (c_int32, [POINTER(moe_dims), c_int32, POINTER(moe_exec_cfg),
                                          POINTER(moe_ws_layout)]),
    "moe_route": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, POINTER(moe_dims), c_float, c_float,
                            c_void_p, c_void_p, c_void_p]),
    "moe_plan": (c_int32, [c_void_p, POINTER(moe_dims), POINTER(moe_plan_t), c_void_p, c_size_t, c_void_p]),
    "moe_experts": (c_int32, [c_void_p, POINTER(moe_plan_t), c_void_p, POINTER(moe_dims),
                              POINTER(moe_experts_w), c_float, c_void_p, c_void_p, c_size_t, c_void_p]),
    "moe_forward": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, POINTER(moe_dims), c_float, c_float,
                              c_float, POINTER(moe_experts_w), c_void_p, c_void_p, POINTER(moe_plan_t),
                              c_void_p, c_void_p, c_size_t, c_void_p]),
    "moe_experts_ex": (c_int32, [c_void_p, POINTER(moe_plan_t), c_void_p, POINTER(moe_dims),
                                 POINTER(moe_experts_w), POINTER(moe_exec_cfg), c_int32, c_void_p, c_float,
                                 c_void_p, c_void_p, c_size_t, c_void_p]),
    "moe_route_ex": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, POINTER(moe_dims), c_float, c_float,
                               POINTER(moe_router_cfg), c_void_p, c_void_p, c_void_p]),
    "moe_forward_ex": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, POINTER(moe_dims), c_float, c_float,
                                 c_float, POINTER(moe_router_cfg), POINTER(moe_exec_cfg), c_void_p,
                                 POINTER(moe_experts_w), c_void_p,
                                 c_void_p, POINTER(moe_plan_t), c_void_p, c_void_p, c_size_t, c_void_p]),
    "moe_shared_expert": (c_int32, [c_void_p, POINTER(moe_experts_w), POINTER(moe_dims), c_void_p, c_void_p,
                                    c_size_t, c_void_p]),
    "moe_shared_expert_ex": (c_int32, [c_void_p, POINTER(moe_experts_w), POINTER(moe_dims),
                                       POINTER(moe_exec_cfg), c_void_p, c_void_p, c_size_t, c_void_p]),
    "moe_forward_host": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, POINTER(moe_dims), c_float,
                                   c_float, c_float, POINTER(moe_experts_w), c_void_p, c_void_p,
                                   POINTER(moe_plan_t), c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "moe_forward_static": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, POINTER(moe_dims), c_float,
                                     c_float, c_float, POINTER(moe_experts_w), c_void_p, c_void_p,
                                     POINTER(moe_plan_t), c_void_p, c_void_p]),
    "moe_profile_hook": (c_int32, [c_void_p, c_void_p, c_int32]),
    "moe_last_launch_count": (c_int32, []),
    "moe_set_dispatch": (c_int32, [c_int32]),
    "moe_set_combine": (c_int32, [c_int32]),
    "moe_device_error": (c_int32, [POINTER(c_int32), c_void_p]),
    "moe_wait_bound_check": (c_int32, [ctypes.c_uint32, c_void_p]),
    "moe_last_error": (c_char_p, []),
    "moe_version": (c_char_p, []),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CUDA library missing at {LIB_PATH}: build it with "
                           "`python -m sigmoid_top_routing_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in PROTOTYPES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES[status] if 0 <= status < 8 else status}: {msg}")


def check(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoEError(status, where, load().moe_last_error().decode(errors="replace"))
