"""Torch-tensor binding of the C ABI (include/moe.h), same names as the C calls.

Only argument marshalling happens here: pointers, sizes and the current CUDA
stream are passed to the library; every step of the block runs in its CUDA
kernels.  Torch provides device memory and streams.
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import Optional

import torch

from . import abi
from .abi import check, load

__all__ = [
    "ExpertWeights", "Plan", "moe_workspace_bytes", "moe_workspace_layout", "moe_route", "moe_plan",
    "moe_experts", "moe_forward", "moe_forward_host", "moe_shared_expert", "moe_set_dispatch", "moe_set_combine",
    "moe_device_error",
    "moe_last_error", "moe_version", "new_plan", "new_workspace", "dims", "moe_profile_hook",
    "moe_last_launch_count", "exec_cfg", "moe_experts_ex",
]


def dims(T: int, H: int, E: int, k: int, I: int) -> abi.moe_dims:
    return abi.moe_dims(T, H, E, k, I)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


@dataclasses.dataclass
class ExpertWeights:
    """Device tensors of the experts (layouts as in include/moe.h)."""
    act: int                          # abi.MOE_ACT_SWIGLU | abi.MOE_ACT_RELU2
    fmt: int                          # abi.MOE_W_BF16 | abi.MOE_W_AFFINE4_G64 | abi.MOE_W_NVFP4
    w1: torch.Tensor
    w2: torch.Tensor
    w1_scale: Optional[torch.Tensor] = None
    w1_bias: Optional[torch.Tensor] = None
    w2_scale: Optional[torch.Tensor] = None
    w2_bias: Optional[torch.Tensor] = None
    swiglu_limit: float = 0.0
    w1_global: Optional[torch.Tensor] = None   # NVFP4: (E,) fp32 global scales
    w2_global: Optional[torch.Tensor] = None

    def c_struct(self) -> abi.moe_experts_w:
        return abi.moe_experts_w(self.fmt, self.act, _ptr(self.w1), _ptr(self.w1_scale), _ptr(self.w1_bias),
                                 _ptr(self.w2), _ptr(self.w2_scale), _ptr(self.w2_bias), self.swiglu_limit,
                                 _ptr(self.w1_global), _ptr(self.w2_global))

    def clone(self) -> "ExpertWeights":
        c = lambda t: None if t is None else t.clone()  # noqa: E731
        return ExpertWeights(act=self.act, fmt=self.fmt, w1=c(self.w1), w2=c(self.w2), w1_scale=c(self.w1_scale),
                             w1_bias=c(self.w1_bias), w2_scale=c(self.w2_scale), w2_bias=c(self.w2_bias),
                             swiglu_limit=self.swiglu_limit, w1_global=c(self.w1_global),
                             w2_global=c(self.w2_global))


def router_cfg(score: str = "sigmoid", norm_topk: bool = True) -> abi.moe_router_cfg:
    return abi.moe_router_cfg({"sigmoid": abi.MOE_SCORE_SIGMOID, "softmax": abi.MOE_SCORE_SOFTMAX}[score],
                              1 if norm_topk else 0)


def exec_cfg(dispatch: Optional[int] = None, combine: Optional[int] = None) -> Optional[abi.moe_exec_cfg]:
    """A per-call execution choice, or None (the library's process-wide
    defaults) when neither is given; a missing one of the two takes the
    library's default value (AUTO dispatch, atomic combine)."""
    if dispatch is None and combine is None:
        return None
    return abi.moe_exec_cfg(abi.MOE_DISPATCH_AUTO if dispatch is None else dispatch,
                            abi.MOE_COMBINE_ATOMIC if combine is None else combine)


def _ref(c):
    return None if c is None else ctypes.byref(c)


@dataclasses.dataclass
class Plan:
    counts: torch.Tensor   # [E] int32
    offsets: torch.Tensor  # [E+1]
    perm: torch.Tensor     # [P]
    inv: torch.Tensor      # [P]
    tiles: torch.Tensor    # [E+1]

    def c_struct(self) -> abi.moe_plan_t:
        return abi.moe_plan_t(_ptr(self.counts), _ptr(self.offsets), _ptr(self.perm), _ptr(self.inv),
                              _ptr(self.tiles))


def new_plan(T: int, E: int, k: int, device="cuda") -> Plan:
    P = max(T * k, 1)
    z = lambda n: torch.empty(n, dtype=torch.int32, device=device)  # noqa: E731
    return Plan(z(E), z(E + 1), z(P), z(P), z(E + 1))


def moe_workspace_bytes(d: abi.moe_dims, fmt: int = abi.MOE_W_BF16, *, dispatch=None, combine=None) -> int:
    return int(load().moe_workspace_bytes_ex(ctypes.byref(d), fmt, _ref(exec_cfg(dispatch, combine))))


def moe_workspace_layout(d: abi.moe_dims, fmt: int = abi.MOE_W_BF16, *, dispatch=None,
                         combine=None) -> abi.moe_ws_layout:
    out = abi.moe_ws_layout()
    check(load().moe_workspace_layout_ex(ctypes.byref(d), fmt, _ref(exec_cfg(dispatch, combine)),
                                         ctypes.byref(out)), "moe_workspace_layout")
    return out


def new_workspace(d: abi.moe_dims, fmt: int = abi.MOE_W_BF16, device="cuda", *, dispatch=None,
                  combine=None) -> torch.Tensor:
    n = moe_workspace_bytes(d, fmt, dispatch=dispatch, combine=combine)
    if n == 0:
        raise ValueError("invalid sizes for a workspace")
    return torch.empty(n, dtype=torch.uint8, device=device)


def moe_route(x=None, logits=None, w_router=None, expert_bias=None, *, E: int, k: int, eps: float = 1e-6,
              scale: float = 1.0, topk_idx=None, topk_w=None, stream=None, score: str = "sigmoid",
              norm_topk: bool = True):
    src = x if x is not None else logits
    T = src.shape[0]
    H = x.shape[1] if x is not None else (w_router.shape[1] if w_router is not None else 64)
    d = abi.moe_dims(T, H, E, k, 64)
    dev = src.device
    if topk_idx is None:
        topk_idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=dev)
    rc = router_cfg(score, norm_topk)
    check(load().moe_route_ex(_ptr(x), _ptr(logits), _ptr(w_router), _ptr(expert_bias), ctypes.byref(d),
                              eps, scale, ctypes.byref(rc), _ptr(topk_idx), _ptr(topk_w), _stream(stream)),
          "moe_route")
    return topk_idx, topk_w


def moe_plan(topk_idx, *, E: int, H: int = 64, I: int = 64, plan: Optional[Plan] = None, ws=None,
             stream=None) -> Plan:
    T, k = topk_idx.shape
    d = abi.moe_dims(T, H, E, k, I)
    plan = plan or new_plan(T, E, k, topk_idx.device)
    ws = ws if ws is not None else new_workspace(d, device=topk_idx.device)
    cp = plan.c_struct()
    check(load().moe_plan(_ptr(topk_idx), ctypes.byref(d), ctypes.byref(cp), _ptr(ws), ws.numel(),
                          _stream(stream)), "moe_plan")
    return plan


def moe_experts(x, plan: Plan, topk_w, W: ExpertWeights, *, E: int, I: int, out_scale: float = 1.0, y=None,
                ws=None, stream=None, skip: int = -1, y_shared=None, dispatch=None, combine=None):
    """Grouped experts + combine over a plan of E plan experts; ``skip`` >= 0
    names a plan expert whose pairs are computed nowhere and left out (W then
    holds E - 1 experts when skip == E - 1)."""
    T, H = x.shape
    k = topk_w.shape[1]
    d = abi.moe_dims(T, H, E, k, I)
    y = y if y is not None else torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    ex = exec_cfg(dispatch, combine)
    ws = ws if ws is not None else new_workspace(d, W.fmt, x.device, dispatch=dispatch, combine=combine)
    cp, cw = plan.c_struct(), W.c_struct()
    check(load().moe_experts_ex(_ptr(x), ctypes.byref(cp), _ptr(topk_w), ctypes.byref(d), ctypes.byref(cw),
                                _ref(ex), skip, _ptr(y_shared), out_scale, _ptr(y), _ptr(ws), ws.numel(),
                                _stream(stream)), "moe_experts")
    return y


moe_experts_ex = moe_experts


def moe_forward(x, W: ExpertWeights, w_router=None, expert_bias=None, *, E: int, k: int, I: int,
                logits=None, eps: float = 1e-6, router_scale: float = 1.0, out_scale: float = 1.0,
                topk_idx=None, topk_w=None, plan: Optional[Plan] = None, y=None, ws=None, stream=None,
                score: str = "sigmoid", norm_topk: bool = True, y_shared=None, dispatch=None, combine=None):
    T, H = x.shape
    d = abi.moe_dims(T, H, E, k, I)
    dev = x.device
    topk_idx = topk_idx if topk_idx is not None else torch.empty((T, k), dtype=torch.int32, device=dev)
    topk_w = topk_w if topk_w is not None else torch.empty((T, k), dtype=torch.float32, device=dev)
    plan = plan or new_plan(T, E, k, dev)
    y = y if y is not None else torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    ex = exec_cfg(dispatch, combine)
    ws = ws if ws is not None else new_workspace(d, W.fmt, dev, dispatch=dispatch, combine=combine)
    cp, cw, rc = plan.c_struct(), W.c_struct(), router_cfg(score, norm_topk)
    check(load().moe_forward_ex(_ptr(x), _ptr(logits), _ptr(w_router), _ptr(expert_bias), ctypes.byref(d), eps,
                                router_scale, out_scale, ctypes.byref(rc), _ref(ex), _ptr(y_shared),
                                ctypes.byref(cw),
                                _ptr(topk_idx), _ptr(topk_w), ctypes.byref(cp), _ptr(y), _ptr(ws), ws.numel(),
                                _stream(stream)), "moe_forward")
    return y, topk_idx, topk_w, plan


def moe_shared_expert(x, Ws: ExpertWeights, *, I: int, y_shared=None, ws=None, stream=None, dispatch=None,
                      combine=None):
    """fp32 (T, H) output of the shared expert (one expert, weight 1, on every token)."""
    T, H = x.shape
    d = abi.moe_dims(T, H, 1, 1, I)
    y_shared = y_shared if y_shared is not None else torch.empty((T, H), dtype=torch.float32, device=x.device)
    ex = exec_cfg(dispatch, combine)
    ws = ws if ws is not None else new_workspace(d, Ws.fmt, x.device, dispatch=dispatch, combine=combine)
    cw = Ws.c_struct()
    check(load().moe_shared_expert_ex(_ptr(x), ctypes.byref(cw), ctypes.byref(d), _ref(ex), _ptr(y_shared),
                                      _ptr(ws), ws.numel(), _stream(stream)), "moe_shared_expert")
    return y_shared


def moe_forward_host(x_host: torch.Tensor, x_dev, W: ExpertWeights, w_router, expert_bias, *, E: int, k: int,
                     I: int, y_dev, y_host: torch.Tensor, topk_idx, topk_w, plan: Plan, ws, eps: float = 1e-6,
                     router_scale: float = 1.0, out_scale: float = 1.0, stream=None):
    """Host token rows in, host output rows out (the call synchronises its stream)."""
    T, H = x_host.shape
    if x_host.is_cuda or y_host.is_cuda:
        raise ValueError("x_host and y_host must be host tensors")
    d = abi.moe_dims(T, H, E, k, I)
    cp, cw = plan.c_struct(), W.c_struct()
    check(load().moe_forward_host(x_host.data_ptr(), _ptr(x_dev), _ptr(w_router), _ptr(expert_bias),
                                  ctypes.byref(d), eps, router_scale, out_scale, ctypes.byref(cw),
                                  _ptr(topk_idx), _ptr(topk_w), ctypes.byref(cp), _ptr(y_dev),
                                  y_host.data_ptr(), _ptr(ws), ws.numel(), _stream(stream)), "moe_forward_host")
    return y_host


def moe_profile_hook(ev_begin, ev_end, stage: int) -> None:
    """One-shot: the next forward/experts call on this thread records the two
    torch.cuda.Events around `stage`'s kernel (None, None clears)."""
    b = ev_begin.cuda_event if ev_begin is not None else None
    e = ev_end.cuda_event if ev_end is not None else None
    check(load().moe_profile_hook(b, e, stage), "moe_profile_hook")


def moe_last_launch_count() -> int:
    return int(load().moe_last_launch_count())


def moe_set_dispatch(mode: int) -> int:
    return int(load().moe_set_dispatch(mode))


def moe_set_combine(mode: int) -> int:
    return int(load().moe_set_combine(mode))


def moe_device_error(stream=None) -> int:
    code = ctypes.c_int32(0)
    st = load().moe_device_error(ctypes.byref(code), _stream(stream))
    if st not in (abi.MOE_OK, abi.MOE_ERR_DEVICE):
        check(st, "moe_device_error")
    return int(code.value)


def moe_last_error() -> str:
    return load().moe_last_error().decode(errors="replace")


def moe_version() -> str:
    return load().moe_version().decode()
