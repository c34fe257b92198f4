"""Copy a seeded workload (``inputs.MoEInputs``) to device tensors in the
layouts of include/moe.h.  Marshalling only."""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

from . import abi
from .api import ExpertWeights
from .inputs import MoEInputs


def bf16_tensor(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def u32_tensor(words: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(words).view(np.int32)).to(device)


def u8_tensor(b: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(b, dtype=np.uint8)).to(device)


def f32_tensor(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def _weights(src: dict, act: int, fmt: str, limit: float, device) -> ExpertWeights:
    """ExpertWeights from a dict with keys w1_bits / w1_q / w1_scale / w1_bias /
    w1_global and the same for w2 (whichever the format uses)."""
    if fmt == "bf16":
        return ExpertWeights(act=act, fmt=abi.MOE_W_BF16, w1=bf16_tensor(src["w1_bits"], device),
                             w2=bf16_tensor(src["w2_bits"], device), swiglu_limit=limit)
    if fmt == "nvfp4":
        return ExpertWeights(act=act, fmt=abi.MOE_W_NVFP4, w1=u8_tensor(src["w1_q"], device),
                             w2=u8_tensor(src["w2_q"], device), w1_scale=u8_tensor(src["w1_scale"], device),
                             w2_scale=u8_tensor(src["w2_scale"], device),
                             w1_global=f32_tensor(src["w1_global"], device),
                             w2_global=f32_tensor(src["w2_global"], device), swiglu_limit=limit)
    return ExpertWeights(act=act, fmt=abi.MOE_W_AFFINE4_G64,
                         w1=u32_tensor(src["w1_q"], device), w2=u32_tensor(src["w2_q"], device),
                         w1_scale=bf16_tensor(src["w1_scale"], device), w1_bias=bf16_tensor(src["w1_bias"], device),
                         w2_scale=bf16_tensor(src["w2_scale"], device), w2_bias=bf16_tensor(src["w2_bias"], device),
                         swiglu_limit=limit)


@dataclasses.dataclass
class DeviceInputs:
    x: torch.Tensor
    w_router: torch.Tensor
    expert_bias: torch.Tensor
    W: ExpertWeights
    logits: Optional[torch.Tensor] = None


def to_device(inp: MoEInputs, device="cuda", with_x: bool = True) -> DeviceInputs:
    wl = inp.wl
    act = abi.MOE_ACT_SWIGLU if wl.act == "swiglu" else abi.MOE_ACT_RELU2
    src = {f: getattr(inp, f) for f in ("w1_bits", "w2_bits", "w1_q", "w2_q", "w1_scale", "w2_scale", "w1_bias",
                                         "w2_bias", "w1_global", "w2_global")}
    W = _weights(src, act, wl.fmt, wl.swiglu_limit, device)
    x = bf16_tensor(inp.x_bits, device) if with_x else None
    return DeviceInputs(x=x, w_router=torch.from_numpy(inp.w_router).to(device),
                        expert_bias=torch.from_numpy(inp.expert_bias).to(device), W=W)


def shared_to_device(inp: MoEInputs, device="cuda") -> Optional[ExpertWeights]:
    """The shared expert's weights (None when the workload has none)."""
    wl, sh = inp.wl, inp.shared
    if not sh:
        return None
    act = abi.MOE_ACT_SWIGLU if wl.act == "swiglu" else abi.MOE_ACT_RELU2
    return _weights(sh, act, wl.fmt, wl.swiglu_limit, device)


def weight_bytes(inp: MoEInputs, experts) -> int:
    """Bytes of the given experts' weights (codes, scales and biases included)."""
    wl = inp.wl
    n1 = (2 if wl.act == "swiglu" else 1) * wl.I
    per = (n1 * wl.H + wl.H * wl.I)
    if wl.fmt == "bf16":
        b = per * 2
    elif wl.fmt == "nvfp4":
        b = per // 2 + per // 16 + 2 * 4
    else:
        b = per // 2 + (per // 64) * 4
    return int(b * len(experts))
