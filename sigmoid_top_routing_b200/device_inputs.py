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
    if wl.fmt == "bf16":
        W = ExpertWeights(act=act, fmt=abi.MOE_W_BF16, w1=bf16_tensor(inp.w1_bits, device),
                          w2=bf16_tensor(inp.w2_bits, device), swiglu_limit=wl.swiglu_limit)
    else:
        W = ExpertWeights(act=act, fmt=abi.MOE_W_AFFINE4_G64,
                          w1=u32_tensor(inp.w1_q, device), w2=u32_tensor(inp.w2_q, device),
                          w1_scale=bf16_tensor(inp.w1_scale, device), w1_bias=bf16_tensor(inp.w1_bias, device),
                          w2_scale=bf16_tensor(inp.w2_scale, device), w2_bias=bf16_tensor(inp.w2_bias, device),
                          swiglu_limit=wl.swiglu_limit)
    x = bf16_tensor(inp.x_bits, device) if with_x else None
    return DeviceInputs(x=x, w_router=torch.from_numpy(inp.w_router).to(device),
                        expert_bias=torch.from_numpy(inp.expert_bias).to(device), W=W)


def shared_to_device(inp: MoEInputs, device="cuda") -> Optional[ExpertWeights]:
    """The shared expert's weights (None when the workload has none)."""
    wl, sh = inp.wl, inp.shared
    if not sh:
        return None
    act = abi.MOE_ACT_SWIGLU if wl.act == "swiglu" else abi.MOE_ACT_RELU2
    if wl.fmt == "bf16":
        return ExpertWeights(act=act, fmt=abi.MOE_W_BF16, w1=bf16_tensor(sh["w1_bits"], device),
                             w2=bf16_tensor(sh["w2_bits"], device), swiglu_limit=wl.swiglu_limit)
    return ExpertWeights(act=act, fmt=abi.MOE_W_AFFINE4_G64,
                         w1=u32_tensor(sh["w1_q"], device), w2=u32_tensor(sh["w2_q"], device),
                         w1_scale=bf16_tensor(sh["w1_scale"], device), w1_bias=bf16_tensor(sh["w1_bias"], device),
                         w2_scale=bf16_tensor(sh["w2_scale"], device), w2_bias=bf16_tensor(sh["w2_bias"], device),
                         swiglu_limit=wl.swiglu_limit)


def weight_bytes(inp: MoEInputs, experts) -> int:
    """Bytes of the given experts' weights (codes, scales and biases included)."""
    wl = inp.wl
    n1 = (2 if wl.act == "swiglu" else 1) * wl.I
    per = (n1 * wl.H + wl.H * wl.I)
    if wl.fmt == "bf16":
        b = per * 2
    else:
        b = per // 2 + (per // 64) * 4
    return int(b * len(experts))
