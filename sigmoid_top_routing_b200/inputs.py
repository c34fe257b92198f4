"""Seeded synthetic inputs for the routed MoE block's workloads.

This module only draws and encodes numbers: it holds none of the block's
arithmetic (no logits, sigmoid, selection, normalisation, expert math or
combine).  Both the CUDA path and the float64 oracle take their inputs from
here and nowhere else.

Recipe (every workload):
  * ``np.random.SeedSequence(seed).spawn(6)`` gives one independent stream per
    tensor, in this order: x, W_router, expert_bias, W1 (gate_up or up),
    W2 (down), extras (NaN rows, hot experts).  A tensor can therefore be
    regenerated without drawing the others.
  * x ~ N(0, 1), expert weights ~ N(0, 0.02), W_router ~ N(0, 0.02) kept in
    fp32, expert_bias ~ U(-0.1, 0.1) fp32.
  * bf16 tensors are fp32 draws rounded to nearest-even; they are carried as
    raw uint16 bit patterns (``*_bits``) so every consumer sees the same bytes.
  * Gated (SwiGLU) experts store gate_up as (E, 2I, H), gate rows first, then
    up rows; down is (E, H, I) (TileGym PR #187, "Weight layout and routing").
    Non-gated relu^2 experts store up as (E, I, H) (vllm.cpp PR #684, "The
    seam decision").
  * MLX-style affine 4-bit experts: each row is cut into groups of 64 along K;
    per group scale = (max - min) / 15 and bias = min, both stored as bf16;
    q = clip(round((w - bias) / scale), 0, 15); eight 4-bit codes per uint32,
    little-endian, the low nibble holding the lowest k.  The dequantised value
    is scale * q + bias.
  * NVFP4 experts in the ModelOpt layout the pages name (TensorFold issue #548:
    "weight uint8 [N, K/2], weight_scale e4m3 [N, K/16], weight_scale_2 as the
    global scale"): per expert and projection a global scale
    g = max|w| / (6 * 448) (fp32); per block of 16 along K a scale
    s = max|w_block| / (6 * g) rounded to the nearest e4m3 code (ties to the
    even code, at most 448); each weight w / (s * g) rounded to the nearest
    e2m1 code (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; ties to the even code,
    at most 6).  Two codes per byte, the low nibble holding the lower k.
    Only the encoding lives here: it picks codes on the two grids below and
    never turns a code back into a value.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "MoEInputs", "make_inputs", "f32_to_bf16_bits",
    "bf16_bits_to_f32", "quantize_affine4_g64", "unpack_affine4", "quantize_nvfp4",
]

AFFINE_GROUP = 64


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shapes and scalars of one synthetic workload."""
    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    act: str = "swiglu"          # "swiglu" | "relu2"
    fmt: str = "bf16"            # "bf16" | "affine4" | "nvfp4"
    eps: float = 1e-6
    router_scale: float = 1.0
    out_scale: float = 1.0
    nan_rows: int = 0            # token rows of x set to NaN (all-NaN router logits)
    hot_experts: int = 0         # experts given a bias offset
    hot_delta: float = 0.0       # that offset (found by bisection on the oracle's routing)
    score: str = "sigmoid"       # router score: "sigmoid" | "softmax"
    norm_topk: bool = True       # divide the picked scores by their sum + eps
    swiglu_limit: float = 0.0    # clamp of the SwiGLU inputs (0: off)
    shared_I: int = 0            # intermediate width of a shared expert (0: none)
    seed: int = 0

    def with_T(self, T: int, name: Optional[str] = None) -> "Workload":
        nan_rows = self.nan_rows
        if nan_rows:
            nan_rows = max(1, int(round(0.01 * T)))
        return dataclasses.replace(self, T=T, nan_rows=nan_rows, name=name or f"{self.name}@T{T}")

    @property
    def P(self) -> int:
        return self.T * self.k


# The hot-expert bias offset below was found by tests/golden/make_golden.py
# (bisection on the oracle's routing of this exact seeded input) so that the
# four hot experts take 40 +- 2 % of the routed pairs.
NEMOTRON_HOT_DELTA = 0.3828125

WORKLOADS = {
    # tiny block: T=16, H=256, E=8, top-2, I=128, SwiGLU
    "tiny": Workload("tiny", T=16, H=256, E=8, k=2, I=128),
    # LFM2-8B-A1B-shaped decode
    "lfm2_decode_t8": Workload("lfm2_decode_t8", T=8, H=2048, E=32, k=4, I=1792),
    # the same block at prefill, 1 % of token rows all-NaN in the router logits
    "lfm2_prefill_t4096": Workload("lfm2_prefill_t4096", T=4096, H=2048, E=32, k=4, I=1792,
                                   nan_rows=41),
    # Nemotron-H-style non-gated relu^2 experts, routed scale on the output
    "nemotron_relu2_t2048": Workload("nemotron_relu2_t2048", T=2048, H=2048, E=64, k=6, I=1024,
                                     act="relu2", out_scale=2.5, hot_experts=4,
                                     hot_delta=NEMOTRON_HOT_DELTA),
}
for _T in (1, 8, 64, 512, 8192):
    WORKLOADS[f"affine4_t{_T}"] = Workload(f"affine4_t{_T}", T=_T, H=2048, E=64, k=4, I=1536,
                                           fmt="affine4")
# the same block with NVFP4 experts (ModelOpt layout)
for _T in (1, 8, 64, 512, 8192):
    WORKLOADS[f"nvfp4_t{_T}"] = Workload(f"nvfp4_t{_T}", T=_T, H=2048, E=64, k=4, I=1536, fmt="nvfp4")


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest-even) and return the uint16 bit pattern.

    NaN stays a quiet NaN."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    rounded = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16))
    out = rounded.astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 exactly."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def quantize_affine4_g64(w: np.ndarray):
    """Encode an fp32 (..., N, K) weight as MLX-style affine 4-bit, group 64.

    Returns (packed uint32 (..., N, K/8), scale bf16 bits (..., N, K/64),
    bias bf16 bits (..., N, K/64)).  This is input encoding only."""
    *lead, N, K = w.shape
    assert K % AFFINE_GROUP == 0
    g = w.reshape(*lead, N, K // AFFINE_GROUP, AFFINE_GROUP).astype(np.float32)
    lo = g.min(axis=-1)
    hi = g.max(axis=-1)
    scale_bits = f32_to_bf16_bits((hi - lo) / np.float32(15.0))
    bias_bits = f32_to_bf16_bits(lo)
    scale = bf16_bits_to_f32(scale_bits)[..., None]
    bias = bf16_bits_to_f32(bias_bits)[..., None]
    safe = np.where(scale == 0, np.float32(1.0), scale)
    q = np.clip(np.rint((g - bias) / safe), 0, 15).astype(np.uint32)
    q = q.reshape(*lead, N, K // 8, 8)
    shifts = (np.arange(8, dtype=np.uint32) * np.uint32(4))
    packed = np.bitwise_or.reduce(q << shifts, axis=-1).astype(np.uint32)
    return packed, scale_bits, bias_bits


# Magnitudes of the e2m1 codes 0..7 (code = sign << 3 | magnitude index), and
# of the finite non-negative e4m3 codes 0..126 (0x7F is NaN): the grids the
# encoder rounds onto, ascending.
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E4M3_GRID = np.array([m / 8.0 * 2.0 ** -6 for m in range(8)] +
                     [(1.0 + m / 8.0) * 2.0 ** (e - 7) for e in range(1, 16) for m in range(8)][:119])


def _round_to_grid(a: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the nearest grid value to each |a| (ties to the even index),
    saturating at the last entry.  Works in the precision of `a`: the grid's
    midpoints are exact in float32."""
    a = np.abs(np.asarray(a))
    mid = ((grid[:-1] + grid[1:]) / 2).astype(a.dtype)
    idx = np.searchsorted(mid, a, side="left")           # a == mid[j] gives j, the lower neighbour
    tie = np.zeros(a.shape, dtype=bool)
    inb = idx < len(mid)
    tie[inb] = a[inb] == mid[idx[inb]]
    return np.where(tie & (idx % 2 == 1), idx + 1, idx).astype(np.int64)


def _round_e2m1(a: np.ndarray) -> np.ndarray:
    """_round_to_grid(a, E2M1_GRID) in three rint regimes: on 2|a| the grid is
    0..4 in steps of 1, then 4..8 in steps of 2, then 8..12 in steps of 4, and
    np.rint rounds ties to even, which is the even code in each regime."""
    a2 = 2 * np.abs(np.asarray(a, dtype=np.float32))
    lo = np.rint(a2)
    mid = np.rint(a2 / 2) + 2
    hi = np.minimum(np.rint(a2 / 4), 3) + 4
    return np.where(a2 < 4, lo, np.where(a2 < 8, mid, hi)).astype(np.int64)


def quantize_nvfp4(w: np.ndarray):
    """Encode an fp32 (N, K) weight as NVFP4 (ModelOpt layout).

    Returns (codes uint8 (N, K/2), block scales uint8 e4m3 codes (N, K/16),
    global scale float32).  Input encoding only."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    assert K % 16 == 0
    amax = float(np.abs(w).max())
    g = np.float32(amax / (6.0 * 448.0)) if amax > 0 else np.float32(1.0)
    blocks = w.reshape(N, K // 16, 16)
    bmax = np.abs(blocks).max(axis=-1).astype(np.float64)
    s_code = _round_to_grid(bmax / (6.0 * float(g)), E4M3_GRID)
    s_val = E4M3_GRID[s_code]
    denom = np.where(s_val == 0, 1.0, s_val * float(g)).astype(np.float32)[..., None]
    mag = _round_e2m1(blocks / denom)
    mag = np.where((s_val == 0)[..., None], 0, mag)
    code = (mag | (np.signbit(blocks) & (mag != 0)).astype(np.int64) << 3).reshape(N, K)
    packed = (code[:, 0::2] | (code[:, 1::2] << 4)).astype(np.uint8)
    return packed, s_code.astype(np.uint8), g


def unpack_affine4(packed: np.ndarray) -> np.ndarray:
    """Unpack (..., K/8) uint32 words into (..., K) 4-bit codes (uint8)."""
    p = np.asarray(packed, dtype=np.uint32)[..., None]
    shifts = (np.arange(8, dtype=np.uint32) * np.uint32(4))
    q = (p >> shifts) & np.uint32(0xF)
    return q.reshape(*p.shape[:-2], p.shape[-2] * 8).astype(np.uint8)


@dataclasses.dataclass
class MoEInputs:
    """One workload's tensors, as host numpy arrays."""
    wl: Workload
    x_bits: np.ndarray                 # (T, H) uint16 bf16
    w_router: np.ndarray               # (E, H) fp32
    expert_bias: np.ndarray            # (E,) fp32
    w1_bits: Optional[np.ndarray]      # bf16: (E, 2I, H) gate-first or (E, I, H) up
    w2_bits: Optional[np.ndarray]      # bf16: (E, H, I)
    w1_q: Optional[np.ndarray] = None  # affine4: (E, N1, H/8) uint32
    w1_scale: Optional[np.ndarray] = None
    w1_bias: Optional[np.ndarray] = None
    w2_q: Optional[np.ndarray] = None  # affine4: (E, H, I/8) uint32
    w2_scale: Optional[np.ndarray] = None
    w2_bias: Optional[np.ndarray] = None
    w1_global: Optional[np.ndarray] = None   # nvfp4: (E,) fp32 global scale of W1 (weight_scale_2)
    w2_global: Optional[np.ndarray] = None   # nvfp4: (E,) fp32 global scale of W2 (the down scale)
    nan_rows: Optional[np.ndarray] = None
    hot: Optional[np.ndarray] = None
    # shared expert (one expert, same format and activation, width shared_I):
    # keys w1_bits, w2_bits (bf16) or w1_q, w1_scale, w1_bias, w2_q, ... (affine),
    # each with a leading dimension of 1
    shared: Optional[dict] = None

    @property
    def n1(self) -> int:
        return (2 if self.wl.act == "swiglu" else 1) * self.wl.I


def _normal_f32(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def _expert_weights(rng, E, N, K, fmt):
    """Draw E experts' (N, K) weights one expert at a time (in stream order)
    and encode them; the encoding of different experts runs on a few threads
    (numpy releases the GIL), which changes no value.
    Returns (bf16 bits, codes, scales, biases or global scales)."""
    if fmt == "bf16":
        out = np.empty((E, N, K), dtype=np.uint16)
        for e in range(E):
            out[e] = f32_to_bf16_bits(_normal_f32(rng, (N, K), 0.02))
        return out, None, None, None
    import concurrent.futures as cf
    import os
    if fmt == "nvfp4":
        q = np.empty((E, N, K // 2), dtype=np.uint8)
        s = np.empty((E, N, K // 16), dtype=np.uint8)
        g = np.empty(E, dtype=np.float32)
    else:
        q = np.empty((E, N, K // 8), dtype=np.uint32)
        s = np.empty((E, N, K // AFFINE_GROUP), dtype=np.uint16)
        g = np.empty((E, N, K // AFFINE_GROUP), dtype=np.uint16)
    enc = quantize_nvfp4 if fmt == "nvfp4" else quantize_affine4_g64

    def one(e, w):
        q[e], s[e], g[e] = enc(w)

    workers = max(1, min(8, os.cpu_count() or 1))
    with cf.ThreadPoolExecutor(max_workers=workers) as ex:
        pending = []
        for e in range(E):
            pending.append(ex.submit(one, e, _normal_f32(rng, (N, K), 0.02)))
            if len(pending) >= 2 * workers:      # bounded memory: at most 2x workers drafts alive
                pending.pop(0).result()
        for f in pending:
            f.result()
    return None, q, s, g


def make_inputs(wl: Workload, *, with_experts: bool = True, hot_delta: Optional[float] = None) -> MoEInputs:
    """Build the seeded inputs of ``wl``.

    ``with_experts=False`` skips the expert weights (router-only studies);
    ``hot_delta`` overrides the recorded hot-expert offset."""
    ss = np.random.SeedSequence(wl.seed).spawn(7)     # the first six streams do not depend on the count
    r_x, r_wr, r_b, r_w1, r_w2, r_extra, r_shared = (np.random.default_rng(s) for s in ss)
    T, H, E, I = wl.T, wl.H, wl.E, wl.I
    x = _normal_f32(r_x, (T, H), 1.0)
    w_router = _normal_f32(r_wr, (E, H), 0.02)
    bias = r_b.uniform(-0.1, 0.1, size=E).astype(np.float32)

    nan_rows = None
    hot = None
    if wl.nan_rows:
        nan_rows = np.sort(r_extra.choice(T, size=wl.nan_rows, replace=False))
        x[nan_rows, :] = np.nan
    if wl.hot_experts:
        hot = np.sort(r_extra.choice(E, size=wl.hot_experts, replace=False))
        delta = wl.hot_delta if hot_delta is None else hot_delta
        bias[hot] += np.float32(delta)

    n1 = (2 if wl.act == "swiglu" else 1) * I
    w1 = w2 = q1 = s1 = b1 = q2 = s2 = b2 = None
    if with_experts:
        w1, q1, s1, b1 = _expert_weights(r_w1, E, n1, H, wl.fmt)
        w2, q2, s2, b2 = _expert_weights(r_w2, E, H, I, wl.fmt)
    g1 = g2 = None
    if wl.fmt == "nvfp4":                       # the fourth value is the global scale
        g1, g2, b1, b2 = b1, b2, None, None
    shared = None
    if with_experts and wl.shared_I:
        Is = wl.shared_I
        sw1, sq1, ss1, sb1 = _expert_weights(r_shared, 1, (2 if wl.act == "swiglu" else 1) * Is, H, wl.fmt)
        sw2, sq2, ss2, sb2 = _expert_weights(r_shared, 1, H, Is, wl.fmt)
        shared = {"w1_bits": sw1, "w2_bits": sw2, "w1_q": sq1, "w1_scale": ss1, "w1_bias": sb1,
                  "w2_q": sq2, "w2_scale": ss2, "w2_bias": sb2}
        if wl.fmt == "nvfp4":                   # the fourth value is the global scale
            shared.update(w1_global=sb1, w2_global=sb2, w1_bias=None, w2_bias=None)
    return MoEInputs(wl=wl, x_bits=f32_to_bf16_bits(x), w_router=w_router, expert_bias=bias,
                     w1_bits=w1, w2_bits=w2, w1_q=q1, w1_scale=s1, w1_bias=b1,
                     w2_q=q2, w2_scale=s2, w2_bias=b2, w1_global=g1, w2_global=g2, nan_rows=nan_rows,
                     hot=hot, shared=shared)
