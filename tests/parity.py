"""Comparison of the CUDA path with the float64 oracle (test helper).

Gates (tolerances fixed in one place):
  * picks: bit-exact except rows whose oracle score margin among the first
    k + 1 ranks is below 1e-6 (near-ties), which are counted;
  * weights: relative 2e-6 (fp32 sigmoid and division against float64);
  * plan: bit-exact against the oracle's plan of the GPU's own picks;
  * output: NaN rows identical; on the rest rel-L2 <= 1e-2 and max-abs <= 5e-2
    for bf16 weights, rel-L2 <= 3e-2 for affine 4-bit weights.  Rows whose
    picks differ (near-ties only) are compared with the oracle's expert stage
    run on the GPU's picks.
"""
from __future__ import annotations

import dataclasses

import numpy as np

import oracle as O

TIE_MARGIN = 1e-6
W_RTOL = 2e-6
BF16_REL_L2 = 1e-2
BF16_MAX_ABS = 5e-2
AFFINE4_REL_L2 = 3e-2


@dataclasses.dataclass
class ParityReport:
    rows: int
    near_ties: int
    idx_mismatch_near_tie: int
    nan_rows: int
    rel_l2: float
    max_abs: float

    def as_dict(self):
        return dataclasses.asdict(self)


def bf16_bits_to_f64(bits):
    return O.bf16_to_f64(bits)


def check(inp, tokens, gpu_idx, gpu_w, gpu_y_bits, *, logits=None, gpu_plan=None, full_plan=True):
    """Compare GPU results for token rows `tokens` against the oracle.

    gpu_* are numpy arrays for those rows only (gpu_plan for all rows when
    full_plan).  Returns a ParityReport; raises AssertionError on a gate."""
    wl = inp.wl
    tokens = np.asarray(tokens)
    ref = O.moe_block(inp, tokens, use_logits=logits)
    margins = O.tie_margins(ref["c"], wl.k)
    near = margins < TIE_MARGIN
    nan_rows = np.all(np.isnan(ref["c"]), axis=1)

    same = np.all(gpu_idx == ref["idx"], axis=1)
    bad = ~same & ~near
    assert not bad.any(), f"picks differ on non-tie rows {tokens[bad][:10].tolist()}"
    # NaN rows pick 0..k-1 on both sides
    if nan_rows.any():
        assert np.all(gpu_idx[nan_rows] == np.arange(wl.k)), "all-NaN row picks"
        assert np.isnan(gpu_w[nan_rows]).all()

    fin = same & ~nan_rows
    np.testing.assert_allclose(gpu_w[fin], ref["w"][fin], rtol=W_RTOL, atol=1e-7)

    y = bf16_bits_to_f64(gpu_y_bits)
    y_ref = ref["y"].copy()
    diff_rows = np.nonzero(~same)[0]
    if len(diff_rows):
        alt = O.moe_block(inp, tokens[diff_rows], use_logits=None if logits is None else logits,
                          idx=gpu_idx[diff_rows])
        y_ref[diff_rows] = alt["y"]
    yn = np.isnan(y).any(axis=1)
    rn = np.isnan(y_ref).any(axis=1)
    assert np.array_equal(yn, rn), f"NaN rows differ: gpu {np.nonzero(yn)[0][:10]} oracle {np.nonzero(rn)[0][:10]}"
    ok = ~rn
    err = y[ok] - y_ref[ok]
    denom = np.linalg.norm(y_ref[ok])
    rel_l2 = float(np.linalg.norm(err) / denom) if denom > 0 else float(np.linalg.norm(err))
    max_abs = float(np.abs(err).max()) if err.size else 0.0
    if wl.fmt == "bf16":
        assert rel_l2 <= BF16_REL_L2, f"rel-L2 {rel_l2}"
        assert max_abs <= BF16_MAX_ABS, f"max-abs {max_abs}"
    else:
        assert rel_l2 <= AFFINE4_REL_L2, f"rel-L2 {rel_l2}"

    if gpu_plan is not None and full_plan:
        want = O.plan(gpu_plan["idx"], wl.E)
        for key in ("counts", "offsets", "perm", "inv", "tiles"):
            assert np.array_equal(np.asarray(gpu_plan[key], dtype=np.int64), want[key]), f"plan.{key}"

    return ParityReport(rows=len(tokens), near_ties=int(near.sum()),
                        idx_mismatch_near_tie=int((~same & near).sum()), nan_rows=int(nan_rows.sum()),
                        rel_l2=rel_l2, max_abs=max_abs)
