"""Pins of the oracle's NVFP4 decoder (TensorFold issue #548: NVFP4 experts
read as stored in the ModelOpt layout, "weight uint8 [N, K/2], weight_scale
e4m3 [N, K/16], weight_scale_2 as the global scale", with a global scale of
its own for the down projection).

Pinned to facts other than the oracle: the e2m1 values written out by hand
from the format (1 sign, 2 exponent, 1 mantissa bit); all 256 e4m3 bytes
against torch's float8_e4m3fn decoder plus hand-decoded bytes; one packed row
decoded by hand (two 16-blocks with different scales, both nibbles of a
byte); a closed form; the brute force over all experts; and planted mutants
(scale per 32, global scale dropped, nibbles swapped) that must go red."""
import dataclasses

import numpy as np
import pytest

import oracle
import oracle.moe_oracle as OM
from sigmoid_top_routing_b200 import inputs as G

torch = pytest.importorskip("torch")

# e2m1 codes 0..15 by hand: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; bit 3 = sign
E2M1_BY_HAND = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def test_e2m1_table_by_hand():
    v = oracle.e2m1_value(np.arange(16))
    assert np.array_equal(v, np.array(E2M1_BY_HAND))
    assert np.signbit(v[8])                       # -0.0 keeps its sign


def test_e4m3_all_bytes_against_torch():
    b = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(b.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_value(b)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2        # 0x7F and 0xFF
    assert np.array_equal(got[~nan], ref[~nan])


@pytest.mark.parametrize("byte,value", [(0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6),
                                        (0x38, 1.0), (0x3C, 1.5), (0x40, 2.0), (0x7E, 448.0), (0xB8, -1.0),
                                        (0x30, 0.5), (0x56, 14.0)])
def test_e4m3_bytes_by_hand(byte, value):
    assert oracle.e4m3_value(np.array([byte]))[0] == value


def _hand_row():
    """K = 32: block 0 scale 0x38 (1.0), block 1 scale 0x40 (2.0); global 0.25.
    Byte j holds k = 2j (low nibble) and k = 2j + 1 (high nibble)."""
    codes_k = [0x1, 0x2, 0x3, 0x4, 0x5, 0x6, 0x7, 0x9, 0xA, 0xB, 0xC, 0xD, 0xE, 0xF, 0x0, 0x8,
               0x7, 0x1, 0x2, 0xF, 0x0, 0x3, 0xC, 0x4, 0x5, 0x6, 0x9, 0xA, 0xB, 0xD, 0xE, 0x2]
    packed = np.array([[codes_k[2 * j] | (codes_k[2 * j + 1] << 4) for j in range(16)]], dtype=np.uint8)
    scales = np.array([[0x38, 0x40]], dtype=np.uint8)
    want = [E2M1_BY_HAND[c] * (1.0 if k < 16 else 2.0) * 0.25 for k, c in enumerate(codes_k)]
    return packed, scales, 0.25, np.array([want])


def test_dequant_row_by_hand():
    packed, scales, g, want = _hand_row()
    assert np.array_equal(oracle.dequant_nvfp4(packed, scales, g), want)


def test_dequant_closed_form_global_scale():
    """Every code 1.0 (0x2), every block scale 1.0 (0x38): w == g."""
    g = np.float32(3.0517578125e-05)
    packed = np.full((3, 64), 0x22, dtype=np.uint8)
    scales = np.full((3, 8), 0x38, dtype=np.uint8)
    assert np.all(oracle.dequant_nvfp4(packed, scales, g) == float(g))


def test_encoder_round_trip_on_representable_weights():
    """Weights that are exactly e2m1 * e4m3 * g with each block's largest
    magnitude 6 * scale come back bit for bit (the encoder picks those codes)."""
    rng = np.random.default_rng(4)
    g = np.float32(2.0 ** -12)
    N, K = 4, 64
    block_scale = np.array([0.5, 1.0, 1.5, 2.0, 28.0, 0.125, 3.0, 1.0])[: K // 16]
    mags = np.array(E2M1_BY_HAND[:8])
    w = np.empty((N, K))
    for n in range(N):
        for b in range(K // 16):
            v = rng.choice(mags, 16) * rng.choice([-1, 1], 16)
            v[rng.integers(16)] = 6.0                      # the block's max is 6 * scale
            w[n, 16 * b: 16 * b + 16] = v * block_scale[b] * float(g)
    g_in = np.float32(np.abs(w).max() / (6 * 448))
    packed, scales, g_out = G.quantize_nvfp4(w.astype(np.float32))
    assert g_out == g_in
    back = oracle.dequant_nvfp4(packed, scales, g_out)
    np.testing.assert_allclose(back, w, rtol=0.07)           # block scales re-rounded to e4m3 under g_out
    rel = np.linalg.norm(back - w) / np.linalg.norm(w)
    assert rel < 0.05


def test_quantized_gaussian_error_is_4bit_sized():
    w = (np.random.default_rng(5).standard_normal((64, 256)) * 0.02).astype(np.float32)
    packed, scales, g = G.quantize_nvfp4(w)
    rel = np.linalg.norm(oracle.dequant_nvfp4(packed, scales, g) - w) / np.linalg.norm(w)
    assert 0.03 < rel < 0.15


def test_nvfp4_block_matches_brute_force_over_all_experts():
    wl = dataclasses.replace(G.WORKLOADS["tiny"], fmt="nvfp4", name="tiny_nvfp4")
    inp = G.make_inputs(wl)
    r = oracle.moe_block(inp)
    acc, _ = oracle.moe_block_all_experts(inp)
    np.testing.assert_allclose(r["acc"], acc, rtol=1e-12, atol=1e-15)
    assert np.abs(r["acc"]).max() > 1e-3


# --------------------------------------------------------------------- mutants

def test_mutant_scale_per_32_goes_red(monkeypatch):
    def bad(codes, scales, global_scale):
        p = np.asarray(codes, dtype=np.uint8)
        q = np.stack([p & 0xF, p >> 4], axis=-1).reshape(*p.shape[:-1], p.shape[-1] * 2)
        s = np.repeat(OM.e4m3_value(scales), 32, axis=-1)[..., : q.shape[-1]]
        return OM.e2m1_value(q) * s * float(global_scale)
    monkeypatch.setattr(oracle, "dequant_nvfp4", bad)
    with pytest.raises(AssertionError):
        test_dequant_row_by_hand()


def test_mutant_global_dropped_goes_red(monkeypatch):
    real = OM.dequant_nvfp4
    monkeypatch.setattr(oracle, "dequant_nvfp4", lambda c, s, g: real(c, s, 1.0))
    with pytest.raises(AssertionError):
        test_dequant_closed_form_global_scale()


def test_mutant_nibbles_swapped_goes_red(monkeypatch):
    real = OM.dequant_nvfp4

    def bad(codes, scales, global_scale):
        p = np.asarray(codes, dtype=np.uint8)
        return real(((p & 0xF) << 4) | (p >> 4), scales, global_scale)
    monkeypatch.setattr(oracle, "dequant_nvfp4", bad)
    with pytest.raises(AssertionError):
        test_dequant_row_by_hand()
