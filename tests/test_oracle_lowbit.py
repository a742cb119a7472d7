"""Pins of the oracle's 4-bit weight functions (CPU only).

Format (tag page "RTX 3090", item on a custom engine for a 27B-class model:
4-bit weights, 16-bit activations; the page names no format, the reading is
the plain group-wise symmetric one): 64 weights per fp32 scale s = max|w|/7,
q = clamp(rint(w / s), -7, 7) stored as the nibble q + 8, weight k in byte
k / 2 with the even weight in the low nibble.

The expected bytes below are worked out by hand from that definition, so a
swapped nibble order, a wrong offset, a floor instead of round-to-nearest
(or ties away from zero instead of to even), a per-row instead of per-group
scale, or a sign error fails one of them.
"""
import numpy as np
import pytest

import oracle
from attention_decode_megakernel_b200 import synth


def _bits(vals, cols=64):
    row = np.zeros(cols, np.float32)
    row[: len(vals)] = vals
    return synth.f32_to_bf16_bits(row[None, :])


def test_hand_worked_group_codes_and_scale():
    # max |w| = 0.875 = 7/8, so s = 1/8 exactly and every value is a multiple
    W = _bits([0.875, -0.875, 0.25, -0.125, 0.0, 0.5])
    codes, scales = oracle.quantize_w4(W)
    assert scales.shape == (1, 1) and scales[0, 0] == np.float32(0.125)
    # q = 7, -7, 2, -1, 0, 4 -> nibbles 15, 1, 10, 7, 8, 12, low nibble first
    assert codes[0, :3].tolist() == [0x1F, 0x7A, 0xC8]
    assert all(b == 0x88 for b in codes[0, 3:])  # the zeros: q = 0 -> 8 | 8 << 4
    Wd = oracle.dequantize_w4(codes, scales)
    assert Wd[0, :6].tolist() == [0.875, -0.875, 0.25, -0.125, 0.0, 0.5]


def test_ties_round_half_to_even():
    # s = 1/8: ratios 0.5, 1.5, 2.5, -0.5, 3.5 -> 0, 2, 2, -0, 4
    W = _bits([0.875, 0.0625, 0.1875, 0.3125, -0.0625, 0.4375])
    codes, _ = oracle.quantize_w4(W)
    nib = [(codes[0, k // 2] >> (4 * (k % 2))) & 0xF for k in range(6)]
    assert nib == [15, 8, 10, 10, 8, 12]


def test_all_zero_group_has_zero_scale():
    W = np.zeros((2, 128), np.uint16)
    codes, scales = oracle.quantize_w4(W)
    assert (scales == 0).all() and (codes == 0x88).all()
    assert (oracle.dequantize_w4(codes, scales) == 0).all()


def test_scale_is_per_group_of_64():
    # group 0 max 0.875 (s = 1/8), group 1 max 14 (s = 2)
    row = np.zeros(128, np.float32)
    row[0] = 0.875
    row[64], row[65] = 14.0, -4.0
    codes, scales = oracle.quantize_w4(synth.f32_to_bf16_bits(row[None, :]))
    assert scales[0].tolist() == [0.125, 2.0]
    assert codes[0, 32] == (15 | (6 << 4))  # 14 / 2 = 7 -> 15; -4 / 2 = -2 -> 6
    Wd = oracle.dequantize_w4(codes, scales)
    assert Wd[0, 64] == 14.0 and Wd[0, 65] == -4.0 and Wd[0, 0] == 0.875


def test_round_trip_error_is_at_most_half_a_step():
    rng = np.random.default_rng(5)
    W = synth.f32_to_bf16_bits(rng.standard_normal((16, 256), dtype=np.float32) * 0.02)
    codes, scales = oracle.quantize_w4(W)
    w = synth.bf16_bits_to_f32(W).astype(np.float64)
    s = np.repeat(scales.astype(np.float64), 64, axis=1)
    err = np.abs(w - oracle.dequantize_w4(codes, scales))
    assert (err <= s / 2 * (1 + 1e-6)).all()
    assert (err > 0.4 * s).any()          # rounding, not truncation to a step
    # the group maximum is represented exactly (q = +-7)
    for r in range(16):
        for g in range(4):
            blk = w[r, 64 * g:64 * (g + 1)]
            k = int(np.argmax(np.abs(blk)))
            assert abs(oracle.dequantize_w4(codes, scales)[r, 64 * g + k] - blk[k]) <= \
                1e-6 * abs(blk[k])


def test_gemv_w4_equals_dequantised_matrix_product():
    rng = np.random.default_rng(6)
    W = synth.f32_to_bf16_bits(rng.standard_normal((33, 320), dtype=np.float32))
    codes, scales = oracle.quantize_w4(W)
    x = rng.standard_normal(320)
    want = oracle.dequantize_w4(codes, scales) @ x
    np.testing.assert_allclose(oracle.gemv_w4(codes, scales, x), want, rtol=1e-12, atol=1e-12)


def test_exactly_representable_weights_match_the_bf16_gemv():
    # w = q * s with s a power of two: quantisation loses nothing
    rng = np.random.default_rng(7)
    q = rng.integers(-7, 8, size=(9, 192))
    q[:, ::64] = 7                         # every group reaches max |q| = 7
    w = (q * 0.25).astype(np.float32)
    W = synth.f32_to_bf16_bits(w)
    codes, scales = oracle.quantize_w4(W)
    assert (scales == 0.25).all()
    assert (oracle.dequantize_w4(codes, scales) == w).all()
    x = rng.standard_normal(192)
    np.testing.assert_allclose(oracle.gemv_w4(codes, scales, x), oracle.gemv(W, x),
                               rtol=1e-12, atol=1e-12)


def test_columns_not_a_multiple_of_64_are_rejected():
    with pytest.raises(ValueError):
        oracle.quantize_w4(np.zeros((1, 96), np.uint16))
