"""Pins for oracle.nvfp4: block scale, codes, per-tensor scale, round trip, nibble order.

The expectations are worked by hand from the format definitions (E2M1 grid
{0, .5, 1, 1.5, 2, 3, 4, 6}, ties to the even code; E4M3 grid with ties to the
even mantissa), or are exact round trips of representable blocks.
"""

import numpy as np
import pytest

from oracle import nvfp4
from oracle.formats import E4M3_TABLE


def test_global_scale_is_smallest_power_of_two_covering_amax():
    assert nvfp4.global_scale(2688.0) == 1.0
    assert nvfp4.global_scale(2688.0001) == 2.0
    assert nvfp4.global_scale(1.0) == 2.0 ** -11        # 2^-11*2688 = 1.3125 >= 1 > 0.656
    assert nvfp4.global_scale(0.0) == 1.0
    rng = np.random.default_rng(0)
    for a in np.exp2(rng.uniform(-30, 30, 2000)):
        g = nvfp4.global_scale(a)
        assert np.log2(g) == int(np.log2(g))
        assert g * 2688 >= a > (g / 2) * 2688


def test_block_by_hand_scale_one():
    # amax 6 with g = 1 -> S = 1.0 (0x38); every value below is its own quotient
    x = np.array([[6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -0.25, -0.75, 0.1, -0.1, 6.0, 0.0, -0.0, 5.5]])
    codes, scales = nvfp4.quantize(x, 1.0)
    assert scales.tolist() == [[0x38]]
    assert codes.tolist() == [[7, 0, 2, 2, 4, 4, 6, 6, 8, 10, 0, 8, 7, 0, 8, 7]]


def test_block_by_hand_scaled():
    # g = 2^-3, S = 1.25 (0x3A): x = m * 1.25 / 8 for grid values m
    g = 2.0 ** -3
    m = np.array([6, 4, 3, 2, 1.5, 1, 0.5, 0, -6, -4, -3, -2, -1.5, -1, -0.5, 1.25])
    x = (m * 1.25 * g)[None, :]
    codes, scales = nvfp4.quantize(x, g)
    assert scales.tolist() == [[0x3A]]
    # last element sits on the 1.0|1.5 midpoint -> even code 2 (value 1.0)
    assert codes.tolist() == [[7, 6, 5, 4, 3, 2, 1, 0, 15, 14, 13, 12, 11, 10, 9, 2]]


def test_block_scale_ties_round_to_even_mantissa():
    # amax/6 = 1.0625 is halfway between 1.0 (0x38) and 1.125 (0x39): even -> 0x38
    x = np.zeros((1, 16)); x[0, 3] = 6.375
    codes, scales = nvfp4.quantize(x, 1.0)
    assert scales[0, 0] == 0x38 and codes[0, 3] == 7          # 6.375 clamps to 6
    # amax/6 = 1.1875 is halfway between 1.125 (0x39) and 1.25 (0x3A): even -> 0x3A
    x = np.zeros((1, 16)); x[0, 0] = -7.125
    codes, scales = nvfp4.quantize(x, 1.0)
    assert scales[0, 0] == 0x3A and codes[0, 0] == 15         # -7.125/1.25 = -5.7 -> -6


def test_zero_and_tiny_blocks_have_zero_scale_and_codes():
    x = np.zeros((2, 32)); x[1, 16:] = -1e-9
    codes, scales = nvfp4.quantize(x, 1.0)
    assert np.all(scales == 0) and np.all(codes == 0)          # S == 0 -> codes 0x0, no sign


def test_saturating_and_subnormal_scales():
    x = np.zeros((1, 32)); x[0, 0] = 6 * 1000.0; x[0, 16] = 6 * 2.0 ** -9
    codes, scales = nvfp4.quantize(x, 1.0)
    assert scales.tolist() == [[0x7E, 0x01]]
    assert codes[0, 0] == 7 and codes[0, 16] == 7


def _representable(rng, rows, K, g):
    """Random codes and scales whose blocks each hold a +-6 element, and their values."""
    codes = rng.integers(0, 16, size=(rows, K)).astype(np.uint8)
    nb = K // 16
    for r in range(rows):
        for b in range(nb):
            codes[r, b * 16 + rng.integers(0, 16)] = 7 if rng.random() < 0.5 else 15
    scales = rng.integers(1, 0x7F, size=(rows, nb)).astype(np.uint8)
    return codes, scales, nvfp4.dequantize(codes, scales, g)


@pytest.mark.parametrize("g", [1.0, 2.0 ** -7, 2.0 ** 5])
def test_round_trip_of_representable_blocks(g):
    rng = np.random.default_rng(3)
    codes, scales, x = _representable(rng, 37, 128, g)
    c2, s2 = nvfp4.quantize(x, g)
    assert np.array_equal(s2, scales)
    assert np.array_equal(c2, codes)
    assert np.array_equal(nvfp4.dequantize(c2, s2, g), x)


def test_dequantize_value_formula():
    codes = np.array([[7] + [0] * 15])
    assert nvfp4.dequantize(codes, np.array([[0x3A]]), 0.5)[0, 0] == 6 * 1.25 * 0.5


def test_nibble_order_low_is_even_element():
    packed = nvfp4.pack_nibbles(np.array([[1, 2, 15, 8]], dtype=np.uint8))
    assert packed.tolist() == [[0x21, 0x8F]]
    assert nvfp4.unpack_nibbles(packed).tolist() == [[1, 2, 15, 8]]


def test_quantization_error_bound():
    # |x - deq(Q(x))| <= half a grid step of the block, and <= S*g for values below the top
    rng = np.random.default_rng(4)
    x = rng.standard_normal((64, 256)) * np.exp2(rng.integers(-6, 6, size=(64, 1)))
    g = nvfp4.global_scale(np.abs(x).max())
    codes, scales = nvfp4.quantize(x, g)
    err = np.abs(nvfp4.dequantize(codes, scales, g) - x).reshape(64, 16, 16)
    Sg = (E4M3_TABLE[scales] * g)[:, :, None]
    amax = np.abs(x).reshape(64, 16, 16).max(axis=2, keepdims=True)
    # grid steps are <= 2 (between 4 and 6); the scale itself is rounded, so allow amax/6 slack
    assert np.all(err <= Sg * 1.0 + np.abs(amax / 6 - Sg) * 6 + 1e-12)
