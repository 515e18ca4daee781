"""E2M1 and E4M3 value tables and exact round-to-nearest-even quantizers (float64).

Test infrastructure (see the package docstring): only tests and the CPU
baseline may import this.

The pages ("Nunchaku Lite", section "Supported quantization types") name the
NVFP4 format (group size 16) without defining its element or scale types.  The
definitions used here are the public ones:

* E2M1 (OCP microscaling): 1 sign bit, 2 exponent bits (bias 1), 1 mantissa
  bit.  Exponent field 0 is subnormal: 0.m * 2^0.  Magnitudes of codes 0..7 are
  0, 0.5, 1, 1.5, 2, 3, 4, 6.  Bit 3 is the sign.
* E4M3 "FN" (OCP FP8): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.
  Exponent field 0 is subnormal: 0.mmm * 2^-6.  No infinities; S.1111.111 is
  NaN.  Largest finite value 1.75 * 2^8 = 448.

Quantizers return the code whose value is nearest; a value exactly halfway
between two neighbours takes the neighbour whose code is even (whose mantissa
LSB is 0), which is round-to-nearest-even on these grids.
"""

import numpy as np

E2M1_MAX = 6.0
E4M3_MAX = 448.0


def e2m1_value_of_code(code):
    """Value of a 4-bit E2M1 code, from its bit fields."""
    code = int(code) & 0xF
    sign = -1.0 if (code >> 3) & 1 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        mag = (m / 2.0) * 2.0 ** 0           # subnormal: 0.m * 2^(1 - bias), bias 1
    else:
        mag = (1.0 + m / 2.0) * 2.0 ** (e - 1)
    return sign * mag


def e4m3_value_of_code(code):
    """Value of an 8-bit E4M3 (FN) code, from its bit fields; NaN codes give nan."""
    code = int(code) & 0xFF
    sign = -1.0 if (code >> 7) & 1 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        mag = (m / 8.0) * 2.0 ** (1 - 7)      # subnormal
    else:
        mag = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return sign * mag


# Full tables indexed by code.
E2M1_TABLE = np.array([e2m1_value_of_code(c) for c in range(16)], dtype=np.float64)
E4M3_TABLE = np.array([e4m3_value_of_code(c) for c in range(256)], dtype=np.float64)

# Non-negative grids (codes 0..7 for E2M1, 0..126 for E4M3), ascending in value.
_E2M1_POS = E2M1_TABLE[:8].copy()
_E4M3_POS = E4M3_TABLE[:127].copy()


def _nearest_even_code(mag, grid):
    """Index of the grid value nearest to each mag (mag >= 0, grid ascending).

    Ties go to the even index.  Values above the top of the grid map to the top
    (saturation).
    """
    mag = np.asarray(mag, dtype=np.float64)
    hi = np.searchsorted(grid, mag, side="left")          # first grid value >= mag
    hi = np.clip(hi, 0, len(grid) - 1)
    lo = np.clip(hi - 1, 0, len(grid) - 1)
    d_lo = mag - grid[lo]
    d_hi = grid[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(mag >= grid[-1], len(grid) - 1, idx)    # saturate
    return idx.astype(np.int64)


def quantize_e4m3(v):
    """E4M3 code of each non-negative v: RNE onto the finite grid, saturating at 448.

    Used for block scales, which are never negative.  Values in (448, inf)
    become 448 (code 0x7E), matching saturating ("satfinite") conversion.
    """
    v = np.asarray(v, dtype=np.float64)
    if np.any(v < 0) or np.any(np.isnan(v)):
        raise ValueError("quantize_e4m3 takes non-negative, non-NaN values")
    return _nearest_even_code(v, _E4M3_POS).astype(np.uint8)


def quantize_e2m1(v):
    """E2M1 code of each v: clamp |v| to 6, RNE onto the grid, keep the sign bit.

    The sign bit follows IEEE sign (np.signbit), so a negative value that rounds
    to zero gives code 0x8 (negative zero).
    """
    v = np.asarray(v, dtype=np.float64)
    mag = np.minimum(np.abs(v), E2M1_MAX)
    code = _nearest_even_code(mag, _E2M1_POS)
    code = code | np.where(np.signbit(v), 8, 0)
    return code.astype(np.uint8)


def bf16_round(x):
    """Round float64 values to the nearest bfloat16 (ties to even), once, as float64.

    bfloat16 has 8 significant bits and the exponent range of float32 (normal down to 2^-126,
    subnormal steps of 2^-133).  The rounding is done straight from the float64 value: going
    through float32 first would round twice, and a value just beside a bf16 midpoint that
    float32 rounds onto the midpoint would then tip by ties-to-even.  Values beyond the largest
    bf16 round to 2^128 (infinity when stored); zeros keep their sign; NaN stays NaN.
    """
    v = np.asarray(x, dtype=np.float64)
    with np.errstate(invalid="ignore", over="ignore"):
        _, e = np.frexp(v)                              # |v| in [2^(e-1), 2^e)
        shift = np.maximum(e - 8, -133)                 # weight of the last kept bit
        out = np.ldexp(np.rint(np.ldexp(v, -shift)), shift)   # rint: to nearest, ties to even
    return np.where((v == 0.0) | ~np.isfinite(v), v, out)
