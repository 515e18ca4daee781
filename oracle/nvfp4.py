"""NVFP4 block quantization (E2M1 codes, one E4M3 scale per 16 K elements, power-of-two
per-tensor scale), exact in float64.

Test infrastructure (see the package docstring).

Source: "Nunchaku Lite" (Diffusers docs), section "Supported quantization types":
svdq_w4a4 with nvfp4 precision uses group size 16.  The pages give no formula;
the steps below are the plain reading of an NVFP4 tensor (E2M1 values, an E4M3
scale per 16 contiguous K elements, an FP32 per-tensor scale), with these
readings fixed once:

1. The per-tensor scale g is a power of two: g = 2^ceil(log2(amax / (6 * 448))),
   or 1 when amax == 0.  It uses the top of the E4M3 range and keeps every later
   division by S*g exact.
2. Block scale S = RNE_E4M3(amax_block / (6 g)), saturating at 448.
3. Codes: if S == 0 every code of the block is 0x0; otherwise
   c = RNE_E2M1(clamp(x / (S g), -6, 6)) with the IEEE sign kept.
4. Dequantized value = E2M1(c) * E4M3(S) * g.

Why float64 arithmetic decides the same codes as exact arithmetic: inputs have
at most 24 significant bits (float32 residuals, or products of two bfloat16
values with 16 bits), S*g has at most 4, grid midpoints have at most 5 (E4M3)
or 3 (E2M1).  A quotient x/(S g) or amax/(6 g) that is not exactly a midpoint
therefore differs from it by a relative 2^-24 or more, far above float64's
2^-53 rounding, and one that is exactly a midpoint is computed exactly.
"""

import math

import numpy as np

from .formats import E2M1_TABLE, E4M3_TABLE, E4M3_MAX, E2M1_MAX, quantize_e2m1, quantize_e4m3

GROUP = 16


def global_scale(amax):
    """Smallest power of two g with g * 6 * 448 >= amax (1.0 when amax == 0)."""
    amax = float(amax)
    if not (amax >= 0.0) or math.isinf(amax):
        raise ValueError("amax must be finite and non-negative")
    if amax == 0.0:
        return 1.0
    limit = E2M1_MAX * E4M3_MAX                      # 2688
    m, e = math.frexp(amax / limit)                  # amax/limit = m * 2^e, m in [0.5, 1)
    g = math.ldexp(1.0, e)                           # candidate >= amax/limit
    while g * limit >= amax and (g / 2.0) * limit >= amax:
        g /= 2.0
    while g * limit < amax:
        g *= 2.0
    return g


def quantize(x, g):
    """Quantize rows of x (shape [rows, K], K % 16 == 0) with per-tensor scale g.

    Returns (codes uint8 [rows, K] holding one 4-bit code each,
             scales uint8 [rows, K/16] holding E4M3 codes).
    """
    x = np.asarray(x, dtype=np.float64)
    rows, K = x.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 16")
    blocks = x.reshape(rows, K // GROUP, GROUP)
    amax = np.max(np.abs(blocks), axis=2)
    scales = quantize_e4m3(amax / (6.0 * g))
    S = E4M3_TABLE[scales]                                        # [rows, K/16]
    denom = (S * g)[:, :, None]
    safe = np.where(denom == 0.0, 1.0, denom)
    v = np.clip(blocks / safe, -E2M1_MAX, E2M1_MAX)
    codes = quantize_e2m1(v)
    codes = np.where((S == 0.0)[:, :, None], np.uint8(0), codes)
    return codes.reshape(rows, K).astype(np.uint8), scales.astype(np.uint8)


def dequantize(codes, scales, g):
    """Values E2M1(c) * E4M3(S) * g for codes [rows, K] and scales [rows, K/16]."""
    codes = np.asarray(codes, dtype=np.int64)
    scales = np.asarray(scales, dtype=np.int64)
    rows, K = codes.shape
    vals = E2M1_TABLE[codes].reshape(rows, K // GROUP, GROUP)
    s = E4M3_TABLE[scales][:, :, None]
    return (vals * s * g).reshape(rows, K)


def pack_nibbles(codes):
    """Two codes per byte: element 2i in the low nibble, element 2i+1 in the high nibble."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)


def unpack_nibbles(packed):
    """Inverse of pack_nibbles: [rows, K/2] bytes -> [rows, K] codes."""
    packed = np.asarray(packed, dtype=np.uint8)
    rows, half = packed.shape
    out = np.empty((rows, half * 2), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out
