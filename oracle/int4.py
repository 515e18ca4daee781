"""SVDQuant W4A4 with INT4 precision and group size 64 (the second svdq_w4a4 row), in float64.

Test infrastructure (see the package docstring).

Source: "Nunchaku Lite" docs, section "Supported quantization types": the svdq_w4a4 method
with int4 precision and group size 64 -- the same SVDQ low-rank correction as the nvfp4 /
group-16 row (the docs add that on Blackwell nvfp4 is the faster of the two).  The pages give
no formula for it; the readings, fixed once:

1. Element codes are signed 4-bit integers, -8..7 (two's complement), two per byte, element 2i
   in the low nibble (as the nvfp4 codes).
2. One scale per 64 contiguous K elements of a row, in the model's 16-bit type (bfloat16):
   s = RNE_bf16(amax / 7), amax the group's largest magnitude, rounded once from the exact
   quotient.  A group with amax = 0 has s = 0 and all-zero codes.
3. Code c = clamp(RNE(x / s), -8, 7), ties to even (2.5 -> 2, -3.5 -> -4).  With an 8-bit
   scale rounded to nearest, |x / s| <= 7 (1 + 2^-8) < 7.5, so every code lies in -7..7 and
   the clamp never acts; it is kept as the statement of the code range.
4. Dequantized value c * s; no per-tensor scale (bf16 scales carry the range).

Layer (as the nvfp4 one, with the int4 quantizer Q):

    X_hat = X * smooth_inv
    y     = deq(Q(X_hat)) deq(Q(R))^T + (X_hat L1) L2 + b
          = sum_g s_x[m, g] s_w[n, g] sum_{k in g} c_x[m, k] c_w[n, k] + (X_hat L1) L2 + b.

Why float64 decides every rounding exactly: x has at most 24 significant bits (float32 R) or
16 (bf16 times bf16), s at most 8, and amax / 7 is rounded straight from float64 (not through
float32, whose rounding could land on a bf16 midpoint and tip a tie): a quotient that is
exactly a half-integer or a bf16 midpoint is computed exactly, and one that is not differs from
it by far more than float64's rounding error.
"""

import numpy as np

from .formats import bf16_round

GROUP = 64
CODE_MIN, CODE_MAX = -8, 7


def bf16_rne(v):
    """float64 values rounded to the nearest bfloat16 (ties to even), once, straight from
    float64 (formats.bf16_round)."""
    return bf16_round(v)


def quantize(x):
    """Codes int8 [rows, K] (-8..7) and scales float64 [rows, K/64] (bfloat16 values) of x."""
    x = np.asarray(x, dtype=np.float64)
    rows, K = x.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 64")
    g = x.reshape(rows, K // GROUP, GROUP)
    amax = np.max(np.abs(g), axis=2)
    s = bf16_rne(amax / 7.0)
    safe = np.where(s == 0.0, 1.0, s)[:, :, None]
    c = np.clip(np.rint(g / safe), CODE_MIN, CODE_MAX)
    c = np.where((s == 0.0)[:, :, None], 0.0, c)
    return c.reshape(rows, K).astype(np.int8), s


def dequantize(codes, scales):
    """Values c s for codes [rows, K] and scales [rows, K/64]."""
    c = np.asarray(codes, dtype=np.float64)
    rows, K = c.shape
    s = np.asarray(scales, dtype=np.float64)[:, :, None]
    return (c.reshape(rows, K // GROUP, GROUP) * s).reshape(rows, K)


def pack_nibbles(codes):
    """Two's-complement nibbles, two per byte: element 2i in the low nibble."""
    u = np.asarray(codes, dtype=np.int8).astype(np.uint8) & 0xF
    return (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed):
    """Inverse of pack_nibbles: [rows, K/2] bytes -> int8 codes [rows, K]."""
    p = np.asarray(packed, dtype=np.uint8)
    rows, half = p.shape
    u = np.empty((rows, 2 * half), dtype=np.uint8)
    u[:, 0::2] = p & 0xF
    u[:, 1::2] = p >> 4
    return np.where(u >= 8, u.astype(np.int16) - 16, u.astype(np.int16)).astype(np.int8)


def smooth(X, smooth_inv):
    """X_hat = X * smooth_inv, column-wise (exact in float64 for bf16 inputs)."""
    return np.asarray(X, dtype=np.float64) * np.asarray(smooth_inv, dtype=np.float64)[None, :]


def quantize_activations(X, smooth_inv):
    return quantize(smooth(X, smooth_inv))


def forward(X, smooth_inv, R, L1, L2, bias):
    """y [M, N] in float64 (bias may be None)."""
    cx, sx = quantize_activations(X, smooth_inv)
    cw, sw = quantize(R)
    y = dequantize(cx, sx) @ dequantize(cw, sw).T
    y = y + (smooth(X, smooth_inv) @ np.asarray(L1, dtype=np.float64)) @ np.asarray(L2, dtype=np.float64)
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y
