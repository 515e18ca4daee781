"""AWQ-style W4A16 weight-only linear layer (int4, group 64 along K), float64.

Test infrastructure (see the package docstring).

Source: "Nunchaku Lite" (Diffusers docs), section "Supported quantization
types": awq_w4a16 / int4 / group 64, an AWQ-style INT4 weight-only kernel; the
article "Memangkas VRAM Model Diffusi ... Lewat Nunchaku Lite" says it serves
the adaptive-normalisation layers with 16-bit activations.  The pages do not
fix the zero-point convention; the reading here is an integer zero point z per
(output row, group) stored as a bfloat16 value, with

    W_deq[n, k] = (q[n, k] - z[n, k // 64]) * s[n, k // 64]
    y           = X @ W_deq^T (+ b)
"""

import numpy as np

GROUP = 64


def dequantize(q, scales, zeros):
    """q int [N, K] (0..15), scales/zeros [N, K/64] -> float64 [N, K]."""
    q = np.asarray(q, dtype=np.float64)
    N, K = q.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 64")
    s = np.repeat(np.asarray(scales, dtype=np.float64), GROUP, axis=1)
    z = np.repeat(np.asarray(zeros, dtype=np.float64), GROUP, axis=1)
    return (q - z) * s


def forward(X, q, scales, zeros, bias=None):
    """y [M, N] = X @ ((q - z) s)^T (+ b), float64."""
    y = np.asarray(X, dtype=np.float64) @ dequantize(q, scales, zeros).T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y


def unpack_qweight(packed):
    """[N, K/2] bytes (element 2i in the low nibble) -> int [N, K]."""
    packed = np.asarray(packed, dtype=np.uint8)
    N, half = packed.shape
    out = np.empty((N, 2 * half), dtype=np.int64)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out
