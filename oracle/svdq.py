"""SVDQuant W4A4 NVFP4 linear layer, dequantize-then-matmul in float64.

Test infrastructure (see the package docstring).

What the layer computes (the article "Memangkas VRAM Model Diffusi ... Lewat
Nunchaku Lite", section on what happens when a diffusion model is quantized:
outliers are moved into a 16-bit low-rank branch, the rest runs as 4-bit
weights times 4-bit activations; "Nunchaku Lite" docs, "Supported quantization
types": svdq_w4a4 / nvfp4 / group 16; "NunchakuLiteQuantizationConfig": rank 32):

    X_hat = X * smooth_inv                      (per input channel, 1/lambda)
    y     = deq(Q(X_hat)) @ deq(Q(R))^T + (X_hat @ L1) @ L2 + b

with R [N, K] the residual weight, L1 [K, r], L2 [r, N] the bfloat16 low-rank
factors, b [N] the bias, and Q the NVFP4 quantizer of ``oracle.nvfp4``.  The
activation per-tensor scale g_a is supplied by the caller (static calibration,
a power of two), or in the dynamic variant taken from the batch's own amax of X_hat
(``dynamic_act_scale``); the weight per-tensor scale g_w comes from amax(R).  The
low-rank intermediate X_hat @ L1 is kept in float64 (not rounded).
"""

import numpy as np

from . import nvfp4


def smooth(X, smooth_inv):
    """X_hat = X * smooth_inv, column-wise; exact in float64 for bfloat16 inputs."""
    X = np.asarray(X, dtype=np.float64)
    s = np.asarray(smooth_inv, dtype=np.float64)
    return X * s[None, :]


def quantize_activations(X, smooth_inv, g_a):
    """NVFP4 codes [M, K] and E4M3 scales [M, K/16] of X_hat with per-tensor scale g_a."""
    return nvfp4.quantize(smooth(X, smooth_inv), g_a)


def dynamic_act_scale(X, smooth_inv):
    """The dynamic variant's activation per-tensor scale: the per-tensor scale rule
    (``nvfp4.global_scale``) applied to the batch's own amax of X_hat instead of a calibrated
    one ("Nunchaku Lite" docs, "Supported quantization types": a per-tensor scale with the
    per-16 block scales)."""
    Xh = smooth(X, smooth_inv)
    return nvfp4.global_scale(np.max(np.abs(Xh)) if Xh.size else 0.0)


def quantize_weights(R):
    """NVFP4 codes [N, K], E4M3 scales [N, K/16] and the per-tensor scale g_w of R."""
    R = np.asarray(R, dtype=np.float64)
    g_w = nvfp4.global_scale(np.max(np.abs(R)) if R.size else 0.0)
    codes, scales = nvfp4.quantize(R, g_w)
    return codes, scales, g_w


def lowrank_down(X, smooth_inv, L1):
    """U = X_hat @ L1, shape [M, r], float64."""
    return smooth(X, smooth_inv) @ np.asarray(L1, dtype=np.float64)


def forward(X, smooth_inv, R, L1, L2, bias, g_a):
    """y [M, N] in float64.  bias may be None."""
    cx, sx = quantize_activations(X, smooth_inv, g_a)
    cw, sw, g_w = quantize_weights(R)
    xq = nvfp4.dequantize(cx, sx, g_a)                 # [M, K]
    wq = nvfp4.dequantize(cw, sw, g_w)                 # [N, K]
    y = xq @ wq.T
    y = y + lowrank_down(X, smooth_inv, L1) @ np.asarray(L2, dtype=np.float64)
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y
