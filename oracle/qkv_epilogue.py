"""The QKV projection's epilogue: per-head RMSNorm of q and k, then rotary position
embedding (RoPE) of q and k, v unchanged -- in float64.

Test infrastructure (see the package docstring).

Method: "Nunchaku Lite" docs, section on fused kernels -- the original engine fuses the
Q, K, V projections with RMSNorm and RoPE (its benchmark table gives the grouped
QKV + norm + RoPE fusion 1.27x and the RMSNorm + RoPE epilogue fusion 1.236x).  The pages
name the operations only; the readings used here (each stated where it applies):

* qkv [M, 3 H D] holds q, k, v side by side, each [M, H, D] head-major (head h at columns
  h D .. h D + D - 1 of its third);
* RMSNorm over each head's D values: x / sqrt(mean(x^2) + eps) * w, with a learned weight
  w [D] per q and per k (shared by the heads) and eps given (the caller's model decides it);
* RoPE rotates consecutive pairs (x[2i], x[2i+1]) of each head by a per-token angle:
  (x0 cos - x1 sin, x0 sin + x1 cos); the angles come in as cos / sin tables [M, D/2]
  (a model's position scheme -- 1-D, or several axes as in image transformers -- only
  changes the tables, so they are an input, not a choice made here).
"""

import numpy as np


def rmsnorm_heads(x, weight, eps):
    """x [M, H, D], weight [D]: each head vector divided by its root mean square (plus eps
    under the root) and scaled by the weight."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(weight, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + float(eps)) * w


def rope(x, cos, sin):
    """x [M, H, D] with D even; cos, sin [M, D/2]: pair i of every head of token m rotated
    by the angle whose cosine and sine are cos[m, i], sin[m, i]."""
    x = np.asarray(x, dtype=np.float64)
    c = np.asarray(cos, dtype=np.float64)[:, None, :]
    s = np.asarray(sin, dtype=np.float64)[:, None, :]
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


def rope_tables(angles):
    """cos and sin tables [M, D/2] of per-token, per-pair angles (radians)."""
    a = np.asarray(angles, dtype=np.float64)
    return np.cos(a), np.sin(a)


def qkv_epilogue(qkv, heads, q_weight, k_weight, eps, cos, sin):
    """qkv [M, 3 H D] -> (q, k, v), each [M, H, D]: q and k RMS-normalised per head and
    rotated, v as it came."""
    qkv = np.asarray(qkv, dtype=np.float64)
    M, width = qkv.shape
    if width % (3 * heads):
        raise ValueError("width is not 3 * heads * head_dim")
    D = width // (3 * heads)
    if D % 2:
        raise ValueError("head_dim must be even")
    q, k, v = (qkv[:, j * heads * D:(j + 1) * heads * D].reshape(M, heads, D) for j in range(3))
    q = rope(rmsnorm_heads(q, q_weight, eps), cos, sin)
    k = rope(rmsnorm_heads(k, k_weight, eps), cos, sin)
    return q, k, v
