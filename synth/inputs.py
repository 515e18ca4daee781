"""Seeded synthetic inputs for the SVDQ W4A4 and AWQ W4A16 linear layers.

Recipe (one ``numpy.random.default_rng(seed)`` stream per workload, drawn in
this order):

SVDQ W4A4 (shapes X [M, K], W [N, K]):
  1. outlier input channels ``idx = rng.choice(K, 8, replace=False)``
  2. ``X = rng.standard_normal((M, K))`` (or GELU(Z), Z ~ N(0,1), for the
     heavy-right-tail MLP-down input), then ``X[:, idx] *= 20``
  3. ``W = 0.02 * rng.standard_normal((N, K))``, then ``W[:, idx] *= 10``
  4. ``b = 0.01 * rng.standard_normal(N)``
  Every drawn tensor is rounded to bfloat16.  Offline preparation, as an
  exporter would do it (float64):
  lambda_j = max_m |X[m, j]|^0.5 / max_n |W[n, j]|^0.5,
  smooth_inv = bf16(1 / lambda), lambda_eff = 1 / smooth_inv,
  W_hat = W * lambda_eff (per input channel), rank-32 factors of W_hat^T with
  the singular values split as sqrt on each side, L1 [K, 32] and L2 [32, N]
  rounded to bfloat16, residual R = W_hat - (L1 L2)^T kept as float32.
  The static activation scale g_a is the power of two
  2^ceil(log2(amax(X * smooth_inv) / 2688)) of the same data.

AWQ W4A16 (X [M, K] ~ N(0, 1), W [N, K] ~ N(0, 0.02)): per output row and
group of 64 along K, s = bf16((max - min) / 15) (1 when max == min),
z = clamp(rint(-min / s), 0, 15), q = clamp(rint(w / s) + z, 0, 15); q packed
two per byte with element 2i in the low nibble.

The rank-32 factors come from a randomized range finder (seeded, four power
iterations) followed by an exact SVD of the projected matrix.  Only the
product L1 L2 and the residual R enter the layer, and R is defined from the
rounded factors, so the factorisation method changes the split between the
branches, never the identity W_hat = R + (L1 L2)^T.
"""

from dataclasses import dataclass
import math

import numpy as np
import torch

RANK = 32
N_OUTLIERS = 8


# ---------------------------------------------------------------- bf16 helpers

def to_bf16(x):
    """Round to bfloat16 (nearest, ties to even); returns float32 values that are exactly bf16."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.to(torch.float32).numpy()


def bf16_bits(x):
    """uint16 bit patterns of float32 values that are exactly representable in bf16."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("values are not bf16-representable")
    return (u >> 16).astype(np.uint16)


def bf16_from_bits(bits):
    """float32 values of uint16 bf16 bit patterns."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def _pow2_calibration_scale(amax):
    """Power of two g with g * 2688 >= amax, the smallest such (1 when amax == 0)."""
    if amax == 0.0:
        return 1.0
    e = math.ceil(math.log2(amax / 2688.0))
    g = math.ldexp(1.0, e)
    while g * 2688.0 < amax:
        g *= 2.0
    while (g / 2.0) * 2688.0 >= amax:
        g /= 2.0
    return g


# ---------------------------------------------------------------- SVDQ W4A4

@dataclass
class SvdqWorkload:
    M: int
    K: int
    N: int
    X: np.ndarray            # float32 [M, K], bf16 values
    smooth_inv: np.ndarray   # float32 [K], bf16 values
    L1: np.ndarray           # float32 [K, r], bf16 values
    L2: np.ndarray           # float32 [r, N], bf16 values
    R: np.ndarray            # float32 [N, K]
    bias: np.ndarray         # float32 [N], bf16 values
    g_a: float               # power of two
    W: np.ndarray            # float32 [N, K], bf16 values (the unquantized weight)
    outliers: np.ndarray     # int [8]


def _topr_factors(A, r, seed):
    """Rank-r factors of A [K, N] (float64): A ~ F1 @ F2, F1 [K, r], F2 [r, N]."""
    rng = np.random.default_rng(seed)
    K, N = A.shape
    p = min(r + 16, min(K, N))
    omega = rng.standard_normal((N, p))
    Q, _ = np.linalg.qr(A @ omega)
    for _ in range(4):
        Q, _ = np.linalg.qr(A.T @ Q)
        Q, _ = np.linalg.qr(A @ Q)
    B = Q.T @ A                                    # [p, N]
    Ub, s, Vt = np.linalg.svd(B, full_matrices=False)
    U = Q @ Ub[:, :r]
    root = np.sqrt(s[:r])
    return U * root[None, :], root[:, None] * Vt[:r]


def svdq_workload(M, K, N, seed=0, gelu_input=False, rank=RANK, with_bias=True):
    rng = np.random.default_rng(seed)
    idx = rng.choice(K, N_OUTLIERS, replace=False) if K >= N_OUTLIERS else np.arange(K)
    Z = rng.standard_normal((M, K))
    if gelu_input:
        Z = torch.nn.functional.gelu(torch.from_numpy(Z), approximate="none").numpy()
    Z[:, idx] *= 20.0
    X = to_bf16(Z)
    W = 0.02 * rng.standard_normal((N, K))
    W[:, idx] *= 10.0
    W = to_bf16(W)
    b = to_bf16(0.01 * rng.standard_normal(N)) if with_bias else np.zeros(N, np.float32)

    xmax = np.max(np.abs(X.astype(np.float64)), axis=0) if M > 0 else np.ones(K)
    wmax = np.max(np.abs(W.astype(np.float64)), axis=0)
    xmax = np.where(xmax == 0.0, 1.0, xmax)
    wmax = np.where(wmax == 0.0, 1.0, wmax)
    lam = np.sqrt(xmax) / np.sqrt(wmax)
    smooth_inv = to_bf16(1.0 / lam)
    lam_eff = 1.0 / smooth_inv.astype(np.float64)

    W_hat = W.astype(np.float64) * lam_eff[None, :]        # [N, K]
    F1, F2 = _topr_factors(W_hat.T, rank, seed + 1)         # W_hat^T ~ F1 F2
    L1 = to_bf16(F1)                                        # [K, r]
    L2 = to_bf16(F2)                                        # [r, N]
    R = (W_hat - (L1.astype(np.float64) @ L2.astype(np.float64)).T).astype(np.float32)

    x_hat_amax = float(np.max(np.abs(X.astype(np.float64) * smooth_inv.astype(np.float64)))) if M > 0 else 0.0
    g_a = _pow2_calibration_scale(x_hat_amax)
    return SvdqWorkload(M, K, N, X, smooth_inv, L1, L2, R, b, g_a, W, idx)


# ---------------------------------------------------------------- AWQ W4A16

AWQ_GROUP = 64


@dataclass
class AwqWorkload:
    M: int
    K: int
    N: int
    X: np.ndarray        # float32 [M, K], bf16 values
    q: np.ndarray        # uint8 [N, K], one code 0..15 per element
    qweight: np.ndarray  # uint8 [N, K/2], element 2i in the low nibble
    scales: np.ndarray   # float32 [N, K/64], bf16 values
    zeros: np.ndarray    # float32 [N, K/64], integer values 0..15 (bf16-exact)
    W: np.ndarray        # float32 [N, K], the unquantized weight (bf16 values)


def awq_workload(M, K, N, seed=0):
    rng = np.random.default_rng(seed)
    X = to_bf16(rng.standard_normal((M, K)))
    W = to_bf16(0.02 * rng.standard_normal((N, K)))
    G = W.astype(np.float64).reshape(N, K // AWQ_GROUP, AWQ_GROUP)
    mn = G.min(axis=2)
    mx = G.max(axis=2)
    s = to_bf16(np.where(mx > mn, (mx - mn) / 15.0, 1.0)).astype(np.float64)
    z = np.clip(np.rint(-mn / s), 0, 15)
    q = np.clip(np.rint(G / s[:, :, None]) + z[:, :, None], 0, 15).astype(np.uint8).reshape(N, K)
    qweight = (q[:, 0::2] & 0xF) | ((q[:, 1::2] & 0xF) << 4)
    return AwqWorkload(M, K, N, X, q, qweight.astype(np.uint8),
                       s.astype(np.float32), z.astype(np.float32), W)
