"""Pins for oracle.svdq: exact rational brute force on tiny shapes, the decomposition
identity for representable residuals, and special cases.
"""

from fractions import Fraction

import numpy as np
import pytest

from oracle import nvfp4, svdq
from oracle.formats import E2M1_TABLE, E4M3_TABLE
import synth


# ------------------------------------------------------------ brute force (exact rationals)

_E4M3_FINITE = [Fraction(float(v)) for v in E4M3_TABLE[:0x7F]]
_E2M1_MAG = [Fraction(float(v)) for v in E2M1_TABLE[:8]]


def _bf_pow2_scale(amax):
    if amax == 0:
        return Fraction(1)
    e = -200
    while Fraction(2) ** e * 2688 < amax:
        e += 1
    return Fraction(2) ** e


def _bf_nearest(target, grid):
    """index of the grid value nearest to target; ties to the even index."""
    best = None
    for i, v in enumerate(grid):
        d = abs(target - v)
        if best is None or d < best[0] or (d == best[0] and i % 2 == 0):
            best = (d, i)
    return best[1]


def _bf_quant_dequant(row, g):
    """Exact dequantized NVFP4 values of one row (list of Fractions)."""
    out = []
    for b in range(0, len(row), 16):
        blk = row[b:b + 16]
        amax = max(abs(v) for v in blk)
        S = _E4M3_FINITE[_bf_nearest(amax / (6 * g), _E4M3_FINITE)]
        for v in blk:
            if S == 0:
                out.append(Fraction(0))
                continue
            q = min(abs(v) / (S * g), Fraction(6))
            mag = _E2M1_MAG[_bf_nearest(q, _E2M1_MAG)]
            out.append((-mag if v < 0 else mag) * S * g)
    return out


def _bf_forward(X, s, R, L1, L2, b, g_a):
    M, K = X.shape
    N = R.shape[0]
    r = L1.shape[1]
    Xh = [[Fraction(float(X[m, k])) * Fraction(float(s[k])) for k in range(K)] for m in range(M)]
    Rf = [[Fraction(float(R[n, k])) for k in range(K)] for n in range(N)]
    g_w = _bf_pow2_scale(max(abs(v) for row in Rf for v in row))
    g_a = Fraction(g_a)
    xq = [_bf_quant_dequant(row, g_a) for row in Xh]
    wq = [_bf_quant_dequant(row, g_w) for row in Rf]
    y = np.empty((M, N))
    for m in range(M):
        U = [sum(Xh[m][k] * Fraction(float(L1[k, j])) for k in range(K)) for j in range(r)]
        for n in range(N):
            acc = sum(xq[m][k] * wq[n][k] for k in range(K))
            acc += sum(U[j] * Fraction(float(L2[j, n])) for j in range(r))
            acc += Fraction(float(b[n]))
            y[m, n] = float(acc)
    return y


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_forward_matches_exact_rational_bruteforce(seed):
    rng = np.random.default_rng(seed)
    M, K, N, r = 3, 32, 5, 3
    X = synth.to_bf16(rng.standard_normal((M, K)) * np.exp2(rng.integers(-3, 4, size=(1, K))))
    s = synth.to_bf16(np.exp2(rng.uniform(-2, 2, K)))
    R = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    L1 = synth.to_bf16(rng.standard_normal((K, r)))
    L2 = synth.to_bf16(rng.standard_normal((r, N)))
    b = synth.to_bf16(rng.standard_normal(N))
    amax = float(np.max(np.abs(X.astype(np.float64) * s)))
    g_a = nvfp4.global_scale(amax) * (2.0 if seed == 2 else 1.0)
    y = svdq.forward(X, s, R, L1, L2, b, g_a)
    y_bf = _bf_forward(X, s, R, L1, L2, b, g_a)
    np.testing.assert_allclose(y, y_bf, rtol=1e-12, atol=1e-12 * np.abs(y_bf).max())


# ------------------------------------------------------------ decomposition identity

def _representable_rows(rng, rows, K, g, top_scale):
    codes = rng.integers(0, 16, size=(rows, K)).astype(np.uint8)
    for rr in range(rows):
        for bb in range(K // 16):
            codes[rr, bb * 16 + rng.integers(0, 16)] = 7 if rng.random() < 0.5 else 15
    scales = rng.integers(1, 0x7F, size=(rows, K // 16)).astype(np.uint8)
    scales[0, 0] = top_scale
    return nvfp4.dequantize(codes, scales, g)


def test_decomposition_identity_reproduces_smoothed_weight():
    """With R and X_hat exactly representable, Q(R) + (L1 L2)^T == W diag(lambda)
    and y == X W^T + b to float64 round-off."""
    rng = np.random.default_rng(7)
    M, K, N, r = 9, 64, 24, 4
    g_w, g_a = 2.0 ** -9, 2.0 ** -3
    R = _representable_rows(rng, N, K, g_w, 0x7E).astype(np.float32)
    X_hat = _representable_rows(rng, M, K, g_a, 0x7E)
    smooth_inv = np.exp2(rng.integers(-3, 4, K)).astype(np.float64)     # powers of two
    X = X_hat / smooth_inv                                              # exact
    assert np.array_equal(synth.to_bf16(X), X)
    L1 = synth.to_bf16(rng.standard_normal((K, r)) * 0.1)
    L2 = synth.to_bf16(rng.standard_normal((r, N)) * 0.1)
    b = synth.to_bf16(rng.standard_normal(N))

    cw, sw, gw = svdq.quantize_weights(R)
    assert gw == g_w
    W_hat = nvfp4.dequantize(cw, sw, gw) + (L1.astype(np.float64) @ L2.astype(np.float64)).T
    np.testing.assert_array_equal(nvfp4.dequantize(cw, sw, gw), R.astype(np.float64))
    W = W_hat * smooth_inv[None, :]              # W diag(lambda_eff)^-1 ... lambda = 1/smooth_inv
    y_direct = X @ W.T + b[None, :]
    y = svdq.forward(X, smooth_inv, R, L1, L2, b, g_a)
    np.testing.assert_allclose(y, y_direct, rtol=1e-12, atol=1e-12 * np.abs(y_direct).max())


def test_zero_residual_leaves_only_the_lowrank_branch():
    rng = np.random.default_rng(8)
    M, K, N, r = 5, 48, 7, 32
    X = synth.to_bf16(rng.standard_normal((M, K)))
    s = synth.to_bf16(np.exp2(rng.uniform(-1, 1, K)))
    L1 = synth.to_bf16(rng.standard_normal((K, r)))
    L2 = synth.to_bf16(rng.standard_normal((r, N)))
    cw, sw, gw = svdq.quantize_weights(np.zeros((N, K), np.float32))
    assert gw == 1.0 and np.all(cw == 0) and np.all(sw == 0)
    y = svdq.forward(X, s, np.zeros((N, K), np.float32), L1, L2, None, 1.0)
    # float32 pairwise products of bf16 values are exact, so an fp64 einsum is an independent evaluation
    Xh = np.einsum("mk,k->mk", X.astype(np.float64), s.astype(np.float64))
    ref = np.einsum("mk,kj,jn->mn", Xh, L1.astype(np.float64), L2.astype(np.float64))
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-10)


def test_identity_smoothing_no_lowrank_is_plain_nvfp4_gemm():
    rng = np.random.default_rng(9)
    M, K, N = 6, 64, 10
    g = 2.0 ** -2
    Xq = _representable_rows(rng, M, K, g, 0x7E)
    Rq = _representable_rows(rng, N, K, g, 0x7E).astype(np.float32)
    assert np.array_equal(synth.to_bf16(Xq), Xq)
    y = svdq.forward(Xq, np.ones(K), Rq, np.zeros((K, 1)), np.zeros((1, N)), None, g)
    np.testing.assert_allclose(y, Xq @ Rq.astype(np.float64).T, rtol=1e-12, atol=1e-12)


def test_synthetic_workload_close_to_unquantized_layer():
    w = synth.svdq_workload(64, 256, 128)
    y = svdq.forward(w.X, w.smooth_inv, w.R, w.L1, w.L2, w.bias, w.g_a)
    ref = w.X.astype(np.float64) @ w.W.astype(np.float64).T + w.bias
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 0.05


# ---------------------------------------------------------------- the dynamic activation scale

def test_dynamic_scale_closed_forms():
    # amax of X_hat exactly 6 * 448 = 2688 -> g = 1; one ulp above -> 2; half of it -> 1/2
    s = np.ones(64)
    X = np.zeros((3, 64))
    X[1, 5] = -2688.0
    assert svdq.dynamic_act_scale(X, s) == 1.0
    X[1, 5] = np.nextafter(2688.0, np.inf)
    assert svdq.dynamic_act_scale(X, s) == 2.0
    X[1, 5] = 1344.0
    assert svdq.dynamic_act_scale(X, s) == 0.5
    X[1, 5] = 1344.0 + 2.0 ** -20
    assert svdq.dynamic_act_scale(X, s) == 1.0
    assert svdq.dynamic_act_scale(np.zeros((2, 64)), s) == 1.0


def test_dynamic_scale_uses_the_smoothed_activations_and_scales_exactly():
    rng = np.random.default_rng(11)
    X = synth.to_bf16(rng.standard_normal((16, 128)) * 3.0)
    s = synth.to_bf16(np.exp2(rng.integers(-3, 4, size=128)).astype(np.float64))   # powers of two
    amax = np.max(np.abs(X * s[None, :]))
    g = svdq.dynamic_act_scale(X, s)
    assert g * 2688.0 >= amax > g * 1344.0 and np.log2(g) == int(np.log2(g))
    for k in (-3, 5):                       # an exact power-of-two rescale of X rescales g exactly
        assert svdq.dynamic_act_scale(X * 2.0 ** k, s) == g * 2.0 ** k
