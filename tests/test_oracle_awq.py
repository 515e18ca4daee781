"""Pins for oracle.awq: integer special case, exact rational brute force, hand values."""

from fractions import Fraction

import numpy as np

from oracle import awq
import synth


def test_dequantize_by_hand():
    q = np.zeros((1, 64), dtype=np.int64); q[0, :3] = [0, 15, 8]
    d = awq.dequantize(q, np.array([[0.5]]), np.array([[8.0]]))
    assert d[0, :3].tolist() == [-4.0, 3.5, 0.0]


def test_unit_scale_zero_eight_is_an_integer_matmul():
    rng = np.random.default_rng(0)
    M, K, N = 7, 192, 33
    X = rng.integers(-50, 50, size=(M, K))
    q = rng.integers(0, 16, size=(N, K))
    y = awq.forward(X.astype(np.float64), q, np.ones((N, K // 64)), np.full((N, K // 64), 8.0))
    ref = X.astype(np.int64) @ (q.astype(np.int64) - 8).T
    assert np.array_equal(y, ref.astype(np.float64))


def test_forward_matches_exact_rational_bruteforce():
    rng = np.random.default_rng(1)
    M, K, N = 2, 128, 3
    X = synth.to_bf16(rng.standard_normal((M, K)))
    q = rng.integers(0, 16, size=(N, K))
    s = synth.to_bf16(np.abs(rng.standard_normal((N, K // 64))) * 0.01)
    z = rng.integers(0, 16, size=(N, K // 64)).astype(np.float64)
    b = synth.to_bf16(rng.standard_normal(N))
    y = awq.forward(X, q, s, z, b)
    for m in range(M):
        for n in range(N):
            acc = Fraction(float(b[n]))
            for k in range(K):
                g = k // 64
                acc += Fraction(float(X[m, k])) * (int(q[n, k]) - Fraction(float(z[n, g]))) * Fraction(float(s[n, g]))
            assert abs(y[m, n] - float(acc)) <= 1e-12 * max(1.0, abs(float(acc)))


def test_unpack_low_nibble_first():
    assert awq.unpack_qweight(np.array([[0x21, 0xF0]], dtype=np.uint8)).tolist() == [[1, 2, 0, 15]]


def test_synthetic_awq_workload_is_valid_minmax_quantization():
    w = synth.awq_workload(4, 256, 16)
    assert w.q.max() <= 15 and w.zeros.max() <= 15 and w.zeros.min() >= 0
    assert np.array_equal(awq.unpack_qweight(w.qweight), w.q.astype(np.int64))
    deq = awq.dequantize(w.q, w.scales, w.zeros)
    # min/max quantization error is at most half a step (plus the zero-point rounding)
    step = np.repeat(w.scales.astype(np.float64), 64, axis=1)
    assert np.all(np.abs(deq - w.W) <= 1.01 * step)
