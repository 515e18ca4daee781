"""Pins of the INT4 group-64 oracle (oracle/int4.py): the bf16 scale rounding straight from the
exact quotient, the integer code rounding and range, exact round trips, an exact-rational brute
force of the whole layer, the decomposition identity and an integer special case."""

from fractions import Fraction
import math

import numpy as np
import torch

from oracle import int4 as Q
import synth


def test_bf16_rne_matches_torch_on_float32_values_and_avoids_double_rounding():
    rng = np.random.default_rng(0)
    v = (rng.standard_normal(20000) * np.exp2(rng.integers(-30, 30, 20000))).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(Q.bf16_rne(v.astype(np.float64)), ref)
    # 1 + 2^-8 is the midpoint between the bf16 values 1 and 1 + 2^-7; a value just above it
    # rounds to that midpoint in float32 and then (ties to even) down to 1 -- the wrong way
    v = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert np.float32(v) == 1.0 + 2.0 ** -8
    assert Q.bf16_rne(np.array([v]))[0] == 1.0 + 2.0 ** -7
    assert Q.bf16_rne(np.array([-v]))[0] == -(1.0 + 2.0 ** -7)
    assert Q.bf16_rne(np.array([1.0 + 2.0 ** -8]))[0] == 1.0          # an exact tie goes to even
    assert Q.bf16_rne(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6


def test_scale_and_code_rounding_by_hand():
    # amax 7 -> s = 1: codes are the nearest integers, ties to even
    x = np.zeros((1, 64))
    x[0, :10] = [7.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, -3.5, 0.49, -7.0]
    c, s = Q.quantize(x)
    assert s[0, 0] == 1.0
    assert c[0, :10].tolist() == [7, 2, 4, -2, 0, 0, 2, -4, 0, -7]
    # a zero group: scale 0, codes 0; the next group independent
    x = np.zeros((1, 128))
    x[0, 64] = -14.0
    c, s = Q.quantize(x)
    assert s[0].tolist() == [0.0, 2.0] and c[0, 64] == -7 and not c[0, :64].any()
    # amax / 7 rounded to bf16: 10 / 7 = 1.428571... -> 1.4296875 (183 / 128)
    x = np.zeros((1, 64))
    x[0, 3] = 10.0
    c, s = Q.quantize(x)
    assert s[0, 0] == 183 / 128 and c[0, 3] == 7


def test_codes_stay_within_seven_and_round_trip_exactly():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((64, 512)) * np.exp2(rng.integers(-8, 8, (64, 1)))
    c, s = Q.quantize(x)
    assert c.min() >= -7 and c.max() <= 7
    # every element within half a step of its group scale
    err = np.abs(Q.dequantize(c, s) - x).reshape(64, 8, 64)
    assert np.all(err <= 0.5 * s[:, :, None] * (1 + 1e-12))
    # representable groups (a +-7 in each, bf16 scales) come back exactly
    codes = rng.integers(-7, 8, (16, 256)).astype(np.int8)
    codes[:, ::64] = 7 * rng.choice([-1, 1], (16, 4))
    scales = synth.to_bf16(np.exp(rng.uniform(-5, 5, (16, 4)))).astype(np.float64)
    c2, s2 = Q.quantize(Q.dequantize(codes, scales))
    assert np.array_equal(c2, codes) and np.array_equal(s2, scales)
    # nibble packing (two's complement, even element low) round-trips
    assert np.array_equal(Q.unpack_nibbles(Q.pack_nibbles(codes)), codes)
    assert Q.pack_nibbles(np.array([[-1, 7, -8, 1] + [0] * 60], dtype=np.int8))[0, :2].tolist() == [0x7F, 0x18]


def _bf16_rne_exact(q):
    """Nearest bfloat16 of a positive Fraction, ties to even, by exact comparison."""
    e = math.floor(math.log2(q.numerator) - math.log2(q.denominator))
    while Fraction(2) ** e > q:
        e -= 1
    while Fraction(2) ** (e + 1) <= q:
        e += 1
    step = Fraction(2) ** (e - 7)
    lo = (q // step) * step
    rem = q - lo
    if rem * 2 > step or (rem * 2 == step and (lo / step) % 2 == 1):
        lo += step
    return lo


def _rint_even(q):
    f = math.floor(q)
    d = q - f
    if d > Fraction(1, 2) or (d == Fraction(1, 2) and f % 2 == 1):
        f += 1
    return f


def _quantize_exact(rowvals):
    out_c, out_s = [], []
    for g in range(len(rowvals) // 64):
        grp = rowvals[64 * g:64 * g + 64]
        amax = max(abs(v) for v in grp)
        if amax == 0:
            out_s.append(Fraction(0))
            out_c += [0] * 64
            continue
        s = _bf16_rne_exact(amax / 7)
        out_s.append(s)
        out_c += [max(-8, min(7, _rint_even(v / s))) for v in grp]
    return out_c, out_s


def test_forward_against_exact_rational_brute_force():
    for seed in range(3):
        rng = np.random.default_rng(seed)
        M, K, N, r = 3, 128, 4, 32
        X = synth.to_bf16(rng.standard_normal((M, K)) * 3)
        sm = synth.to_bf16(np.exp(rng.uniform(-1, 1, K)))
        R = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
        L1 = synth.to_bf16(rng.standard_normal((K, r)) * 0.1)
        L2 = synth.to_bf16(rng.standard_normal((r, N)) * 0.1)
        b = synth.to_bf16(rng.standard_normal(N) * 0.01)
        y = Q.forward(X, sm, R, L1, L2, b)
        F = Fraction
        for m in range(M):
            xh = [F(float(X[m, k])) * F(float(sm[k])) for k in range(K)]
            cx, sx = _quantize_exact(xh)
            u = [sum(xh[k] * F(float(L1[k, j])) for k in range(K)) for j in range(r)]
            for n in range(N):
                cw, sw = _quantize_exact([F(float(R[n, k])) for k in range(K)])
                acc = sum(sx[k // 64] * sw[k // 64] * cx[k] * cw[k] for k in range(K))
                acc += sum(u[j] * F(float(L2[j, n])) for j in range(r)) + F(float(b[n]))
                assert abs(float(acc) - y[m, n]) <= 1e-12 * max(1.0, abs(float(acc)))


def test_decomposition_identity_and_integer_special_case():
    rng = np.random.default_rng(7)
    M, K, N = 5, 256, 6
    # R representable: codes in -7..7 with a +-7 per group, bf16 scales
    cw = rng.integers(-7, 8, (N, K)).astype(np.int8)
    cw[:, ::64] = 7
    sw = synth.to_bf16(np.exp(rng.uniform(-6, -2, (N, K // 64)))).astype(np.float64)
    R = Q.dequantize(cw, sw)
    assert np.array_equal(R.astype(np.float32).astype(np.float64), R)
    L1 = synth.to_bf16(rng.standard_normal((K, 32)) * 0.1)
    L2 = synth.to_bf16(rng.standard_normal((32, N)) * 0.1)
    sm = synth.to_bf16(np.exp(rng.uniform(-1, 1, K)))
    # X_hat representable too, so Q is the identity on both sides
    cx = rng.integers(-7, 8, (M, K)).astype(np.int8)
    cx[:, ::64] = -7
    sx = synth.to_bf16(np.exp(rng.uniform(-2, 2, (M, K // 64)))).astype(np.float64)
    Xh = Q.dequantize(cx, sx)
    X = Xh / sm.astype(np.float64)[None, :]
    W = R + (L1.astype(np.float64) @ L2.astype(np.float64)).T                 # W diag(lambda)
    y = Q.forward(X, sm, R.astype(np.float32), L1, L2, None)
    assert np.allclose(y, Xh @ W.T, rtol=1e-12, atol=1e-12)
    # identity smoothing, no low-rank: sum_g s_x s_w (integer dot product)
    y0 = Q.forward(Xh, np.ones(K), R.astype(np.float32), np.zeros((K, 32)), np.zeros((32, N)), None)
    ref = np.zeros((M, N))
    for g in range(K // 64):
        dot = cx[:, 64 * g:64 * g + 64].astype(np.int64) @ cw[:, 64 * g:64 * g + 64].astype(np.int64).T
        ref += sx[:, g:g + 1] * sw[:, g][None, :] * dot
    assert np.allclose(y0, ref, rtol=1e-13, atol=0)
