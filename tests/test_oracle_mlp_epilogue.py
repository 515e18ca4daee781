"""Pins of the MLP epilogue oracle (GELU, then the down projection's activation pass)."""

import math

import numpy as np

from oracle import mlp_epilogue as E
from oracle import nvfp4, svdq
import synth


def test_gelu_closed_forms_exclude_the_tanh_approximation():
    assert E.gelu(0.0) == 0.0
    assert abs(E.gelu(1.0) - 0.8413447460685429) < 1e-15                 # Phi(1); tanh form gives 0.84119
    assert abs(E.gelu(-1.0) + 0.15865525393145707) < 1e-15
    assert E.gelu(10.0) == 10.0
    x = np.linspace(-6, 6, 97)
    assert np.allclose(E.gelu(x) - E.gelu(-x), x, rtol=0, atol=1e-14)     # x Phi(x) + x Phi(-x) = x


def test_hidden_state_rounds_before_and_after_gelu():
    y = np.array([1.0 + 2.0 ** -10])                                      # not a bf16 value
    # bf16(y) = 1 -> GELU = 0.84134... -> bf16 0.83984375; without the first rounding it would be 0.84375
    assert E.hidden_state(y)[0] == 0.83984375
    assert E.hidden_state(np.array([0.0, -20.0, 20.0])).tolist() == [0.0, -0.0, 20.0]


def test_requantize_applies_the_down_projection_smoothing_and_scale():
    rng = np.random.default_rng(5)
    M, F = 16, 256
    y = synth.to_bf16(rng.standard_normal((M, F)) * 2.0)
    L1 = synth.to_bf16(rng.standard_normal((F, 32)) * 0.1)
    h = E.hidden_state(y)
    s1 = np.ones(F)
    g = nvfp4.global_scale(np.max(np.abs(h)))
    c1, sc1, u1 = E.gelu_requantize(y, s1, g, L1)
    # smoothing by 2^3 with the per-tensor scale times 2^3: the same codes and scales, U times 8
    c8, sc8, u8 = E.gelu_requantize(y, s1 * 8.0, g * 8.0, L1)
    assert np.array_equal(c1, c8) and np.array_equal(sc1, sc8)
    assert np.allclose(u8, 8.0 * u1, rtol=1e-15)
    cx, sx = svdq.quantize_activations(h, s1, g)
    assert np.array_equal(c1, cx) and np.array_equal(sc1, sx)


def _gelu_decimal(x, digits=60):
    """x Phi(x) from the Maclaurin series of erf in `digits`-digit decimal arithmetic (an
    evaluation independent of math.erf / math.erfc; with enough digits it stays accurate in the
    tails, where the series' terms grow to about e^(x^2 / 2) before they cancel)."""
    from decimal import Decimal, getcontext
    getcontext().prec = digits
    X = Decimal(x)
    # pi to 64 digits (a constant of mathematics)
    pi = Decimal("3.141592653589793238462643383279502884197169399375105820974944592")
    z = X / Decimal(2).sqrt()
    term, total, n = z, z, 0
    while True:
        n += 1
        term = -term * z * z / n
        add = term / (2 * n + 1)
        total += add
        if abs(add) < Decimal(10) ** -(digits - 5):
            break
    erf = 2 * total / pi.sqrt()
    return X * (1 + erf) / 2


def test_hidden_state_rounds_the_exact_gelu_at_its_nearest_bf16_midpoint():
    # Among all bf16 y with 2^-4 <= |y| <= 4, take the one whose GELU lies closest (relative) to
    # a bf16 rounding midpoint: there an fp32 evaluation may round either way, and the oracle
    # must take the side the exact value is on.
    from decimal import Decimal
    mags = np.array([m * 2.0 ** e for e in range(-4, 2) for m in np.arange(128, 256) / 128.0] + [4.0])
    ys = np.concatenate([mags, -mags])
    g = E.gelu(ys)
    ulp = np.exp2(np.floor(np.log2(np.abs(g))) - 7)
    frac = np.abs(g) / ulp - np.floor(np.abs(g) / ulp)
    dist = np.abs(frac - 0.5) * ulp / np.abs(g)           # relative distance to the nearest midpoint
    i = int(np.argmin(dist))
    assert dist[i] < 2.0 ** -18                           # within reach of fp32 evaluation error
    exact = _gelu_decimal(float(ys[i]))
    lo = math.floor(abs(g[i]) / ulp[i]) * ulp[i]
    mid = Decimal(lo) + Decimal(ulp[i]) / 2
    up = abs(exact) > mid                                 # the side of the midpoint the exact value is on
    expect = math.copysign(lo + ulp[i] if up else lo, g[i])
    assert E.hidden_state(np.array([ys[i]]))[0] == expect
    # and float64 agrees with the 60-digit evaluation to well below the distance
    assert abs(Decimal(float(g[i])) - exact) < Decimal(float(dist[i] * abs(g[i]))) / 1000


def test_gelu_keeps_relative_accuracy_in_the_negative_tail():
    # at x = -10, Phi(x) = 7.6e-24: 1 + erf(x / sqrt 2) rounds to 0 in float64, the erfc form
    # keeps full relative accuracy.  The reference is the decimal series at 150 digits.
    from decimal import Decimal
    for x in (-6.0, -8.0, -10.0, -12.5):
        exact = _gelu_decimal(x, digits=150)
        got = E.gelu(np.array([x]))[0]
        assert got != 0.0
        assert abs(Decimal(got) - exact) <= abs(exact) * Decimal("1e-13"), (x, got, exact)
    # and its bf16 rounding is a normal, non-zero value there
    assert E.hidden_state(np.array([-10.0]))[0] < 0.0


def _hidden_bits(patterns):
    """bf16 bit patterns of hidden_state over bf16 inputs given as bit patterns."""
    u = np.asarray(patterns, dtype=np.uint32)
    with np.errstate(all="ignore"):
        x = (u << 16).view(np.float32).astype(np.float64)
        h = E.hidden_state(x)
    return (np.asarray(h, dtype=np.float32).view(np.uint32) >> 16).astype(np.int64)


def test_hidden_state_closed_forms_over_every_bf16_pattern():
    """Outside a window of magnitudes the table of bf16(x Phi(x)) over bf16 x has closed forms:
    x for x >= 4 (1 - Phi(x) < 2^-14 is below half an ulp), -0 for x <= -16 (x Phi(x) underflows
    below half the smallest bf16 subnormal), x / 2 exactly for 2^-125 <= |x| < 2^-31 (the x^2 /
    sqrt(2 pi) term is below half an ulp of x / 2), and on the subnormal grid x / 2 rounded to
    nearest even.  The fused MLP epilogue reads a window [2^-31, 256) of the table and applies
    these forms elsewhere; this pins them on the oracle over all 65536 patterns."""
    u = np.arange(65536, dtype=np.int64)
    h = _hidden_bits(u)
    w, s = u & 0x7FFF, u >> 15
    finite = w < 0x7F80
    big = finite & (w >= 0x4380)                       # |x| >= 256
    assert np.array_equal(h[big & (s == 0)], u[big & (s == 0)])
    assert np.all(h[big & (s == 1)] == 0x8000)
    assert np.all(h[(w >= 0x4080) & finite & (s == 0)] == u[(w >= 0x4080) & finite & (s == 0)])   # x >= 4
    assert np.all(h[(w >= 0x4180) & finite & (s == 1)] == 0x8000)                                # x <= -16
    mid = (w >= 0x100) & (w < 0x3000)                  # 2^-125 <= |x| < 2^-31
    assert np.array_equal(h[mid], u[mid] - 0x80)
    sub = w < 0x100
    half_even = (w >> 1) + (w & (w >> 1) & 1)
    assert np.array_equal(h[sub], (u[sub] & 0x8000) | half_even[sub])
    assert h[0x7F80] == 0x7F80 and h[0xFF80] == 0xFFC0
    nan = (w > 0x7F80)
    assert np.array_equal(h[nan], u[nan] | 0x40)
