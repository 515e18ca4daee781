"""Pins for oracle.formats: code tables and round-to-nearest-even quantizers.

Independent checks: the published value lists of the formats, torch's
float8_e4m3fn conversion (a library routine), and brute-force nearest search.
"""

import numpy as np
import torch

from oracle import formats as F


def test_e2m1_table_matches_published_values():
    # OCP microscaling E2M1: magnitudes of codes 0..7; bit 3 is the sign.
    expected = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert list(F.E2M1_TABLE[:8]) == expected
    assert list(-F.E2M1_TABLE[8:]) == expected
    assert np.signbit(F.E2M1_TABLE[8])                   # code 0x8 is -0
    assert F.E2M1_TABLE[7] == 1.5 * 2 ** 2               # largest: 1.1b x 2^2


def test_e4m3_table_landmarks():
    t = F.E4M3_TABLE
    assert t[0x7E] == 448.0 == 1.75 * 2 ** 8
    assert t[0x01] == 2.0 ** -9                           # smallest subnormal
    assert t[0x08] == 2.0 ** -6                           # smallest normal
    assert t[0x38] == 1.0
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert np.signbit(t[0x80]) and t[0x80] == 0.0
    finite = t[:0x7F]
    assert np.all(np.diff(finite) > 0)                    # codes 0..126 ascending


def test_e4m3_table_matches_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    both_nan = np.isnan(ref) & np.isnan(F.E4M3_TABLE)
    assert np.all(both_nan | (ref == F.E4M3_TABLE))


def _torch_e4m3_code(v):
    return torch.from_numpy(np.asarray(v, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_quantize_e4m3_all_bf16_values_vs_torch():
    # every non-negative finite bf16 value below 464 (the saturation midpoint)
    bits = np.arange(0, 0x7F80, dtype=np.uint32)
    vals = (bits << 16).view(np.float32)
    vals = vals[vals < 464.0]
    assert np.array_equal(F.quantize_e4m3(vals), _torch_e4m3_code(vals))


def test_quantize_e4m3_float32_samples_and_midpoints_vs_torch():
    rng = np.random.default_rng(1)
    samples = np.concatenate([
        rng.uniform(0, 464, 200000),
        np.exp2(rng.uniform(-14, 8.85, 200000)),
    ]).astype(np.float32)
    # exact midpoints between neighbouring finite E4M3 values
    grid = F.E4M3_TABLE[:0x7F]
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    vals = np.concatenate([samples, mids, grid.astype(np.float32)])
    vals = vals[vals < 464.0]
    assert np.array_equal(F.quantize_e4m3(vals), _torch_e4m3_code(vals))


def test_quantize_e4m3_saturates():
    assert F.quantize_e4m3(np.array([448.0, 460.0, 1e6]))[0] == 0x7E
    assert np.all(F.quantize_e4m3(np.array([448.0, 460.0, 1e6])) == 0x7E)


def _bruteforce_e2m1(v):
    """argmin over all 16 codes of |clamp(v) - value|; ties to the even code; sign from signbit."""
    out = np.empty(v.shape, dtype=np.uint8)
    vals = F.E2M1_TABLE
    for i, x in enumerate(v):
        c = min(max(float(x), -6.0), 6.0)
        best = None
        for code in range(16):
            if (code >> 3) != (1 if np.signbit(x) else 0):
                continue
            d = abs(c - vals[code])
            if best is None or d < best[0] or (d == best[0] and code % 2 == 0):
                best = (d, code)
        out[i] = best[1]
    return out


def test_quantize_e2m1_bruteforce_all_bf16():
    bits = np.arange(0, 0x10000, dtype=np.uint32)
    vals = (bits << 16).view(np.float32)
    vals = vals[np.isfinite(vals)]
    # scale into the interesting range so that every midpoint is crossed
    for scale in (2.0 ** -2, 1.0):
        v = (vals.astype(np.float64) * scale)
        v = v[np.abs(v) < 16]
        assert np.array_equal(F.quantize_e2m1(v), _bruteforce_e2m1(v))


def test_quantize_e2m1_midpoints_by_hand():
    # value -> code, ties to the even code
    cases = [(0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6),
             (0.2499, 0), (0.2501, 1), (5.0001, 7), (6.0, 7), (9.0, 7),
             (-0.25, 8), (-0.75, 10), (-5.0, 14), (-6.5, 15), (-0.0, 8), (0.0, 0)]
    v = np.array([c[0] for c in cases])
    assert [int(c) for c in F.quantize_e2m1(v)] == [c[1] for c in cases]


def test_bf16_round_vs_torch():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.standard_normal(100000) * 10, rng.uniform(-1, 1, 1000) * 1e-30]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(F.bf16_round(x), ref)


def test_bf16_round_is_a_single_rounding_from_float64_including_subnormals():
    # float32 values (normal and subnormal): the same as torch's float32 -> bfloat16 cast
    rng = np.random.default_rng(9)
    v = (rng.standard_normal(50000) * np.exp2(rng.integers(-149, 127, 50000))).astype(np.float32)
    v = v[np.isfinite(v)]
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(F.bf16_round(v.astype(np.float64)), ref)
    # a float64 just above the midpoint 1 + 2^-8 rounds up, although float32 would first land on
    # the midpoint and then tie to even (down)
    x = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert F.bf16_round(np.array([x]))[0] == 1.0 + 2.0 ** -7
    # bf16 subnormals: steps of 2^-133; a quarter step rounds down, three quarters up, a half to even
    s = 2.0 ** -133
    assert F.bf16_round(np.array([8 * s + s / 4, 8 * s + 3 * s / 4, 9 * s + s / 2, 10 * s + s / 2])).tolist() == \
        [8 * s, 9 * s, 10 * s, 10 * s]
    assert F.bf16_round(np.array([s / 2, s / 2 + 2.0 ** -160])).tolist() == [0.0, s]
    # signs, zeros, infinities, NaN, overflow
    out = F.bf16_round(np.array([-0.0, np.inf, -np.inf, np.nan, 2.0 ** 128 * 0.9999]))
    assert np.signbit(out[0]) and out[0] == 0.0 and out[1] == np.inf and out[2] == -np.inf and np.isnan(out[3])
    assert out[4] == 2.0 ** 128
