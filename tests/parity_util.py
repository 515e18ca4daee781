"""Helpers shared by the parity tests (test code; imports the oracle, never the reverse)."""

import numpy as np


def swizzled_offset(row, group, K):
    """Byte offset of the scale of (row, group) in the documented 128x4 atom layout."""
    rb, r = row // 128, row % 128
    atom, j = group // 4, group % 4
    return (rb * (K // 64) + atom) * 512 + (r % 32) * 16 + (r // 32) * 4 + j


def unswizzle(buf, rows, K):
    """numpy restatement of the header's scale layout: bytes -> [rows, K/16]."""
    buf = np.asarray(buf, dtype=np.uint8).reshape(-1)
    r = np.arange(rows)[:, None]
    g = np.arange(K // 16)[None, :]
    return buf[swizzled_offset(r, g, K)]


def bf16_ulp(v):
    """Spacing of bf16 values at |v| (for v != 0)."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    a = np.where(a == 0, np.finfo(np.float32).tiny, a)
    e = np.floor(np.log2(a))
    return np.exp2(e - 7)


def check_output(y_gpu, y_ref, rel_l2_max=5e-3, elem_rel_rms=1e-2):
    """Tolerance of the layer outputs (bf16) against the float64 oracle.

    * relative L2 error <= 5e-3 against the unrounded oracle;
    * per element |y_gpu - bf16(y_ref)| <= max(1e-2 * rms(y_ref), 1 bf16 ulp of y_ref).
    Returns a dict of statistics; raises AssertionError when a bound fails."""
    from oracle.formats import bf16_round
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    yr = bf16_round(y_ref)
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    denom = np.linalg.norm(y_ref)
    rel = float(np.linalg.norm(y_gpu - y_ref) / denom) if denom > 0 else float(np.linalg.norm(y_gpu))
    d = np.abs(y_gpu - yr)
    tol = np.maximum(elem_rel_rms * rms, bf16_ulp(yr))
    bad = d > tol
    stats = {"rel_l2": rel, "max_abs_over_rms": float(d.max() / rms) if rms > 0 else float(d.max()),
             "n_bad": int(bad.sum()), "frac_literal_over": float(np.mean(np.abs(y_gpu - y_ref) > elem_rel_rms * rms))}
    assert rel <= rel_l2_max, stats
    assert not bad.any(), (stats, np.argwhere(bad)[:5])
    return stats
