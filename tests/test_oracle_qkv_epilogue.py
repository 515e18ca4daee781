"""Pins of the QKV epilogue oracle (per-head RMSNorm + RoPE): closed forms, the pairing and
sign conventions, invariants of rotations, and the q / k / v layout."""

import math

import numpy as np
import pytest

from oracle import qkv_epilogue as E


def test_rmsnorm_closed_forms():
    # mean (not sum) of squares: [1, 1, 1, 1] stays 1; [3, 4] -> [3, 4] / sqrt(12.5)
    assert np.allclose(E.rmsnorm_heads(np.ones((1, 1, 4)), np.ones(4), 0.0), 1.0, rtol=0, atol=1e-15)
    out = E.rmsnorm_heads(np.array([[[3.0, 4.0]]]), np.array([2.0, 0.5]), 0.0)
    assert np.allclose(out, [[[2 * 3 / math.sqrt(12.5), 0.5 * 4 / math.sqrt(12.5)]]], rtol=1e-15)
    # eps sits under the root: [1, 1] with eps = 1 -> 1 / sqrt(2)
    assert np.allclose(E.rmsnorm_heads(np.ones((1, 1, 2)), np.ones(2), 1.0), 1 / math.sqrt(2.0), rtol=1e-15)


def test_rmsnorm_is_scale_invariant_and_per_head():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, 4, 16))
    w = rng.standard_normal(16)
    base = E.rmsnorm_heads(x, w, 0.0)
    assert np.allclose(E.rmsnorm_heads(x * 7.5, w, 0.0), base, rtol=1e-13)
    y = x.copy()
    y[:, 2] *= 100.0                                       # rescaling one head leaves the others alone
    assert np.allclose(E.rmsnorm_heads(y, w, 0.0), base, rtol=1e-13)
    assert np.allclose(np.sqrt(np.mean(E.rmsnorm_heads(x, np.ones(16), 0.0) ** 2, axis=-1)), 1.0, rtol=1e-13)


def test_rope_pairs_are_consecutive_and_rotate_counterclockwise():
    x = np.array([[[1.0, 2.0, 3.0, 4.0]]])
    cos = np.array([[0.0, 1.0]])                           # pair 0 by a quarter turn, pair 1 not at all
    sin = np.array([[1.0, 0.0]])
    assert np.array_equal(E.rope(x, cos, sin), [[[-2.0, 1.0, 3.0, 4.0]]])
    c, s = E.rope_tables(np.array([[0.3]]))
    assert np.allclose(E.rope(np.array([[[1.0, 0.0]]]), c, s), [[[math.cos(0.3), math.sin(0.3)]]], rtol=1e-15)
    assert np.array_equal(E.rope(x, np.ones((1, 2)), np.zeros((1, 2))), x)


def test_rope_preserves_pair_norms_and_composes():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 3, 8))
    a, b = rng.uniform(-4, 4, (5, 4)), rng.uniform(-4, 4, (5, 4))
    r = E.rope(x, *E.rope_tables(a))
    assert np.allclose(np.hypot(r[..., 0::2], r[..., 1::2]), np.hypot(x[..., 0::2], x[..., 1::2]), rtol=1e-13)
    assert np.allclose(E.rope(r, *E.rope_tables(b)), E.rope(x, *E.rope_tables(a + b)), rtol=0, atol=1e-12)


def test_rope_scores_depend_only_on_the_position_difference():
    rng = np.random.default_rng(3)
    D = 8
    freqs = 1.0 / 10000.0 ** (np.arange(D // 2) / (D // 2))
    q, k = rng.standard_normal((1, 1, D)), rng.standard_normal((1, 1, D))

    def at(v, pos):
        return E.rope(v, *E.rope_tables(pos * freqs[None, :]))

    s1 = np.sum(at(q, 7) * at(k, 3))
    s2 = np.sum(at(q, 104) * at(k, 100))
    assert abs(s1 - s2) < 1e-12


def test_epilogue_layout_and_v_passthrough():
    rng = np.random.default_rng(4)
    M, H, D = 3, 2, 4
    qkv = rng.standard_normal((M, 3 * H * D))
    w_q, w_k = rng.standard_normal(D), rng.standard_normal(D)
    cos, sin = E.rope_tables(rng.uniform(-3, 3, (M, D // 2)))
    q, k, v = E.qkv_epilogue(qkv, H, w_q, w_k, 1e-6, cos, sin)
    assert np.array_equal(v, qkv[:, 2 * H * D:].reshape(M, H, D))
    head1_of_k = qkv[:, H * D + D:H * D + 2 * D][:, None, :]
    assert np.allclose(k[:, 1:2], E.rope(E.rmsnorm_heads(head1_of_k, w_k, 1e-6), cos, sin), rtol=1e-14)
    head0_of_q = qkv[:, :D][:, None, :]
    assert np.allclose(q[:, 0:1], E.rope(E.rmsnorm_heads(head0_of_q, w_q, 1e-6), cos, sin), rtol=1e-14)
    with pytest.raises(ValueError):
        E.qkv_epilogue(qkv[:, :-1], H, w_q, w_k, 1e-6, cos, sin)
