"""Host weight packing (C++) against the oracle: bit-exact codes, scales and g_w."""

import numpy as np
import pytest

import bit_diffusion_transformer_act_b200 as P  # noqa: E402  (conftest has built the library)

from oracle import nvfp4, svdq  # noqa: E402
import synth  # noqa: E402
from parity_util import unswizzle  # noqa: E402


def _sections(blob, N, K, rank=32):
    al = lambda x: (x + 1023) // 1024 * 1024  # noqa: E731
    off = 1024
    l1s = off; off = al(off + 2 * rank * K * 2)
    codes = off; off = al(off + N * K // 2)
    scales = off; off = al(off + ((N + 127) // 128 * 128) * (K // 16))
    l2t = off; off = al(off + N * rank * 2)
    bias = off; off = al(off + (N + 255) // 256 * 256 * 2)       # zero-padded to 256 columns
    assert off == blob.size
    assert not blob[bias + N * 2:off].any()
    return {
        "l1s": blob[l1s:l1s + 2 * rank * K * 2].view(np.uint16).reshape(2, rank, K),
        "codes": blob[codes:codes + N * K // 2].reshape(N, K // 2),
        "scales": blob[scales:scales + ((N + 127) // 128 * 128) * (K // 16)],
        "l2t": blob[l2t:l2t + N * rank * 2].view(np.uint16).reshape(N, rank),
        "bias": blob[bias:bias + N * 2].view(np.uint16),
    }


def _check_pack(R, L1, L2, b, smooth):
    N, K = R.shape
    blob, gw = P.svdq_pack_weights(R, synth.bf16_bits(L1), synth.bf16_bits(L2),
                                   None if b is None else synth.bf16_bits(b), synth.bf16_bits(smooth))
    cw, sw, gw_ref = svdq.quantize_weights(R)
    assert gw == gw_ref
    s = _sections(blob, N, K)
    assert np.array_equal(s["codes"], nvfp4.pack_nibbles(cw))
    assert np.array_equal(unswizzle(s["scales"], N, K), sw)
    # (diag(smooth) L1)^T = hi + lo exactly, hi the nearest bf16
    prod = (smooth.astype(np.float64)[:, None] * L1.astype(np.float64)).T
    hi = synth.bf16_from_bits(s["l1s"][0]).astype(np.float64)
    lo = synth.bf16_from_bits(s["l1s"][1]).astype(np.float64)
    assert np.array_equal(hi + lo, prod)
    assert np.array_equal(hi, synth.to_bf16(prod).astype(np.float64))
    # L2 / g_w, transposed
    assert np.array_equal(synth.bf16_from_bits(s["l2t"]).astype(np.float64), L2.astype(np.float64).T / gw)
    assert np.array_equal(s["bias"], np.zeros(N, np.uint16) if b is None else synth.bf16_bits(b))
    assert bytes(blob[:8]) == b"SVDQNVF4"
    return blob


def test_pack_synthetic_tiny_layer_is_bit_exact():
    w = synth.svdq_workload(256, 512, 512)
    _check_pack(w.R, w.L1, w.L2, w.bias, w.smooth_inv)


def test_pack_ragged_width_is_bit_exact():
    # N % 128 == 64: scale rows padded to 128 with zeros, bias padded to 256 columns
    w = synth.svdq_workload(64, 256, 320)
    blob = _check_pack(w.R, w.L1, w.L2, w.bias, w.smooth_inv)
    s = _sections(blob, 320, 256)
    assert not unswizzle_all_rows(s["scales"], 320, 256)[320:].any()


def unswizzle_all_rows(scales, N, K):
    return unswizzle(scales, (N + 127) // 128 * 128, K)


def test_pack_attention_layer_is_bit_exact():
    w = synth.svdq_workload(64, 3072, 3072)
    _check_pack(w.R, w.L1, w.L2, None, w.smooth_inv)


def test_pack_ties_zero_blocks_and_subnormal_scales():
    rng = np.random.default_rng(5)
    N, K = 128, 256
    g = 2.0 ** -4
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0])
    R = np.zeros((N, K))
    for n in range(N):
        kind = n % 5
        if kind == 0:
            continue                                        # zero row -> zero scales and codes
        S = nvfp4.E4M3_TABLE[rng.integers(1, 0x7F)] if kind != 3 else 2.0 ** -9
        blk = rng.choice(mids, size=K) * rng.choice([-1.0, 1.0], size=K) * S * g
        blk[::16] = 6.0 * S * g                             # every block's amax is 6 S g
        if kind == 4:
            blk[1::16] = 6.375 * S * g                      # amax/6 lands between two E4M3 values
        R[n] = blk
    R[1, 0] = 6.0 * 448 * g                                 # pins g_w
    R = R.astype(np.float32)
    L1 = synth.to_bf16(rng.standard_normal((K, 32)))
    L2 = synth.to_bf16(rng.standard_normal((32, N)))
    _check_pack(R, L1, L2, synth.to_bf16(rng.standard_normal(N)), synth.to_bf16(np.exp2(rng.uniform(-3, 3, K))))


def test_pack_rejects_bad_shapes_and_values():
    L1 = np.zeros((64, 32), np.uint16)
    L2 = np.zeros((32, 128), np.uint16)
    sm = np.full(64, 0x3F80, np.uint16)
    with pytest.raises(P.SvdqError):
        P.svdq_pack_weights(np.zeros((100, 64), np.float32), L1, np.zeros((32, 100), np.uint16), None, sm)
    R = np.zeros((128, 64), np.float32)
    R[3, 5] = np.nan
    with pytest.raises(P.SvdqError):
        P.svdq_pack_weights(R, L1, L2, None, sm)


def test_int4_packer_matches_the_oracle_bit_for_bit():
    # codes (as E4M3 bytes of the integers), the bf16 scales (widened, group-major), L2^T and bias
    import torch
    from oracle import int4 as Q
    rng = np.random.default_rng(17)
    N, K = 256, 320
    R = (rng.standard_normal((N, K)) * np.exp2(rng.integers(-6, 2, (N, 1)))).astype(np.float32)
    R[3] = 0.0                                                      # a zero row: scales 0, codes 0
    R[5, 64:128] = 7.0 * 0.5                                        # a group of exact code 7 at s = 0.5
    L1 = synth.to_bf16(rng.standard_normal((K, 32)) * 0.1)
    L2 = synth.to_bf16(rng.standard_normal((32, N)) * 0.1)
    b = synth.to_bf16(rng.standard_normal(N) * 0.01)
    sm = synth.to_bf16(np.exp(rng.uniform(-1, 1, K)))
    blob = P.svdq_int4_pack_weights(R, synth.bf16_bits(L1), synth.bf16_bits(L2), synth.bf16_bits(b),
                                    synth.bf16_bits(sm))
    off_l1s = 1024
    off_codes = off_l1s + ((2 * 32 * K * 2 + 1023) // 1024) * 1024
    codes = blob[off_codes:off_codes + N * K].reshape(N, K)
    off_sc = off_codes + ((N * K + 1023) // 1024) * 1024
    scales = blob[off_sc:off_sc + N * (K // 64) * 4].view(np.float32).reshape(K // 64, N)
    c_ref, s_ref = Q.quantize(R)
    vals = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(vals, c_ref.astype(np.float64))
    assert np.array_equal(scales.T.astype(np.float64), s_ref)
    assert bytes(blob[:8]) == b"SVDQINT4"
    off_l2t = off_sc + ((N * (K // 64) * 4 + 1023) // 1024) * 1024
    l2t = blob[off_l2t:off_l2t + N * 32 * 2].view(np.uint16).reshape(N, 32)
    assert np.array_equal(l2t, synth.bf16_bits(L2).T)
    off_b = off_l2t + ((N * 32 * 2 + 1023) // 1024) * 1024
    assert np.array_equal(blob[off_b:off_b + 2 * N].view(np.uint16), synth.bf16_bits(b))
    assert P.LIB.svdq_int4_packed_weight_bytes(N, K, 32) == blob.size
