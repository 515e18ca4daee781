"""GPU parity of every kernel against the float64 oracle, through the C ABI: the SVDQ
activation pass and GEMM (NVFP4 and int4 / group 64, static and dynamic activation scale),
the fused QKV (RMSNorm + RoPE) and MLP-up (GELU + re-quantization) epilogues, and both AWQ
W4A16 kernels.

Bars: packed activation codes and scales bit-exact; the low-rank activations
within fp32 accumulation error of the exact product; layer outputs within
relative L2 5e-3 and, per element, max(1e-2 rms(y), 1 bf16 ulp) of the
oracle rounded to bf16.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import awq as oawq
from oracle import nvfp4, svdq
from parity_util import check_output, unswizzle

pytestmark = pytest.mark.gpu


def _bf16_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()


def _pack(P, w, with_bias=True):
    blob, gw = P.svdq_pack_weights(w.R, synth.bf16_bits(w.L1), synth.bf16_bits(w.L2),
                                   synth.bf16_bits(w.bias) if with_bias else None, synth.bf16_bits(w.smooth_inv))
    return torch.from_numpy(blob).cuda(), gw


def _run_svdq(P, X, smooth, packed, g_a, g_w, N):
    M, K = X.shape
    Xd, sd = _bf16_dev(X), _bf16_dev(smooth)
    codes, scales, U = P.svdq_quantize_act_lowrank_down(Xd, sd, packed, g_a)
    Y = P.svdq_w4a4_nvfp4_linear(codes, scales, U, g_a, packed, g_w, M, N, K)
    torch.cuda.synchronize()
    # the low-rank activations come back as bf16 hi and lo parts of U / g_a
    Uc = U.float().cpu().numpy().astype(np.float64)
    U_full = g_a * (Uc[:, :32] + Uc[:, 32:])
    return codes.cpu().numpy(), scales.cpu().numpy(), U_full, Y.float().cpu().numpy()


def _check_act(codes, scales, U, X, smooth, L1, g_a):
    M, K = X.shape
    cx, sx = svdq.quantize_activations(X, smooth, g_a)
    assert np.array_equal(codes, nvfp4.pack_nibbles(cx)), np.argwhere(codes != nvfp4.pack_nibbles(cx))[:5]
    rows = (M + 127) // 128 * 128
    sg = unswizzle(scales, rows, K)
    assert np.array_equal(sg[:M], sx), np.argwhere(sg[:M] != sx)[:5]
    assert np.all(sg[M:] == 0)
    Xh = svdq.smooth(X, smooth)
    U_ref = Xh @ L1.astype(np.float64)
    # fp32 accumulation over K plus the bf16 hi/lo representation (2^-16 relative)
    bound = 1e-5 * (np.abs(Xh) @ np.abs(L1.astype(np.float64))) + 2.0 ** -15 * np.abs(U_ref) + 1e-30
    assert np.all(np.abs(U - U_ref) <= bound), np.max(np.abs(U - U_ref) / bound)


# ---------------------------------------------------------------- edge-case activations

def _edge_activations(M, K, seed):
    """bf16 activations with zero rows, negative zeros, exact E2M1 and E4M3 midpoints."""
    rng = np.random.default_rng(seed)
    smooth = np.exp2(rng.integers(-2, 3, size=K)).astype(np.float32)       # powers of two: x_hat exact
    g_a = 2.0 ** -2
    X = synth.to_bf16(rng.standard_normal((M, K)) * np.exp2(rng.integers(-3, 4, size=(M, 1))))
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1.0, 3.0, 6.0])
    for m in range(M):
        kind = m % 7
        if kind == 1:
            X[m] = 0.0
        elif kind == 2:
            X[m, ::3] = -0.0
            X[m, 1::3] = synth.to_bf16(np.full(len(X[m, 1::3]), -1e-30))
        elif kind in (3, 4):
            if kind == 3:
                S = nvfp4.E4M3_TABLE[rng.integers(1, 0x7F, size=K // 16)].repeat(16)
            else:                                                          # powers of two keep 6.375 S in bf16
                S = np.exp2(rng.integers(-9, 9, size=K // 16)).repeat(16)
            v = rng.choice(mids, size=K) * rng.choice([-1.0, 1.0], size=K) * S * g_a
            v[::16] = 6.0 * S[::16] * g_a
            if kind == 4:
                v[5::16] = -6.375 * S[5::16] * g_a                        # scale tie: amax/6 on a midpoint
            X[m] = (v / smooth).astype(np.float32)
    assert np.array_equal(synth.to_bf16(X), X)
    return X, smooth, g_a


@pytest.fixture(scope="module")
def P(cuda_lib):
    return cuda_lib


def test_tiny_layer(P):
    w = synth.svdq_workload(256, 512, 512)
    packed, gw = _pack(P, w)
    codes, scales, U, Y = _run_svdq(P, w.X, w.smooth_inv, packed, w.g_a, gw, 512)
    _check_act(codes, scales, U, w.X, w.smooth_inv, w.L1, w.g_a)
    y_ref = svdq.forward(w.X, w.smooth_inv, w.R, w.L1, w.L2, w.bias, w.g_a)
    check_output(Y, y_ref)
    assert P.svdq_device_status() == 0


# N % 128 == 64 (64, 320, 704: a ragged 128-wide last tile) and N % 192 == 0 (576) next to the
# 128- and 256-multiples
@pytest.mark.parametrize("M,K,N", [(1, 64, 128), (63, 192, 256), (65, 320, 128), (127, 512, 384),
                                   (129, 256, 640), (200, 1024, 256), (300, 448, 512),
                                   (7, 128, 64), (130, 256, 320), (300, 512, 704), (257, 192, 576)])
def test_edge_shapes_and_values(P, M, K, N):
    X, smooth, g_a = _edge_activations(M, K, seed=M * 7 + K)
    rng = np.random.default_rng(K + N)
    R = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    R[N // 2] = 0.0                                                        # a zero weight row
    L1 = synth.to_bf16(rng.standard_normal((K, 32)) * 0.1)
    L2 = synth.to_bf16(rng.standard_normal((32, N)) * 0.1)
    b = synth.to_bf16(rng.standard_normal(N) * 0.01)
    blob, gw = P.svdq_pack_weights(R, synth.bf16_bits(L1), synth.bf16_bits(L2), synth.bf16_bits(b),
                                   synth.bf16_bits(smooth))
    packed = torch.from_numpy(blob).cuda()
    codes, scales, U, Y = _run_svdq(P, X, smooth, packed, g_a, gw, N)
    _check_act(codes, scales, U, X, smooth, L1, g_a)
    check_output(Y, svdq.forward(X, smooth, R, L1, L2, b, g_a))


def test_no_bias_and_empty_batch(P):
    w = synth.svdq_workload(96, 256, 128, with_bias=False)
    packed, gw = _pack(P, w, with_bias=False)
    *_, Y = _run_svdq(P, w.X, w.smooth_inv, packed, w.g_a, gw, 128)
    check_output(Y, svdq.forward(w.X, w.smooth_inv, w.R, w.L1, w.L2, None, w.g_a))
    # M == 0: a valid empty call
    Xd = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    codes, scales, U = P.svdq_quantize_act_lowrank_down(Xd, _bf16_dev(w.smooth_inv), packed, w.g_a)
    Y0 = P.svdq_w4a4_nvfp4_linear(codes, scales, U, w.g_a, packed, gw, 0, 128, 256)
    assert Y0.shape == (0, 128)


def test_repeat_calls_are_deterministic(P):
    w = synth.svdq_workload(384, 1024, 512)
    packed, gw = _pack(P, w)
    a = _run_svdq(P, w.X, w.smooth_inv, packed, w.g_a, gw, 512)
    b = _run_svdq(P, w.X, w.smooth_inv, packed, w.g_a, gw, 512)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


# ---------------------------------------------------------------- full-size layers (sampled outputs)

def sample_rows(M, seed, extra=128):
    """Rows of a full-size output to check against the oracle: one random row from every
    128-row half of every 256-row M tile (each CTA of a pair, each tile), the last row (the M
    tail), and `extra` more random rows."""
    rng = np.random.default_rng(seed)
    rows = {int(rng.integers(lo, min(M, lo + 128))) for lo in range(0, M, 128)}
    rows.add(M - 1)
    rows.update(int(r) for r in rng.choice(M, size=min(M, extra), replace=False))
    return np.array(sorted(rows))


FULL = [
    ("attention 4096x3072->3072", 4096, 3072, 3072, False),
    ("mlp-up 4608x3072->12288", 4608, 3072, 12288, False),
    ("mlp-down 4608x12288->3072 (gelu)", 4608, 12288, 3072, True),
    ("qkv 64x3072->9216", 64, 3072, 9216, False),
    ("qkv 256x3072->9216", 256, 3072, 9216, False),
    ("qkv 1024x3072->9216", 1024, 3072, 9216, False),
    ("qkv 4608x3072->9216", 4608, 3072, 9216, False),
    ("qkv 18432x3072->9216", 18432, 3072, 9216, False),
    # N not a multiple of 256: 192- and 128-wide output tiles, several per CTA pair
    ("192-wide tiles 8192x1024->1152", 8192, 1024, 1152, False),
    ("128-wide tiles 8192x512->640", 8192, 512, 640, False),
]


@pytest.mark.parametrize("name,M,K,N,gelu", FULL, ids=[f[0] for f in FULL])
def test_full_size_layer(P, name, M, K, N, gelu):
    w = synth.svdq_workload(M, K, N, gelu_input=gelu)
    packed, gw = _pack(P, w)
    codes, scales, U, Y = _run_svdq(P, w.X, w.smooth_inv, packed, w.g_a, gw, N)
    rows = sample_rows(M, 11)
    # activation codes and scales: every row (bit-exact), low-rank on the sampled rows
    cx, sx = svdq.quantize_activations(w.X, w.smooth_inv, w.g_a)
    assert np.array_equal(codes, nvfp4.pack_nibbles(cx))
    assert np.array_equal(unswizzle(scales, (M + 127) // 128 * 128, K)[:M], sx)
    Xh = svdq.smooth(w.X[rows], w.smooth_inv)
    U_ref = Xh @ w.L1.astype(np.float64)
    assert np.all(np.abs(U[rows] - U_ref) <= 1e-5 * (np.abs(Xh) @ np.abs(w.L1.astype(np.float64)))
                  + 2.0 ** -15 * np.abs(U_ref) + 1e-30)
    y_ref = svdq.forward(w.X[rows], w.smooth_inv, w.R, w.L1, w.L2, w.bias, w.g_a)
    check_output(Y[rows], y_ref)
    assert P.svdq_device_status() == 0


# ---------------------------------------------------------------- fused QKV epilogue (RMSNorm + RoPE)

def rope_tables(M, D):
    """fp32 cos / sin tables [M, D/2]: token m at position m, pair i at the inverse frequency
    10000^(-i / (D/2)) (the usual one-axis scheme; the kernel takes any tables)."""
    ang = np.arange(M, dtype=np.float64)[:, None] * 10000.0 ** (-np.arange(D // 2) / (D // 2))[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


QKV = [
    ("3 heads, 128-wide tiles, M tail 300x512->1152", 300, 512, 3),
    ("2 heads, 256-wide tiles 8192x256->768", 8192, 256, 2),
    ("qkv 64x3072->9216 (24 heads)", 64, 3072, 24),
    ("qkv 4608x3072->9216 (24 heads)", 4608, 3072, 24),
]


@pytest.mark.parametrize("name,M,K,heads", QKV, ids=[q[0] for q in QKV])
def test_qkv_rmsnorm_rope_epilogue(P, name, M, K, heads):
    from oracle import qkv_epilogue as E
    D, eps = 128, 1e-6
    N = 3 * heads * D
    w = synth.svdq_workload(M, K, N)
    packed, gw = _pack(P, w)
    codes, scales, U = P.svdq_quantize_act_lowrank_down(_bf16_dev(w.X), _bf16_dev(w.smooth_inv), packed, w.g_a)
    rng = np.random.default_rng(heads + M)
    wq = synth.to_bf16(1.0 + 0.2 * rng.standard_normal(D))
    wk = synth.to_bf16(1.0 + 0.2 * rng.standard_normal(D))
    cos, sin = rope_tables(M, D)
    Y = P.svdq_w4a4_nvfp4_linear_qkv(codes, scales, U, w.g_a, packed, gw, M, N, K, heads, _bf16_dev(wq),
                                     _bf16_dev(wk), eps, torch.from_numpy(np.ascontiguousarray(cos.T)).cuda(),
                                     torch.from_numpy(np.ascontiguousarray(sin.T)).cuda())
    torch.cuda.synchronize()
    Yg = Y.float().cpu().numpy()
    rows = sample_rows(M, 21)
    y_ref = svdq.forward(w.X[rows], w.smooth_inv, w.R, w.L1, w.L2, w.bias, w.g_a)
    q, k, v = E.qkv_epilogue(y_ref, heads, wq, wk, eps, cos[rows].astype(np.float64), sin[rows].astype(np.float64))
    HD = heads * D
    r = len(rows)
    check_output(Yg[rows, :HD], q.reshape(r, HD))
    check_output(Yg[rows, HD:2 * HD], k.reshape(r, HD))
    check_output(Yg[rows, 2 * HD:], v.reshape(r, HD))
    if heads % 2 == 0:
        # same tile width as the plain call: v is the plain layer's output bit for bit
        Yp = P.svdq_w4a4_nvfp4_linear(codes, scales, U, w.g_a, packed, gw, M, N, K)
        torch.cuda.synchronize()
        assert np.array_equal(Yp.float().cpu().numpy()[:, 2 * HD:], Yg[:, 2 * HD:])
    assert P.svdq_device_status() == 0


# ---------------------------------------------------------------- fused MLP up projection (GELU + re-quantization)

def test_gelu_table_is_the_oracle_hidden_state_of_every_bf16_value(P):
    from oracle import mlp_epilogue as E
    table = P.svdq_gelu_table_fill()
    torch.cuda.synchronize()
    got = table.cpu().numpy().view(np.uint16)
    x = synth.bf16_from_bits(np.arange(65536, dtype=np.uint32).astype(np.uint16)).astype(np.float64)
    with np.errstate(invalid="ignore", over="ignore"):
        ref = E.hidden_state(x)
    ref_bits = (ref.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(synth.bf16_from_bits(got)), nan)
    assert np.array_equal(got[~nan], ref_bits[~nan]), np.argwhere(got[~nan] != ref_bits[~nan])[:5]


MLP = [
    ("tiny 300x256->512, down ->256", 300, 256, 512, 256),
    ("M tail and row blocks over pairs 1000x512->1536, down ->384", 1000, 512, 1536, 384),
    ("mlp 4608x3072->12288, down ->3072", 4608, 3072, 12288, 3072),
]


@pytest.mark.parametrize("name,M,K,F,Nd", MLP, ids=[c[0] for c in MLP])
def test_mlp_up_gelu_requantize_epilogue(P, name, M, K, F, Nd):
    from oracle import mlp_epilogue as E
    up = synth.svdq_workload(M, K, F)
    dn = synth.svdq_workload(min(M, 512), F, Nd, gelu_input=True)   # the down layer; its X only calibrates
    pu, gwu = _pack(P, up)
    pd, gwd = _pack(P, dn)
    g_dn = dn.g_a
    codes, scales, U = P.svdq_quantize_act_lowrank_down(_bf16_dev(up.X), _bf16_dev(up.smooth_inv), pu, up.g_a)
    sd = _bf16_dev(dn.smooth_inv)
    h = torch.empty((M, F), dtype=torch.bfloat16, device="cuda")
    c1, s1, u1 = P.svdq_w4a4_nvfp4_linear_gelu_quant(codes, scales, U, up.g_a, pu, gwu, M, F, K, sd, pd, g_dn,
                                                     h_out=h)
    c2, s2, u2 = P.svdq_w4a4_nvfp4_linear_gelu_quant(codes, scales, U, up.g_a, pu, gwu, M, F, K, sd, pd, g_dn)
    torch.cuda.synchronize()
    hg = h.float().cpu().numpy().astype(np.float64)
    c1, s1, u1 = c1.cpu().numpy(), s1.cpu().numpy(), u1.float().cpu().numpy().astype(np.float64)
    # without the hidden-state output, and again: the same bits
    assert np.array_equal(c1, c2.cpu().numpy()) and np.array_equal(s1, s2.cpu().numpy())
    assert np.array_equal(u1, u2.float().cpu().numpy())
    # the hidden state against the oracle's (from the oracle's up projection), sampled rows
    rows = sample_rows(M, 31)
    y_ref = svdq.forward(up.X[rows], up.smooth_inv, up.R, up.L1, up.L2, up.bias, up.g_a)
    check_output(hg[rows], E.hidden_state(y_ref))
    # the down projection's activation pass on this h: codes and scales bit for bit, every row
    cx, sx = svdq.quantize_activations(hg, dn.smooth_inv, g_dn)
    assert np.array_equal(c1, nvfp4.pack_nibbles(cx)), np.argwhere(c1 != nvfp4.pack_nibbles(cx))[:5]
    sg = unswizzle(s1, (M + 127) // 128 * 128, F)
    assert np.array_equal(sg[:M], sx), np.argwhere(sg[:M] != sx)[:5]
    assert np.all(sg[M:] == 0)
    # U = h_hat L1 within fp32 accumulation (over the pairs' partials) and the hi + lo split
    Hh = svdq.smooth(hg, dn.smooth_inv)
    L1 = dn.L1.astype(np.float64)
    U_ref = Hh @ L1
    Ug = g_dn * (u1[:, :32] + u1[:, 32:])
    bound = 2e-5 * (np.abs(Hh) @ np.abs(L1)) + 2.0 ** -15 * np.abs(U_ref) + 1e-30
    assert np.all(np.abs(Ug - U_ref) <= bound), np.max(np.abs(Ug - U_ref) / bound)
    # and the down projection run on them against the oracle's down projection of this h
    Yd = P.svdq_w4a4_nvfp4_linear(torch.from_numpy(c1).cuda(), torch.from_numpy(s1).cuda(),
                                  torch.from_numpy(u1.astype(np.float32)).to(torch.bfloat16).cuda(), g_dn, pd, gwd,
                                  M, Nd, F)
    torch.cuda.synchronize()
    check_output(Yd.float().cpu().numpy()[rows], svdq.forward(hg[rows], dn.smooth_inv, dn.R, dn.L1, dn.L2, dn.bias, g_dn))
    assert P.svdq_device_status() == 0


def test_mlp_up_hidden_state_of_every_finite_bf16_value(P):
    """The fused epilogue's GELU (a shared-memory window of the table plus its closed forms
    outside it) over every finite bf16 pre-activation: X = 0 makes the up projection's
    accumulator zero, so y is the bias, which runs through all finite bf16 patterns (-0 comes out
    as +0 from the fma)."""
    import dataclasses
    from oracle import mlp_epilogue as E
    M, K, F, Nd = 1, 256, 65536, 128
    up = synth.svdq_workload(M, K, F, seed=3)
    pat = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    bias = synth.bf16_from_bits(pat).astype(np.float32)
    bias[~np.isfinite(bias)] = 0.0
    up = dataclasses.replace(up, X=np.zeros((M, K), np.float32), bias=bias)
    dn = synth.svdq_workload(M, F, Nd, seed=4, gelu_input=True)
    pu, gwu = _pack(P, up)
    pd, _ = _pack(P, dn)
    codes, scales, U = P.svdq_quantize_act_lowrank_down(_bf16_dev(up.X), _bf16_dev(up.smooth_inv), pu, up.g_a)
    h = torch.empty((M, F), dtype=torch.bfloat16, device="cuda")
    P.svdq_w4a4_nvfp4_linear_gelu_quant(codes, scales, U, up.g_a, pu, gwu, M, F, K, _bf16_dev(dn.smooth_inv), pd,
                                        dn.g_a, h_out=h)
    torch.cuda.synchronize()
    got = h.cpu().view(torch.int16).numpy().view(np.uint16)[0]
    y = bias.astype(np.float64) + 0.0                  # -0 + 0 = +0, as the fma gives
    ref = E.hidden_state(y)
    ref_bits = (ref.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(got, ref_bits), [(hex(pat[i]), hex(got[i]), hex(ref_bits[i]))
                                          for i in np.argwhere(got != ref_bits)[:5, 0]]
    assert P.svdq_device_status() == 0


# ---------------------------------------------------------------- SVDQ W4A4, int4 / group 64

INT4 = [
    ("tiny 256x512->512", 256, 512, 512),
    ("M tail and an odd group count 300x320->384", 300, 320, 384),
    ("attention 4096x3072->3072", 4096, 3072, 3072),
]


@pytest.mark.parametrize("name,M,K,N", INT4, ids=[c[0] for c in INT4])
def test_int4_layer(P, name, M, K, N):
    from oracle import int4 as Q
    w = synth.svdq_workload(M, K, N)
    blob = P.svdq_int4_pack_weights(w.R, synth.bf16_bits(w.L1), synth.bf16_bits(w.L2), synth.bf16_bits(w.bias),
                                    synth.bf16_bits(w.smooth_inv))
    packed = torch.from_numpy(blob).cuda()
    codes, scales, U = P.svdq_int4_quantize_act_lowrank_down(_bf16_dev(w.X), _bf16_dev(w.smooth_inv), packed)
    Y = P.svdq_w4a4_int4_linear(codes, scales, U, packed, M, N, K)
    torch.cuda.synchronize()
    # activation codes (E4M3 bytes of the integers) and bf16 scales: bit-exact, every row
    cx, sx = Q.quantize_activations(w.X, w.smooth_inv)
    vals = codes.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(vals, cx.astype(np.float64)), np.argwhere(vals != cx)[:5]
    sg = scales.float().cpu().numpy().astype(np.float64)
    assert sg.shape == (K // 64, (M + 127) // 128 * 128)
    assert np.array_equal(sg[:, :M].T, sx)
    assert np.all(sg[:, M:] == 0)
    # the low-rank activations (U = hi + lo, no per-tensor scale in this format)
    Uc = U.float().cpu().numpy().astype(np.float64)
    Ug = Uc[:, :32] + Uc[:, 32:]
    rows = sample_rows(M, 41)
    Xh = Q.smooth(w.X[rows], w.smooth_inv)
    U_ref = Xh @ w.L1.astype(np.float64)
    assert np.all(np.abs(Ug[rows] - U_ref) <= 1e-5 * (np.abs(Xh) @ np.abs(w.L1.astype(np.float64)))
                  + 2.0 ** -15 * np.abs(U_ref) + 1e-30)
    # the layer
    check_output(Y.float().cpu().numpy()[rows], Q.forward(w.X[rows], w.smooth_inv, w.R, w.L1, w.L2, w.bias))
    assert P.svdq_device_status() == 0


# ---------------------------------------------------------------- AWQ W4A16

def _run_awq(P, a, bias=None):
    X = _bf16_dev(a.X)
    qw = torch.from_numpy(a.qweight).cuda()
    s = _bf16_dev(a.scales)
    z = _bf16_dev(a.zeros)
    bd = _bf16_dev(bias) if bias is not None else None
    Y = P.awq_w4a16_linear(X, qw, s, z, bd)
    torch.cuda.synchronize()
    return Y.float().cpu().numpy()


# M <= 8: the mma.sync kernel; M >= 9: the tcgen05 kernel with 16, 32 or 64 token columns (and,
# past 64 tokens, one row of CTAs per 64-token tile, the last one ragged); K % 64 == 0 with a
# partial last 256-K stage (K = 64, 320, 448, 832)
@pytest.mark.parametrize("M,K,N", [(1, 256, 64), (3, 512, 128), (8, 768, 192), (2, 1024, 320), (7, 1536, 192),
                                   (9, 256, 64), (12, 512, 192),
                                   (16, 1024, 256), (24, 1024, 384), (33, 512, 320), (48, 768, 448),
                                   (64, 256, 128), (64, 1536, 512),
                                   (1, 64, 64), (5, 320, 128), (8, 832, 192), (20, 448, 256), (64, 320, 128),
                                   (65, 512, 128), (100, 320, 192), (200, 1024, 256), (129, 64, 64)])
def test_awq_shapes(P, M, K, N):
    a = synth.awq_workload(M, K, N, seed=M + K)
    b = synth.to_bf16(np.random.default_rng(N).standard_normal(N) * 0.1) if M % 2 else None
    Y = _run_awq(P, a, b)
    check_output(Y, oawq.forward(a.X, a.q, a.scales, a.zeros, b))


@pytest.mark.parametrize("M,K", [(5, 512), (40, 512), (6, 2048), (3, 320), (70, 448)])
def test_awq_integer_case_is_exact(P, M, K):
    # s = 1, z = 8, small integer activations: every partial sum is an exact integer in fp32
    rng = np.random.default_rng(3)
    N = 128
    a = synth.awq_workload(M, K, N)
    a.X[:] = rng.integers(-4, 5, size=(M, K))
    a.scales[:] = 1.0
    a.zeros[:] = 8.0
    Y = _run_awq(P, a)
    ref = a.X.astype(np.int64) @ (a.q.astype(np.int64) - 8).T
    assert np.array_equal(Y, synth.to_bf16(ref.astype(np.float64)))


@pytest.mark.parametrize("M,K,N", [(1, 1024, 192), (8, 3072, 320), (5, 4096, 128), (4, 4608, 128),
                                   (16, 1024, 192), (40, 3072, 128), (70, 2048, 64)])
def test_awq_scale_paths_agree(P, M, K, N):
    # both AWQ kernels read the scale and zero rows from shared memory when K % 512 == 0, K <= 4096
    # and both are 16-byte aligned, else from global memory (8-byte loads of four groups when 8-byte
    # aligned, 2-byte loads otherwise): the same values in the same order, so the outputs are
    # bit-identical
    a = synth.awq_workload(M, K, N, seed=K + N)
    X = _bf16_dev(a.X)
    qw = torch.from_numpy(a.qweight).cuda()
    outs = []
    for off in (0, 4, 1):                          # elements: 16-, 8- and 2-byte aligned copies
        sb = torch.zeros((a.scales.size + 8,), dtype=torch.bfloat16, device="cuda")
        zb = torch.zeros_like(sb)
        s = sb[off:off + a.scales.size].view(a.scales.shape)
        z = zb[off:off + a.zeros.size].view(a.zeros.shape)
        s.copy_(_bf16_dev(a.scales))
        z.copy_(_bf16_dev(a.zeros))
        outs.append(P.awq_w4a16_linear(X, qw, s, z))
    torch.cuda.synchronize()
    assert P.svdq_device_status() == 0
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
    check_output(outs[0].float().cpu().numpy(), oawq.forward(a.X, a.q, a.scales, a.zeros, None))


@pytest.fixture(scope="module")
def awq_full():
    a = synth.awq_workload(64, 3072, 18432)
    deq = oawq.dequantize(a.q, a.scales, a.zeros)
    return a, deq


@pytest.mark.parametrize("M", [1, 2, 4, 8, 12, 16, 32, 64])
def test_awq_adaln_full_size(P, awq_full, M):
    a, deq = awq_full
    sub = synth.AwqWorkload(M, a.K, a.N, a.X[:M].copy(), a.q, a.qweight, a.scales, a.zeros, a.W)
    Y = _run_awq(P, sub)
    check_output(Y, a.X[:M].astype(np.float64) @ deq.T)
    assert P.svdq_device_status() == 0


# ---------------------------------------------------------------- dynamic activation scale (kernel 5)

def _run_svdq_dyn(P, X, smooth, packed, g_w, N):
    M, K = X.shape
    Xd, sd = _bf16_dev(X), _bf16_dev(smooth)
    amax = P.svdq_act_amax(Xd, sd)
    codes, scales, U = P.svdq_quantize_act_lowrank_down_dyn(Xd, sd, packed, amax)
    Y = P.svdq_w4a4_nvfp4_linear_dyn(codes, scales, U, amax, packed, g_w, M, N, K)
    torch.cuda.synchronize()
    words = amax.cpu()
    assert words[1] == 0 and words[2] == 0                              # left clean for the next call
    a = float(words[:1].view(torch.float32).item())
    return a, codes, scales, U, Y


def test_dynamic_scale_amax_is_exact_and_layer_matches_the_oracle(P):
    w = synth.svdq_workload(256, 512, 512)
    packed, gw = _pack(P, w)
    a, codes, scales, U, Y = _run_svdq_dyn(P, w.X, w.smooth_inv, packed, gw, 512)
    assert a == np.max(np.abs(svdq.smooth(w.X, w.smooth_inv)))          # bit-exact amax
    g = svdq.dynamic_act_scale(w.X, w.smooth_inv)
    Uc = U.float().cpu().numpy().astype(np.float64)
    _check_act(codes.cpu().numpy(), scales.cpu().numpy(), g * (Uc[:, :32] + Uc[:, 32:]), w.X, w.smooth_inv, w.L1, g)
    check_output(Y.float().cpu().numpy(), svdq.forward(w.X, w.smooth_inv, w.R, w.L1, w.L2, w.bias, g))
    # the same kernels with that scale passed in: identical outputs
    cs, ss, us, ys = _run_svdq(P, w.X, w.smooth_inv, packed, g, gw, 512)
    assert np.array_equal(cs, codes.cpu().numpy()) and np.array_equal(ss, scales.cpu().numpy())
    assert np.array_equal(ys, Y.float().cpu().numpy())
    assert P.svdq_device_status() == 0


@pytest.mark.parametrize("factor", [0.0, 2.0 ** 12, 2.0 ** -9])
def test_dynamic_scale_zero_and_extreme_batches(P, factor):
    w = synth.svdq_workload(128, 256, 256)
    packed, gw = _pack(P, w)
    X = synth.to_bf16(w.X * factor)
    a, codes, scales, U, Y = _run_svdq_dyn(P, X, w.smooth_inv, packed, gw, 256)
    g = svdq.dynamic_act_scale(X, w.smooth_inv)
    assert a == np.max(np.abs(svdq.smooth(X, w.smooth_inv)))
    cx, sx = svdq.quantize_activations(X, w.smooth_inv, g)
    assert np.array_equal(codes.cpu().numpy(), nvfp4.pack_nibbles(cx))
    assert np.array_equal(unswizzle(scales.cpu().numpy(), 128, 256)[:128], sx)
    check_output(Y.float().cpu().numpy(), svdq.forward(X, w.smooth_inv, w.R, w.L1, w.L2, w.bias, g))


def test_dynamic_scale_full_attention_layer(P):
    M, K, N = 4096, 3072, 3072
    w = synth.svdq_workload(M, K, N)
    packed, gw = _pack(P, w)
    a, codes, scales, U, Y = _run_svdq_dyn(P, w.X, w.smooth_inv, packed, gw, N)
    assert a == np.max(np.abs(svdq.smooth(w.X, w.smooth_inv)))
    g = svdq.dynamic_act_scale(w.X, w.smooth_inv)
    cx, sx = svdq.quantize_activations(w.X, w.smooth_inv, g)
    assert np.array_equal(codes.cpu().numpy(), nvfp4.pack_nibbles(cx))
    assert np.array_equal(unswizzle(scales.cpu().numpy(), M, K)[:M], sx)
    rows = sample_rows(M, 12)
    check_output(Y.float().cpu().numpy()[rows],
                 svdq.forward(w.X[rows], w.smooth_inv, w.R, w.L1, w.L2, w.bias, g))
    assert P.svdq_device_status() == 0


def test_dynamic_scale_product_out_of_range_is_clamped_and_reported(P):
    # g_a g_w formed on the device above 2^126: the GEMM clamps it and records the range status
    # (the static call refuses such a product on the host).  X holds one 2^127 (amax = 2^127,
    # g_a = 2^116) and R values near 2^22 (g_w = 2^11): the product is 2^127.
    rng = np.random.default_rng(5)
    M, K, N = 128, 256, 128
    X = synth.to_bf16(rng.standard_normal((M, K)))
    X[3, 17] = 2.0 ** 127
    smooth = np.ones(K, np.float32)
    R = (rng.standard_normal((N, K)) * 2.0 ** 20).astype(np.float32)
    L1 = np.zeros((K, 32), np.float32)
    L2 = np.zeros((32, N), np.float32)
    blob, gw = P.svdq_pack_weights(R, synth.bf16_bits(L1), synth.bf16_bits(L2), None, synth.bf16_bits(smooth))
    assert gw == 2.0 ** 11
    assert P.svdq_device_status() == 0
    a, *_ = _run_svdq_dyn(P, X, smooth, torch.from_numpy(blob).cuda(), gw, N)
    assert a == 2.0 ** 127
    assert P.svdq_device_status(clear=True) == 6
    assert P.svdq_device_status() == 0                                  # cleared
    with pytest.raises(P.SvdqError):                                    # the static call refuses it
        P.svdq_w4a4_nvfp4_linear(*P.svdq_quantize_act_lowrank_down(_bf16_dev(X), _bf16_dev(smooth),
                                                                   torch.from_numpy(blob).cuda(), 2.0 ** 116),
                                 2.0 ** 116, torch.from_numpy(blob).cuda(), gw, M, N, K)
    # an in-range batch afterwards runs clean
    w = synth.svdq_workload(128, 256, 256)
    packed, gw2 = _pack(P, w)
    _run_svdq_dyn(P, w.X, w.smooth_inv, packed, gw2, 256)
    assert P.svdq_device_status() == 0


def test_dynamic_scale_buffer_is_reused_cleanly_eager_and_in_graphs(P):
    w = synth.svdq_workload(128, 256, 256)
    s = _bf16_dev(w.smooth_inv)
    buf = torch.zeros(4, dtype=torch.int32, device="cuda")
    big, small = synth.to_bf16(w.X * 64.0), w.X

    def amax_ref(X):
        return np.max(np.abs(svdq.smooth(X, w.smooth_inv)))

    def read():
        torch.cuda.synchronize()
        words = buf.cpu()
        assert words[1] == 0 and words[2] == 0
        return float(words[:1].view(torch.float32).item())

    for X in (big, small, big, small):                     # a smaller batch after a larger one
        P.svdq_act_amax(_bf16_dev(X), s, buf)
        assert read() == amax_ref(X)
    Xg = _bf16_dev(big)
    g = torch.cuda.CUDAGraph()
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        P.svdq_act_amax(Xg, s, buf)                         # warm-up on the capture stream
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=stream):
        P.svdq_act_amax(Xg, s, buf)
    for X in (big, small, big):
        Xg.copy_(_bf16_dev(X))
        g.replay()
        assert read() == amax_ref(X)
