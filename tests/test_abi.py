"""The C-ABI library loads, exports every declared symbol, and checks its arguments
(host-side logic only; no kernel runs here)."""

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

import bit_diffusion_transformer_act_b200 as P  # noqa: E402  (conftest has built the library)

from parity_util import swizzled_offset, unswizzle  # noqa: E402

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "svdq.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)) - {"if"}


def test_header_declares_the_expected_entry_points():
    decl = _declared_functions()
    for name in ("svdq_pack_weights", "svdq_quantize_act_lowrank_down", "svdq_w4a4_nvfp4_linear",
                 "awq_w4a16_linear"):
        assert name in decl
    assert decl == set(P.EXPORTED)


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", P.ops.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in _declared_functions():
        assert name in exported, name
        assert getattr(P.LIB, name) is not None


def test_status_strings_and_version():
    for s in range(7):
        assert P.LIB.svdq_status_string(s)
    assert P.LIB.svdq_status_string(99) == b"unknown status"
    assert P.LIB.svdq_abi_version() == 2


def test_sizes():
    assert P.svdq_packed_weight_bytes(3072, 3072) > 3072 * 1536
    assert P.svdq_packed_weight_bytes(100, 3072) == 0          # N % 64
    assert P.svdq_packed_weight_bytes(320, 3072) > 0           # N % 64 == 0 with N % 128 == 64
    assert P.svdq_packed_weight_bytes(128, 100) == 0           # K % 64
    assert P.svdq_packed_weight_bytes(128, 64, 16) == 0        # rank
    assert P.svdq_act_scale_bytes(1, 64) == 128 * 4
    assert P.svdq_act_scale_bytes(129, 128) == 256 * 8
    assert P.svdq_act_scale_bytes(0, 64) == 0


FAKE = ctypes.c_void_p(1 << 20)       # aligned, never dereferenced: every case below fails its checks first


def test_gpu_entry_points_reject_bad_arguments_before_any_device_work():
    L = P.LIB
    # null pointers
    assert L.svdq_quantize_act_lowrank_down(None, FAKE, FAKE, 4, 64, 32, 1.0, FAKE, FAKE, FAKE, None) == 1
    assert L.svdq_w4a4_nvfp4_linear(FAKE, FAKE, None, 1.0, FAKE, 1.0, 4, 128, 64, 32, FAKE, None) == 1
    assert L.awq_w4a16_linear(FAKE, FAKE, FAKE, FAKE, None, 4, 64, 256, None, None) == 1
    # scales that are not powers of two
    assert L.svdq_quantize_act_lowrank_down(FAKE, FAKE, FAKE, 4, 64, 32, 0.3, FAKE, FAKE, FAKE, None) == 1
    assert L.svdq_w4a4_nvfp4_linear(FAKE, FAKE, FAKE, 1.0, FAKE, -2.0, 4, 128, 64, 32, FAKE, None) == 1
    # unsupported shapes
    assert L.svdq_quantize_act_lowrank_down(FAKE, FAKE, FAKE, 4, 96, 32, 1.0, FAKE, FAKE, FAKE, None) == 2
    assert L.svdq_quantize_act_lowrank_down(FAKE, FAKE, FAKE, 4, 64, 16, 1.0, FAKE, FAKE, FAKE, None) == 2
    assert L.svdq_w4a4_nvfp4_linear(FAKE, FAKE, FAKE, 1.0, FAKE, 1.0, 4, 96, 64, 32, FAKE, None) == 2
    assert L.awq_w4a16_linear(FAKE, FAKE, FAKE, FAKE, None, 65, 96, 256, FAKE, None) == 2      # N % 64
    assert L.awq_w4a16_linear(FAKE, FAKE, FAKE, FAKE, None, 4, 64, 96, FAKE, None) == 2        # K % 64
    # misaligned pointers
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert L.svdq_quantize_act_lowrank_down(odd, FAKE, FAKE, 4, 64, 32, 1.0, FAKE, FAKE, FAKE, None) == 1
    assert L.svdq_w4a4_nvfp4_linear(FAKE, FAKE, FAKE, 1.0, FAKE, 1.0, 4, 128, 64, 32, odd, None) == 1
    odd2 = ctypes.c_void_p((1 << 20) + 1)
    assert L.awq_w4a16_linear(FAKE, FAKE, odd2, FAKE, None, 4, 64, 320, FAKE, None) == 1     # scales
    # negative sizes
    assert L.svdq_quantize_act_lowrank_down(FAKE, FAKE, FAKE, -1, 64, 32, 1.0, FAKE, FAKE, FAKE, None) == 1
    # an empty batch is valid even with null buffers, and needs no device
    assert L.svdq_quantize_act_lowrank_down(None, None, None, 0, 64, 32, 1.0, None, None, None, None) == 0
    assert L.svdq_w4a4_nvfp4_linear(None, None, None, 1.0, None, 1.0, 0, 128, 64, 32, None, None) == 0
    assert L.awq_w4a16_linear(None, None, None, None, None, 0, 64, 256, None, None) == 0


def test_qkv_entry_point_rejects_bad_arguments_before_any_device_work():
    L = P.LIB
    odd = ctypes.c_void_p((1 << 20) + 8)

    def qkv(M=4, N=768, K=64, heads=2, D=128, eps=1e-6, wq=FAKE, cos=FAKE):
        return L.svdq_w4a4_nvfp4_linear_qkv(FAKE, FAKE, FAKE, 1.0, FAKE, 1.0, M, N, K, 32, heads, D, wq, FAKE,
                                            eps, cos, FAKE, FAKE, None)
    assert qkv(D=64, N=384) == 2                       # head_dim 128 only
    assert qkv(N=640) == 2                             # N = 3 heads head_dim
    assert qkv(heads=0) == 1
    assert qkv(eps=-1.0) == 1
    assert qkv(eps=float("inf")) == 1
    assert qkv(wq=None) == 1
    assert qkv(cos=odd) == 1
    assert qkv(K=96) == 2                              # the plain call's checks follow
    assert qkv(M=0, wq=None, cos=None) == 0            # an empty batch needs neither tables nor a device


def test_gelu_quant_entry_point_rejects_bad_arguments_before_any_device_work():
    L = P.LIB

    def call(M=4, N=256, K=64, g=1.0, gd=1.0, ws=FAKE, wsb=1 << 30, h=None, codes=FAKE, table=FAKE):
        return L.svdq_w4a4_nvfp4_linear_gelu_quant(FAKE, FAKE, FAKE, g, FAKE, 1.0, M, N, K, 32, FAKE, FAKE, gd,
                                                   codes, FAKE, FAKE, ws, wsb, table, h, None)
    assert call(N=96) == 2 and call(N=192) == 2         # N % 128 (the fused epilogue's tiles)
    assert call(K=96) == 2
    assert call(g=0.3) == 1 and call(gd=3.0) == 1       # scales must be powers of two
    assert call(ws=None) == 1 and call(codes=None) == 1 and call(table=None) == 1
    assert call(table=ctypes.c_void_p((1 << 20) + 2)) == 1
    assert call(h=ctypes.c_void_p((1 << 20) + 8)) == 1  # misaligned optional output
    assert call(M=-1) == 1
    assert call(M=0, ws=None, codes=None) == 0          # empty batch: nothing needed
    assert P.svdq_gelu_quant_workspace_bytes(4, 200) == 0
    assert P.LIB.svdq_gelu_table_bytes() == 131072
    assert L.svdq_gelu_table_fill(None, None) == 1


def test_int4_entry_points_reject_bad_arguments_before_any_device_work():
    L = P.LIB
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert L.svdq_int4_packed_weight_bytes(128, 64, 32) > 0
    assert L.svdq_int4_packed_weight_bytes(100, 64, 32) == 0 and L.svdq_int4_packed_weight_bytes(128, 96, 32) == 0
    assert L.svdq_int4_quantize_act_lowrank_down(None, FAKE, FAKE, 4, 64, 32, FAKE, FAKE, FAKE, None) == 1
    assert L.svdq_int4_quantize_act_lowrank_down(FAKE, FAKE, FAKE, 4, 96, 32, FAKE, FAKE, FAKE, None) == 2
    assert L.svdq_int4_quantize_act_lowrank_down(odd, FAKE, FAKE, 4, 64, 32, FAKE, FAKE, FAKE, None) == 1
    assert L.svdq_w4a4_int4_linear(FAKE, FAKE, FAKE, FAKE, 4, 192, 64, 32, FAKE, None) == 2
    assert L.svdq_w4a4_int4_linear(FAKE, FAKE, FAKE, FAKE, 4, 128, 64, 16, FAKE, None) == 2
    assert L.svdq_w4a4_int4_linear(FAKE, None, FAKE, FAKE, 4, 128, 64, 32, FAKE, None) == 1
    assert L.svdq_w4a4_int4_linear(FAKE, FAKE, FAKE, FAKE, 4, 128, 64, 32, odd, None) == 1
    assert L.svdq_w4a4_int4_linear(None, None, None, None, 0, 128, 64, 32, None, None) == 0


def test_dynamic_scale_entry_points_reject_bad_arguments_before_any_device_work():
    L = P.LIB
    odd2 = ctypes.c_void_p((1 << 20) + 2)
    odd8 = ctypes.c_void_p((1 << 20) + 8)
    # svdq_act_amax: the 16-byte amax buffer, K % 64, M >= 0, inputs present when M > 0
    assert L.svdq_act_amax(FAKE, FAKE, 4, 64, None, None) == 1
    assert L.svdq_act_amax(FAKE, FAKE, 4, 64, odd8, None) == 1
    assert L.svdq_act_amax(FAKE, FAKE, 4, 96, FAKE, None) == 1
    assert L.svdq_act_amax(FAKE, FAKE, -1, 64, FAKE, None) == 1
    assert L.svdq_act_amax(None, FAKE, 4, 64, FAKE, None) == 1
    # svdq_act_amax_noalloc: a 4-byte-aligned result word, the same size and input checks
    assert L.svdq_act_amax_noalloc(FAKE, FAKE, 4, 64, None, None) == 1
    assert L.svdq_act_amax_noalloc(FAKE, FAKE, 4, 64, odd2, None) == 1
    assert L.svdq_act_amax_noalloc(FAKE, FAKE, 4, 96, FAKE, None) == 1
    assert L.svdq_act_amax_noalloc(FAKE, FAKE, -1, 64, FAKE, None) == 1
    assert L.svdq_act_amax_noalloc(None, FAKE, 4, 64, FAKE, None) == 1
    assert L.svdq_act_amax_noalloc(FAKE, odd8, 4, 64, FAKE, None) == 1
    # the *_dyn calls need the amax word (4-byte aligned); the static calls' checks apply otherwise
    assert L.svdq_quantize_act_lowrank_down_dyn(FAKE, FAKE, FAKE, 4, 64, 32, None, FAKE, FAKE, FAKE, None) == 1
    assert L.svdq_quantize_act_lowrank_down_dyn(FAKE, FAKE, FAKE, 4, 64, 32, odd2, FAKE, FAKE, FAKE, None) == 1
    assert L.svdq_quantize_act_lowrank_down_dyn(FAKE, FAKE, FAKE, 4, 96, 32, FAKE, FAKE, FAKE, FAKE, None) == 2
    assert L.svdq_w4a4_nvfp4_linear_dyn(FAKE, FAKE, FAKE, None, FAKE, 1.0, 4, 128, 64, 32, FAKE, None) == 1
    assert L.svdq_w4a4_nvfp4_linear_dyn(FAKE, FAKE, FAKE, FAKE, FAKE, 0.3, 4, 128, 64, 32, FAKE, None) == 1
    assert L.svdq_w4a4_nvfp4_linear_dyn(FAKE, FAKE, FAKE, FAKE, FAKE, 1.0, 4, 96, 64, 32, FAKE, None) == 2
    # an empty batch is valid and needs no device
    assert L.svdq_quantize_act_lowrank_down_dyn(None, None, None, 0, 64, 32, FAKE, None, None, None, None) == 0
    assert L.svdq_w4a4_nvfp4_linear_dyn(None, None, None, FAKE, None, 1.0, 0, 128, 64, 32, None, None) == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_a_device_reports_a_cuda_error():
    assert P.LIB.svdq_quantize_act_lowrank_down(FAKE, FAKE, FAKE, 4, 64, 32, 1.0, FAKE, FAKE, FAKE, None) == 4


def test_swizzle_helpers_follow_the_documented_layout():
    rng = np.random.default_rng(0)
    for rows, K in [(1, 64), (130, 192), (256, 512)]:
        plain = rng.integers(0, 256, size=(rows, K // 16)).astype(np.uint8)
        sw = P.svdq_swizzle_scales(plain, rows, K)
        assert sw.size == P.svdq_act_scale_bytes(rows, K)
        assert np.array_equal(unswizzle(sw, rows, K), plain)
        assert np.array_equal(P.svdq_unswizzle_scales(sw, rows, K), plain)
    # one byte placed by hand: row 37 (lane 5 of quarter 1), group 6 (atom 1, slot 2), K = 128
    assert swizzled_offset(37, 6, 128) == 512 + 5 * 16 + 1 * 4 + 2


def test_python_wrappers_refuse_host_tensors_before_calling_the_library():
    # device calls take raw pointers: a host tensor must never reach a kernel
    X = torch.zeros((4, 64), dtype=torch.bfloat16)
    s = torch.zeros((64,), dtype=torch.bfloat16)
    blob = torch.zeros((P.svdq_packed_weight_bytes(128, 64),), dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA tensor"):
        P.svdq_quantize_act_lowrank_down(X, s, blob, 1.0)
    with pytest.raises(ValueError, match="CUDA tensor"):
        P.svdq_act_amax(X, s)
    with pytest.raises(ValueError, match="CUDA tensor"):
        P.awq_w4a16_linear(X, torch.zeros((64, 32), dtype=torch.uint8), torch.zeros((64, 1), dtype=torch.bfloat16),
                           torch.zeros((64, 1), dtype=torch.bfloat16))
    codes = torch.zeros((4, 32), dtype=torch.uint8)
    scales = torch.zeros((P.svdq_act_scale_bytes(4, 64),), dtype=torch.uint8)
    low = torch.zeros((4, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        P.svdq_w4a4_nvfp4_linear(codes, scales, low, 1.0, blob, 1.0, 4, 128, 64)
    # the activation calls read the blob's header and low-rank section (1 KB + 4 rank K bytes):
    # a shorter blob is refused before any device call, in both the static and dynamic wrappers
    short = torch.zeros((1024 + 4 * 32 * 64 - 16,), dtype=torch.uint8)
    amax = torch.zeros((4,), dtype=torch.int32)
    with pytest.raises(ValueError, match="at least 9216 bytes"):
        P.svdq_quantize_act_lowrank_down(X, s, short, 1.0)
    with pytest.raises(ValueError, match="at least 9216 bytes"):
        P.svdq_quantize_act_lowrank_down_dyn(X, s, short, amax)
    wide = torch.zeros((4, 128), dtype=torch.bfloat16)              # K = 128 needs 17408 bytes
    with pytest.raises(ValueError, match="at least 17408 bytes"):
        P.svdq_quantize_act_lowrank_down(wide, torch.zeros((128,), dtype=torch.bfloat16), blob[:9216], 1.0)
    with pytest.raises(ValueError, match="CUDA tensor"):                # long enough: the device check follows
        P.svdq_quantize_act_lowrank_down_dyn(X, s, short[:0].new_zeros(9216), amax)
    # the guards' own checks (size and shape come before the device check)
    with pytest.raises(ValueError, match="at least"):                  # a blob too short for N, K
        P.ops._require_blob(blob[:100], "packed_w", P.svdq_packed_weight_bytes(128, 64))
    with pytest.raises(ValueError, match="expected"):                  # codes of the wrong shape
        P.ops._require(codes[:, :16], torch.uint8, (4, 32), "act_codes")
