"""Python binding of libsvdq (include/svdq.h): argument marshalling only.

Every function keeps the C name and forwards raw pointers and the current CUDA
stream of PyTorch; PyTorch only provides device memory and streams.  There is
no fallback: if the library is missing the import fails, and on a device that
is not sm_100 the calls raise.
"""

import ctypes
import os

import numpy as np
import torch

from .build import LIB_PATH

RANK = 32

_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "device is not sm_100 (B200)",
           4: "CUDA error", 5: "kernel wait timed out", 6: "device-side scale product out of range (clamped)"}


class SvdqError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {_STATUS.get(status, 'unknown')} (status {status})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libsvdq.so not built at {LIB_PATH}; run `python bit_diffusion_transformer_act_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sig = {
        "svdq_status_string": ([i], ctypes.c_char_p),
        "svdq_abi_version": ([], i),
        "svdq_packed_weight_bytes": ([i, i, i], sz),
        "svdq_pack_weights": ([vp, vp, vp, vp, vp, i, i, i, vp, sz, ctypes.POINTER(ctypes.c_float)], i),
        "svdq_act_scale_bytes": ([i, i], sz),
        "svdq_quantize_act_lowrank_down": ([vp, vp, vp, i, i, i, f, vp, vp, vp, vp], i),
        "svdq_w4a4_nvfp4_linear": ([vp, vp, vp, f, vp, f, i, i, i, i, vp, vp], i),
        "svdq_w4a4_nvfp4_linear_qkv": ([vp, vp, vp, f, vp, f, i, i, i, i, i, i, vp, vp, f, vp, vp, vp, vp], i),
        "svdq_gelu_quant_workspace_bytes": ([i, i], sz),
        "svdq_gelu_table_bytes": ([], sz),
        "svdq_int4_packed_weight_bytes": ([i, i, i], sz),
        "svdq_int4_pack_weights": ([vp, vp, vp, vp, vp, i, i, i, vp, sz], i),
        "svdq_int4_quantize_act_lowrank_down": ([vp, vp, vp, i, i, i, vp, vp, vp, vp], i),
        "svdq_w4a4_int4_linear": ([vp, vp, vp, vp, i, i, i, i, vp, vp], i),
        "svdq_gelu_table_fill": ([vp, vp], i),
        "svdq_w4a4_nvfp4_linear_gelu_quant": ([vp, vp, vp, f, vp, f, i, i, i, i, vp, vp, f, vp, vp, vp, vp, sz, vp, vp,
                                               vp], i),
        "awq_w4a16_linear": ([vp, vp, vp, vp, vp, i, i, i, vp, vp], i),
        "svdq_act_amax": ([vp, vp, i, i, vp, vp], i),
        "svdq_act_amax_noalloc": ([vp, vp, i, i, vp, vp], i),
        "svdq_quantize_act_lowrank_down_dyn": ([vp, vp, vp, i, i, i, vp, vp, vp, vp, vp], i),
        "svdq_w4a4_nvfp4_linear_dyn": ([vp, vp, vp, vp, vp, f, i, i, i, i, vp, vp], i),
        "svdq_unswizzle_scales": ([vp, i, i, vp], i),
        "svdq_swizzle_scales": ([vp, i, i, vp], i),
        "svdq_device_status": ([i], i),
        "svdq_selftest_wait_timeout": ([vp], i),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


LIB = _load()
EXPORTED = ("svdq_status_string", "svdq_abi_version", "svdq_packed_weight_bytes", "svdq_pack_weights",
            "svdq_act_scale_bytes", "svdq_quantize_act_lowrank_down", "svdq_w4a4_nvfp4_linear",
            "awq_w4a16_linear", "svdq_unswizzle_scales", "svdq_swizzle_scales", "svdq_device_status",
            "svdq_act_amax", "svdq_quantize_act_lowrank_down_dyn", "svdq_w4a4_nvfp4_linear_dyn",
            "svdq_act_amax_noalloc", "svdq_w4a4_nvfp4_linear_qkv", "svdq_gelu_quant_workspace_bytes",
            "svdq_w4a4_nvfp4_linear_gelu_quant", "svdq_selftest_wait_timeout", "svdq_gelu_table_bytes",
            "svdq_gelu_table_fill", "svdq_int4_packed_weight_bytes", "svdq_int4_pack_weights",
            "svdq_int4_quantize_act_lowrank_down", "svdq_w4a4_int4_linear")


def _check(fn, st):
    if st != 0:
        raise SvdqError(fn, st)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _np_ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _on_device(t, name):
    """Device calls take raw pointers: a host tensor (or one on another GPU) would be read as
    device memory, so it is refused here, before the call."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device.index is not None and t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}, the current device is cuda:{torch.cuda.current_device()}")


def _require(t, dtype, shape, name):
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected {dtype} tensor of shape {tuple(shape)}, got "
                         f"{getattr(t, 'dtype', type(t))} {tuple(getattr(t, 'shape', ()))}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    _on_device(t, name)


def _l1_section_end(K, rank):
    """Bytes of the packed blob that the activation kernel reads: the 1 KB header and the
    low-rank down factor section that follows it (two bf16 [rank, K] parts, hi and lo).  The C
    call has no size argument, so this is the only guard against a blob that is too short
    (or packed for a smaller K)."""
    return 1024 + 4 * rank * K


def _require_blob(t, name, min_bytes=0):
    if not isinstance(t, torch.Tensor) or t.dtype != torch.uint8 or not t.is_contiguous() or t.numel() < min_bytes:
        raise ValueError(f"{name}: expected a contiguous uint8 tensor of at least {min_bytes} bytes")
    _on_device(t, name)


# ---------------------------------------------------------------- host side

def svdq_packed_weight_bytes(N, K, rank=RANK):
    return int(LIB.svdq_packed_weight_bytes(N, K, rank))


def svdq_act_scale_bytes(M, K):
    return int(LIB.svdq_act_scale_bytes(M, K))


def svdq_pack_weights(R, L1_bits, L2_bits, bias_bits, smooth_bits):
    """R float32 [N, K]; L1 bf16 bits uint16 [K, r]; L2 bits [r, N]; bias bits [N] or None;
    smooth_inv bits [K] (the same vector later given to the activation kernel).

    Returns (blob uint8 numpy array, w_global_scale float)."""
    R = np.ascontiguousarray(R, dtype=np.float32)
    N, K = R.shape
    L1_bits = np.ascontiguousarray(L1_bits, dtype=np.uint16)
    L2_bits = np.ascontiguousarray(L2_bits, dtype=np.uint16)
    rank = L1_bits.shape[1]
    if L1_bits.shape != (K, rank) or L2_bits.shape != (rank, N):
        raise ValueError("L1 must be [K, r] and L2 [r, N]")
    if bias_bits is not None:
        bias_bits = np.ascontiguousarray(bias_bits, dtype=np.uint16)
        if bias_bits.shape != (N,):
            raise ValueError("bias must be [N]")
    smooth_bits = np.ascontiguousarray(smooth_bits, dtype=np.uint16)
    if smooth_bits.shape != (K,):
        raise ValueError("smooth_inv must be [K]")
    nbytes = svdq_packed_weight_bytes(N, K, rank)
    if nbytes == 0:
        _check("svdq_pack_weights", 2)
    out = np.empty(nbytes, dtype=np.uint8)
    g = ctypes.c_float(0.0)
    st = LIB.svdq_pack_weights(_np_ptr(R), _np_ptr(L1_bits), _np_ptr(L2_bits), _np_ptr(bias_bits),
                               _np_ptr(smooth_bits), N, K, rank, _np_ptr(out), nbytes, ctypes.byref(g))
    _check("svdq_pack_weights", st)
    return out, float(g.value)


def svdq_int4_pack_weights(R, L1_bits, L2_bits, bias_bits, smooth_bits):
    """The int4 / group-64 row's packed weights (numpy uint8 blob) of R float32 [N, K], L1 bits
    [K, r], L2 bits [r, N], bias bits [N] or None, smooth_inv bits [K]."""
    R = np.ascontiguousarray(R, dtype=np.float32)
    N, K = R.shape
    L1_bits = np.ascontiguousarray(L1_bits, dtype=np.uint16)
    L2_bits = np.ascontiguousarray(L2_bits, dtype=np.uint16)
    rank = L1_bits.shape[1]
    if L1_bits.shape != (K, rank) or L2_bits.shape != (rank, N):
        raise ValueError("L1 must be [K, r] and L2 [r, N]")
    if bias_bits is not None:
        bias_bits = np.ascontiguousarray(bias_bits, dtype=np.uint16)
        if bias_bits.shape != (N,):
            raise ValueError("bias must be [N]")
    smooth_bits = np.ascontiguousarray(smooth_bits, dtype=np.uint16)
    if smooth_bits.shape != (K,):
        raise ValueError("smooth_inv must be [K]")
    nbytes = int(LIB.svdq_int4_packed_weight_bytes(N, K, rank))
    if nbytes == 0:
        _check("svdq_int4_pack_weights", 2)
    out = np.empty(nbytes, dtype=np.uint8)
    _check("svdq_int4_pack_weights", LIB.svdq_int4_pack_weights(_np_ptr(R), _np_ptr(L1_bits), _np_ptr(L2_bits),
                                                                 _np_ptr(bias_bits), _np_ptr(smooth_bits), N, K,
                                                                 rank, _np_ptr(out), nbytes))
    return out


def svdq_unswizzle_scales(swizzled, rows, K):
    """Swizzled scale bytes (numpy uint8 or a torch tensor) -> numpy uint8 [rows, K/16]."""
    if isinstance(swizzled, torch.Tensor):
        swizzled = swizzled.detach().cpu().numpy()
    sw = np.ascontiguousarray(swizzled, dtype=np.uint8)
    out = np.empty((rows, K // 16), dtype=np.uint8)
    _check("svdq_unswizzle_scales", LIB.svdq_unswizzle_scales(_np_ptr(sw), rows, K, _np_ptr(out)))
    return out


def svdq_swizzle_scales(plain, rows, K):
    plain = np.ascontiguousarray(plain, dtype=np.uint8)
    out = np.empty(svdq_act_scale_bytes(rows, K), dtype=np.uint8)
    _check("svdq_swizzle_scales", LIB.svdq_swizzle_scales(_np_ptr(plain), rows, K, _np_ptr(out)))
    return out


def svdq_device_status(clear=True):
    """Synchronizes the device and returns the library's status word (0 or 5)."""
    return int(LIB.svdq_device_status(1 if clear else 0))


# ---------------------------------------------------------------- device side

def svdq_quantize_act_lowrank_down(X, smooth_inv, packed_w, act_global_scale, rank=RANK,
                                   act_codes=None, act_scales=None, lowrank_act=None):
    """X bf16 [M, K] cuda; smooth_inv bf16 [K]; packed_w uint8 cuda (the blob).

    Returns (act_codes uint8 [M, K/2], act_scales uint8 [svdq_act_scale_bytes],
    lowrank_act bf16 [M, 2r] holding U / g_a as a high part then a low part)."""
    M, K = X.shape
    dev = X.device
    _require_blob(packed_w, "packed_w", _l1_section_end(K, rank))
    _require(X, torch.bfloat16, (M, K), "X")
    _require(smooth_inv, torch.bfloat16, (K,), "smooth_inv")
    if act_codes is None:
        act_codes = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
    if act_scales is None:
        act_scales = torch.empty((svdq_act_scale_bytes(M, K),), dtype=torch.uint8, device=dev)
    if lowrank_act is None:
        lowrank_act = torch.empty((M, 2 * rank), dtype=torch.bfloat16, device=dev)
    _require(act_codes, torch.uint8, (M, K // 2), "act_codes")
    _require(act_scales, torch.uint8, (svdq_act_scale_bytes(M, K),), "act_scales")
    _require(lowrank_act, torch.bfloat16, (M, 2 * rank), "lowrank_act")
    st = LIB.svdq_quantize_act_lowrank_down(_ptr(X), _ptr(smooth_inv), _ptr(packed_w), M, K, rank,
                                            float(act_global_scale), _ptr(act_codes), _ptr(act_scales),
                                            _ptr(lowrank_act), _stream())
    _check("svdq_quantize_act_lowrank_down", st)
    return act_codes, act_scales, lowrank_act


def svdq_w4a4_nvfp4_linear(act_codes, act_scales, lowrank_act, act_global_scale, packed_w, w_global_scale,
                           M, N, K, rank=RANK, Y=None):
    """Returns Y bf16 [M, N] = bf16(g_a g_w Q(X_hat) Q(R)^T + lowrank_act L2 + b)."""
    _require(act_codes, torch.uint8, (M, K // 2), "act_codes")
    _require(act_scales, torch.uint8, (svdq_act_scale_bytes(M, K),), "act_scales")
    _require(lowrank_act, torch.bfloat16, (M, 2 * rank), "lowrank_act")
    _require_blob(packed_w, "packed_w", svdq_packed_weight_bytes(N, K, rank))
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=act_codes.device)
    _require(Y, torch.bfloat16, (M, N), "Y")
    st = LIB.svdq_w4a4_nvfp4_linear(_ptr(act_codes), _ptr(act_scales), _ptr(lowrank_act),
                                    float(act_global_scale), _ptr(packed_w), float(w_global_scale),
                                    M, N, K, rank, _ptr(Y), _stream())
    _check("svdq_w4a4_nvfp4_linear", st)
    return Y


def svdq_w4a4_nvfp4_linear_qkv(act_codes, act_scales, lowrank_act, act_global_scale, packed_w, w_global_scale,
                               M, N, K, heads, norm_wq, norm_wk, eps, rope_cos, rope_sin, rank=RANK, Y=None):
    """The fused Q/K/V projection: Y bf16 [M, N = 3 heads 128] holding q, k (RMS-normalised per
    head with norm_wq / norm_wk bf16 [128], then rotated by rope_cos / rope_sin float32 [64, M],
    pair-major) and v."""
    D = 128
    _require(act_codes, torch.uint8, (M, K // 2), "act_codes")
    _require(act_scales, torch.uint8, (svdq_act_scale_bytes(M, K),), "act_scales")
    _require(lowrank_act, torch.bfloat16, (M, 2 * rank), "lowrank_act")
    _require_blob(packed_w, "packed_w", svdq_packed_weight_bytes(N, K, rank))
    _require(norm_wq, torch.bfloat16, (D,), "norm_wq")
    _require(norm_wk, torch.bfloat16, (D,), "norm_wk")
    _require(rope_cos, torch.float32, (D // 2, M), "rope_cos")
    _require(rope_sin, torch.float32, (D // 2, M), "rope_sin")
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=act_codes.device)
    _require(Y, torch.bfloat16, (M, N), "Y")
    st = LIB.svdq_w4a4_nvfp4_linear_qkv(_ptr(act_codes), _ptr(act_scales), _ptr(lowrank_act),
                                        float(act_global_scale), _ptr(packed_w), float(w_global_scale),
                                        M, N, K, rank, heads, D, _ptr(norm_wq), _ptr(norm_wk), float(eps),
                                        _ptr(rope_cos), _ptr(rope_sin), _ptr(Y), _stream())
    _check("svdq_w4a4_nvfp4_linear_qkv", st)
    return Y


def svdq_gelu_quant_workspace_bytes(M, N):
    return int(LIB.svdq_gelu_quant_workspace_bytes(M, N))


def svdq_gelu_table_fill(table=None, device=None):
    """The GELU table (uint8 [svdq_gelu_table_bytes()] CUDA tensor) filled by the library."""
    if table is None:
        table = torch.empty((int(LIB.svdq_gelu_table_bytes()),), dtype=torch.uint8,
                            device=device if device is not None else torch.device("cuda", torch.cuda.current_device()))
    _require_blob(table, "gelu_table", int(LIB.svdq_gelu_table_bytes()))
    _check("svdq_gelu_table_fill", LIB.svdq_gelu_table_fill(_ptr(table), _stream()))
    return table


_GELU_TABLES = {}


def _gelu_table(device):
    """A filled GELU table per device, made on first use (on the current stream)."""
    key = device.index if device.index is not None else torch.cuda.current_device()
    if key not in _GELU_TABLES:
        _GELU_TABLES[key] = svdq_gelu_table_fill(device=torch.device("cuda", key))
    return _GELU_TABLES[key]


def svdq_w4a4_nvfp4_linear_gelu_quant(act_codes, act_scales, lowrank_act, act_global_scale, packed_w, w_global_scale,
                                      M, N, K, down_smooth_inv, down_packed_w, down_act_global_scale, rank=RANK,
                                      out_codes=None, out_scales=None, out_lowrank_act=None, workspace=None,
                                      h_out=None, gelu_table=None):
    """The MLP up projection with GELU and the down projection's activation pass fused: returns the
    down projection's (act_codes uint8 [M, N/2], act_scales, lowrank_act bf16 [M, 2r]) for its
    smooth_inv (bf16 [N]), packed weights (its low-rank section is used) and g_a.  h_out (bf16
    [M, N]), if given, also receives the hidden state."""
    _require(act_codes, torch.uint8, (M, K // 2), "act_codes")
    _require(act_scales, torch.uint8, (svdq_act_scale_bytes(M, K),), "act_scales")
    _require(lowrank_act, torch.bfloat16, (M, 2 * rank), "lowrank_act")
    _require_blob(packed_w, "packed_w", svdq_packed_weight_bytes(N, K, rank))
    _require(down_smooth_inv, torch.bfloat16, (N,), "down_smooth_inv")
    _require_blob(down_packed_w, "down_packed_w", _l1_section_end(N, rank))
    dev = act_codes.device
    if out_codes is None:
        out_codes = torch.empty((M, N // 2), dtype=torch.uint8, device=dev)
    if out_scales is None:
        out_scales = torch.empty((svdq_act_scale_bytes(M, N),), dtype=torch.uint8, device=dev)
    if out_lowrank_act is None:
        out_lowrank_act = torch.empty((M, 2 * rank), dtype=torch.bfloat16, device=dev)
    ws_bytes = svdq_gelu_quant_workspace_bytes(M, N)
    if workspace is None:
        workspace = torch.empty((max(ws_bytes, 16),), dtype=torch.uint8, device=dev)
    _require(out_codes, torch.uint8, (M, N // 2), "out_codes")
    _require(out_scales, torch.uint8, (svdq_act_scale_bytes(M, N),), "out_scales")
    _require(out_lowrank_act, torch.bfloat16, (M, 2 * rank), "out_lowrank_act")
    _require_blob(workspace, "workspace", ws_bytes)
    if gelu_table is None:
        gelu_table = _gelu_table(dev)
    _require_blob(gelu_table, "gelu_table", int(LIB.svdq_gelu_table_bytes()))
    if h_out is not None:
        _require(h_out, torch.bfloat16, (M, N), "h_out")
    st = LIB.svdq_w4a4_nvfp4_linear_gelu_quant(_ptr(act_codes), _ptr(act_scales), _ptr(lowrank_act),
                                               float(act_global_scale), _ptr(packed_w), float(w_global_scale),
                                               M, N, K, rank, _ptr(down_smooth_inv), _ptr(down_packed_w),
                                               float(down_act_global_scale), _ptr(out_codes), _ptr(out_scales),
                                               _ptr(out_lowrank_act), _ptr(workspace), workspace.numel(),
                                               _ptr(gelu_table), _ptr(h_out), _stream())
    _check("svdq_w4a4_nvfp4_linear_gelu_quant", st)
    return out_codes, out_scales, out_lowrank_act


def int4_padded_rows(M):
    """Rows of the int4 row's activation-scale array: M rounded up to a multiple of 128."""
    return (M + 127) // 128 * 128


def svdq_int4_quantize_act_lowrank_down(X, smooth_inv, packed_w, rank=RANK, act_codes=None, act_scales=None,
                                        lowrank_act=None):
    """The int4 row's activation pass: (act_codes uint8 [M, K] (E4M3 bytes of the int4 codes),
    act_scales bf16 [K/64, Mp] (group-major, rows padded to Mp = a multiple of 128 with zero
    scales), lowrank_act bf16 [M, 2r] (U as hi then lo))."""
    M, K = X.shape
    Mp = int4_padded_rows(M)
    dev = X.device
    _require_blob(packed_w, "packed_w", _l1_section_end(K, rank))
    _require(X, torch.bfloat16, (M, K), "X")
    _require(smooth_inv, torch.bfloat16, (K,), "smooth_inv")
    if act_codes is None:
        act_codes = torch.empty((M, K), dtype=torch.uint8, device=dev)
    if act_scales is None:
        act_scales = torch.empty((K // 64, Mp), dtype=torch.bfloat16, device=dev)
    if lowrank_act is None:
        lowrank_act = torch.empty((M, 2 * rank), dtype=torch.bfloat16, device=dev)
    _require(act_codes, torch.uint8, (M, K), "act_codes")
    _require(act_scales, torch.bfloat16, (K // 64, Mp), "act_scales")
    _require(lowrank_act, torch.bfloat16, (M, 2 * rank), "lowrank_act")
    st = LIB.svdq_int4_quantize_act_lowrank_down(_ptr(X), _ptr(smooth_inv), _ptr(packed_w), M, K, rank,
                                                 _ptr(act_codes), _ptr(act_scales), _ptr(lowrank_act), _stream())
    _check("svdq_int4_quantize_act_lowrank_down", st)
    return act_codes, act_scales, lowrank_act


def svdq_w4a4_int4_linear(act_codes, act_scales, lowrank_act, packed_w, M, N, K, rank=RANK, Y=None):
    """Y bf16 [M, N] of the int4 / group-64 row."""
    _require(act_codes, torch.uint8, (M, K), "act_codes")
    _require(act_scales, torch.bfloat16, (K // 64, int4_padded_rows(M)), "act_scales")
    _require(lowrank_act, torch.bfloat16, (M, 2 * rank), "lowrank_act")
    _require_blob(packed_w, "packed_w", int(LIB.svdq_int4_packed_weight_bytes(N, K, rank)))
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=act_codes.device)
    _require(Y, torch.bfloat16, (M, N), "Y")
    st = LIB.svdq_w4a4_int4_linear(_ptr(act_codes), _ptr(act_scales), _ptr(lowrank_act), _ptr(packed_w), M, N, K,
                                   rank, _ptr(Y), _stream())
    _check("svdq_w4a4_int4_linear", st)
    return Y


def svdq_act_amax(X, smooth_inv, act_amax=None):
    """Returns the 16-byte device buffer (int32 [4]) whose word 0 holds the bits of
    max |X smooth_inv| (the dynamic scale's input); a buffer passed in must have been
    zero-filled once (the call leaves words 1-3 zero)."""
    M, K = X.shape
    _require(X, torch.bfloat16, (M, K), "X")
    _require(smooth_inv, torch.bfloat16, (K,), "smooth_inv")
    if act_amax is None:
        act_amax = torch.zeros((4,), dtype=torch.int32, device=X.device)
    _require(act_amax, torch.int32, (4,), "act_amax")
    st = LIB.svdq_act_amax(_ptr(X), _ptr(smooth_inv), M, K, _ptr(act_amax), _stream())
    _check("svdq_act_amax", st)
    return act_amax


def svdq_act_amax_noalloc(X, smooth_inv, amax):
    """max |X smooth_inv| into `amax` (a float32 [1] CUDA tensor), through the C call that
    allocates nothing (its scratch is the library's own static array; calls must not overlap
    on the GPU)."""
    M, K = X.shape
    _require(X, torch.bfloat16, (M, K), "X")
    _require(smooth_inv, torch.bfloat16, (K,), "smooth_inv")
    _require(amax, torch.float32, (1,), "amax")
    st = LIB.svdq_act_amax_noalloc(_ptr(X), _ptr(smooth_inv), M, K, _ptr(amax), _stream())
    _check("svdq_act_amax_noalloc", st)
    return amax


def svdq_quantize_act_lowrank_down_dyn(X, smooth_inv, packed_w, act_amax, rank=RANK,
                                       act_codes=None, act_scales=None, lowrank_act=None):
    """As svdq_quantize_act_lowrank_down with g_a formed on the device from act_amax."""
    M, K = X.shape
    dev = X.device
    _require_blob(packed_w, "packed_w", _l1_section_end(K, rank))
    _require(X, torch.bfloat16, (M, K), "X")
    _require(smooth_inv, torch.bfloat16, (K,), "smooth_inv")
    _require(act_amax, torch.int32, (4,), "act_amax")
    if act_codes is None:
        act_codes = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
    if act_scales is None:
        act_scales = torch.empty((svdq_act_scale_bytes(M, K),), dtype=torch.uint8, device=dev)
    if lowrank_act is None:
        lowrank_act = torch.empty((M, 2 * rank), dtype=torch.bfloat16, device=dev)
    _require(act_codes, torch.uint8, (M, K // 2), "act_codes")
    _require(act_scales, torch.uint8, (svdq_act_scale_bytes(M, K),), "act_scales")
    _require(lowrank_act, torch.bfloat16, (M, 2 * rank), "lowrank_act")
    st = LIB.svdq_quantize_act_lowrank_down_dyn(_ptr(X), _ptr(smooth_inv), _ptr(packed_w), M, K, rank,
                                                _ptr(act_amax), _ptr(act_codes), _ptr(act_scales),
                                                _ptr(lowrank_act), _stream())
    _check("svdq_quantize_act_lowrank_down_dyn", st)
    return act_codes, act_scales, lowrank_act


def svdq_w4a4_nvfp4_linear_dyn(act_codes, act_scales, lowrank_act, act_amax, packed_w, w_global_scale,
                               M, N, K, rank=RANK, Y=None):
    """As svdq_w4a4_nvfp4_linear with g_a formed on the device from act_amax."""
    _require(act_codes, torch.uint8, (M, K // 2), "act_codes")
    _require(act_scales, torch.uint8, (svdq_act_scale_bytes(M, K),), "act_scales")
    _require(lowrank_act, torch.bfloat16, (M, 2 * rank), "lowrank_act")
    _require(act_amax, torch.int32, (4,), "act_amax")
    _require_blob(packed_w, "packed_w", svdq_packed_weight_bytes(N, K, rank))
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=act_codes.device)
    _require(Y, torch.bfloat16, (M, N), "Y")
    st = LIB.svdq_w4a4_nvfp4_linear_dyn(_ptr(act_codes), _ptr(act_scales), _ptr(lowrank_act), _ptr(act_amax),
                                        _ptr(packed_w), float(w_global_scale), M, N, K, rank, _ptr(Y), _stream())
    _check("svdq_w4a4_nvfp4_linear_dyn", st)
    return Y


def awq_w4a16_linear(X, qweight, scales, zeros, bias=None, Y=None):
    """X bf16 [M, K]; qweight uint8 [N, K/2]; scales, zeros bf16 [N, K/64]; bias bf16 [N] or None.

    With K % 512 == 0, K <= 4096 and scales / zeros 16-byte aligned (tensors of their own are)
    the kernels stage the scale and zero rows in shared memory: the faster path, with results
    bit-identical to those of any other alignment."""
    M, K = X.shape
    N = qweight.shape[0]
    _require(X, torch.bfloat16, (M, K), "X")
    _require(qweight, torch.uint8, (N, K // 2), "qweight")
    _require(scales, torch.bfloat16, (N, K // 64), "scales")
    _require(zeros, torch.bfloat16, (N, K // 64), "zeros")
    if bias is not None:
        _require(bias, torch.bfloat16, (N,), "bias")
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _require(Y, torch.bfloat16, (M, N), "Y")
    st = LIB.awq_w4a16_linear(_ptr(X), _ptr(qweight), _ptr(scales), _ptr(zeros), _ptr(bias), M, N, K,
                              _ptr(Y), _stream())
    _check("awq_w4a16_linear", st)
    return Y


# ---------------------------------------------------------------- layers

class SvdqW4A4Linear:
    """An SVDQuant W4A4 NVFP4 linear layer held on one GPU.

    Built from the exporter's parameters: residual R [N, K] (float32), L1 [K, r],
    L2 [r, N], bias [N] (bf16 bit patterns as uint16, or None), smooth_inv [K]
    (bf16 bits) and the static activation scale g_a (a power of two)."""

    def __init__(self, R, L1_bits, L2_bits, bias_bits, smooth_inv_bits, act_global_scale, device="cuda"):
        blob, g_w = svdq_pack_weights(R, L1_bits, L2_bits, bias_bits, smooth_inv_bits)
        self.N, self.K = R.shape
        self.rank = L1_bits.shape[1]
        self.packed = torch.from_numpy(blob).to(device)
        self.w_global_scale = g_w
        self.act_global_scale = float(act_global_scale)
        self.smooth_inv = torch.from_numpy(np.ascontiguousarray(smooth_inv_bits, np.uint16).view(np.int16)) \
            .view(torch.bfloat16).to(device)

    def __call__(self, X, Y=None):
        M = X.shape[0]
        codes, scales, U = svdq_quantize_act_lowrank_down(X, self.smooth_inv, self.packed, self.act_global_scale,
                                                          self.rank)
        return svdq_w4a4_nvfp4_linear(codes, scales, U, self.act_global_scale, self.packed, self.w_global_scale,
                                      M, self.N, self.K, self.rank, Y)


class AwqW4A16Linear:
    """An AWQ-style W4A16 int4 (group 64) linear layer held on one GPU."""

    def __init__(self, qweight, scales, zeros, bias=None):
        self.qweight, self.scales, self.zeros, self.bias = qweight, scales, zeros, bias

    def __call__(self, X, Y=None):
        return awq_w4a16_linear(X, self.qweight, self.scales, self.zeros, self.bias, Y)
