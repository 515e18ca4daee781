"""PyTorch operator registration and nn.Module layers over libsvdq.

The three device calls of include/svdq.h are registered as ``torch.library`` custom
operators (namespace ``svdq``) with fake implementations, so that the layers can be
traced by ``torch.compile(fullgraph=True)`` / ``torch.export`` without graph breaks; the
real implementations are the ctypes calls of ``ops.py`` (the CUDA kernels, on the current
stream).  Method: "Nunchaku Lite" docs, "Supported quantization types" and the
``NunchakuLiteQuantizationConfig`` section (the layers replace nn.Linear in a model).

Operators (all tensors on one CUDA device):
  svdq::quantize_act_lowrank_down(X bf16 [M,K], smooth_inv bf16 [K], packed_w u8,
      act_global_scale float, rank int) -> (codes u8 [M,K/2], scales u8 [svdq_act_scale_bytes],
      lowrank_act bf16 [M,2 rank])
  svdq::w4a4_nvfp4_linear(codes, scales, lowrank_act, act_global_scale, packed_w,
      w_global_scale float, N int, rank int) -> Y bf16 [M,N]
  svdq::awq_w4a16_linear(X bf16 [M,K], qweight u8 [N,K/2], scales bf16 [N,K/64],
      zeros bf16 [N,K/64], bias bf16 [N] or None) -> Y bf16 [M,N]
"""

from typing import Callable, Optional, Tuple

import numpy as np
import torch
from torch import nn

from . import ops


# ---------------------------------------------------------------- operators

@torch.library.custom_op("svdq::quantize_act_lowrank_down", mutates_args=())
def quantize_act_lowrank_down(X: torch.Tensor, smooth_inv: torch.Tensor, packed_w: torch.Tensor,
                              act_global_scale: float, rank: int) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    return ops.svdq_quantize_act_lowrank_down(X, smooth_inv, packed_w, act_global_scale, rank)


@quantize_act_lowrank_down.register_fake
def _(X, smooth_inv, packed_w, act_global_scale, rank):
    M, K = X.shape
    # swizzled scales: rows padded to the 128-row atom, one byte per 16 K
    return (X.new_empty((M, K // 2), dtype=torch.uint8),
            X.new_empty((((M + 127) // 128) * 128 * (K // 16),), dtype=torch.uint8),
            X.new_empty((M, 2 * rank), dtype=torch.bfloat16))


@torch.library.custom_op("svdq::w4a4_nvfp4_linear", mutates_args=())
def w4a4_nvfp4_linear(act_codes: torch.Tensor, act_scales: torch.Tensor, lowrank_act: torch.Tensor,
                      act_global_scale: float, packed_w: torch.Tensor, w_global_scale: float, N: int,
                      rank: int) -> torch.Tensor:
    M, half_k = act_codes.shape
    return ops.svdq_w4a4_nvfp4_linear(act_codes, act_scales, lowrank_act, act_global_scale, packed_w,
                                      w_global_scale, M, N, 2 * half_k, rank)


@w4a4_nvfp4_linear.register_fake
def _(act_codes, act_scales, lowrank_act, act_global_scale, packed_w, w_global_scale, N, rank):
    return act_codes.new_empty((act_codes.shape[0], N), dtype=torch.bfloat16)


@torch.library.custom_op("svdq::awq_w4a16_linear", mutates_args=())
def awq_w4a16_linear(X: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                     bias: Optional[torch.Tensor]) -> torch.Tensor:
    return ops.awq_w4a16_linear(X, qweight, scales, zeros, bias)


@awq_w4a16_linear.register_fake
def _(X, qweight, scales, zeros, bias):
    return X.new_empty((X.shape[0], qweight.shape[0]), dtype=torch.bfloat16)


# ---------------------------------------------------------------- layers

def _as_2d(x: torch.Tensor, K: int) -> torch.Tensor:
    if x.shape[-1] != K:
        raise ValueError(f"last dimension {x.shape[-1]} != in_features {K}")
    return x.reshape(-1, K).contiguous()


class SvdqLinear(nn.Module):
    """SVDQuant W4A4 NVFP4 linear layer (rank-32 16-bit low-rank branch), a drop-in for
    nn.Linear on bf16 inputs of any leading shape.

    Built from the exporter's parameters (see ``from_exported``); holds the packed weight
    blob, the bf16 smoothing factors and the two power-of-two per-tensor scales."""

    def __init__(self, in_features: int, out_features: int, rank: int, packed_w: torch.Tensor,
                 smooth_inv: torch.Tensor, act_global_scale: float, w_global_scale: float):
        super().__init__()
        self.in_features, self.out_features, self.rank = in_features, out_features, rank
        self.register_buffer("packed_w", packed_w)
        self.register_buffer("smooth_inv", smooth_inv)
        self.act_global_scale = float(act_global_scale)
        self.w_global_scale = float(w_global_scale)

    @classmethod
    def from_exported(cls, R: np.ndarray, L1_bits: np.ndarray, L2_bits: np.ndarray,
                      bias_bits: Optional[np.ndarray], smooth_inv_bits: np.ndarray, act_global_scale: float,
                      device="cuda") -> "SvdqLinear":
        """R float32 [N, K] (residual), L1 / L2 bf16 bit patterns [K, r] / [r, N], bias [N] or None,
        smooth_inv [K] (bf16 bits), act_global_scale a power of two (calibration)."""
        blob, g_w = ops.svdq_pack_weights(R, L1_bits, L2_bits, bias_bits, smooth_inv_bits)
        N, K = R.shape
        smooth = torch.from_numpy(np.ascontiguousarray(smooth_inv_bits, np.uint16).view(np.int16)) \
            .view(torch.bfloat16)
        return cls(K, N, L1_bits.shape[1], torch.from_numpy(blob).to(device), smooth.to(device),
                   act_global_scale, g_w)

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        lead = x.shape[:-1]
        x2 = _as_2d(x, self.in_features)
        codes, scales, lowrank = torch.ops.svdq.quantize_act_lowrank_down(
            x2, self.smooth_inv, self.packed_w, self.act_global_scale, self.rank)
        y = torch.ops.svdq.w4a4_nvfp4_linear(codes, scales, lowrank, self.act_global_scale, self.packed_w,
                                             self.w_global_scale, self.out_features, self.rank)
        return y.reshape(*lead, self.out_features)

    def get_extra_state(self):
        # the per-tensor scales and sizes travel with state_dict() next to the buffers
        return {"in_features": self.in_features, "out_features": self.out_features, "rank": self.rank,
                "act_global_scale": self.act_global_scale, "w_global_scale": self.w_global_scale}

    def set_extra_state(self, state):
        self.in_features, self.out_features = int(state["in_features"]), int(state["out_features"])
        self.rank = int(state["rank"])
        self.act_global_scale = float(state["act_global_scale"])
        self.w_global_scale = float(state["w_global_scale"])

    def extra_repr(self) -> str:
        return f"in_features={self.in_features}, out_features={self.out_features}, rank={self.rank}, nvfp4"


class AwqLinear(nn.Module):
    """AWQ-style W4A16 int4 (group 64) linear layer, a drop-in for nn.Linear on bf16 inputs
    of any leading shape (built for the few rows of the adaptive normalisation; more than 64
    rows after flattening run in 64-row tiles that each re-read the weights)."""

    def __init__(self, qweight: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                 bias: Optional[torch.Tensor] = None):
        super().__init__()
        self.out_features, half_k = qweight.shape
        self.in_features = 2 * half_k
        self.register_buffer("qweight", qweight)
        self.register_buffer("scales", scales)
        self.register_buffer("zeros", zeros)
        self.register_buffer("bias", bias)

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        lead = x.shape[:-1]
        y = torch.ops.svdq.awq_w4a16_linear(_as_2d(x, self.in_features), self.qweight, self.scales, self.zeros,
                                            self.bias)
        return y.reshape(*lead, self.out_features)

    def extra_repr(self) -> str:
        return f"in_features={self.in_features}, out_features={self.out_features}, int4 group 64"


def swap_linears(model: nn.Module, factory: Callable[[str, nn.Linear], Optional[nn.Module]]) -> int:
    """Replaces, in place, every nn.Linear of ``model`` for which ``factory(qualified_name, linear)``
    returns a module (for instance an SvdqLinear or AwqLinear built from that layer's exported
    parameters); returns how many were replaced."""
    replaced = 0
    for parent_name, parent in list(model.named_modules()):
        for child_name, child in list(parent.named_children()):
            if isinstance(child, nn.Linear):
                name = f"{parent_name}.{child_name}" if parent_name else child_name
                new = factory(name, child)
                if new is not None:
                    setattr(parent, child_name, new)
                    replaced += 1
    return replaced
