"""The MLP up-projection's epilogue: GELU, then the NVFP4 quantization and rank-32 down
projection that the MLP down-projection's first kernel applies to the hidden state -- in
float64.

Test infrastructure (see the package docstring).

Method: "Nunchaku Lite" docs, section on fused kernels -- the original engine runs the MLP
with a fused GELU kernel (the benchmark table gives the GELU-MLP fusion 1.06x).  The pages
name the operation only; the readings used here:

* GELU is the exact (erf) form, x * Phi(x);
* the fused epilogue is to give what the unfused pipeline gives: the up projection's output
  y stored as bf16, GELU of that stored as bf16 (the hidden state h), then the down
  projection's activation pass on h -- smoothing by its smooth_inv, NVFP4 codes and scales with
  its per-tensor scale g_a, and U = h_hat L1 of its low-rank factor.
"""

import math

import numpy as np

from . import svdq
from .formats import bf16_round


def gelu(x):
    """x * Phi(x) with the standard normal distribution function Phi (the erf form of GELU),
    evaluated as Phi(x) = erfc(-x / sqrt 2) / 2: the same function as (1 + erf(x / sqrt 2)) / 2,
    but float64 keeps its relative accuracy where Phi is tiny (1 + erf cancels for x below about
    -7, and is exactly 0 from about -8.3 on although x Phi(x) is still a normal bf16 value)."""
    x = np.asarray(x, dtype=np.float64)
    erfc = np.vectorize(math.erfc, otypes=[np.float64])
    return 0.5 * x * erfc(-x / math.sqrt(2.0))


def hidden_state(y_up):
    """h = bf16(GELU(bf16(y))): the hidden state as the unfused pipeline stores it -- the up
    projection's output rounded to bf16, its GELU evaluated here in float64 (the erfc form:
    essentially exact, relative error about 1e-16 everywhere) and rounded once to bf16.

    Since bf16(y) takes 65536 values, h is a function of 16 bits; a kernel may take it from a
    table of this function (computed in double precision and rounded once, it equals this one
    for every input).  A kernel that evaluates GELU in fp32 instead rounds the same way except
    where the exact value lies within that evaluation's error of a bf16 midpoint.  The contract
    a fused kernel is held to is stated on its own intermediate values: its h equals (or, with
    an fp32 GELU, lies within one bf16 ulp of) hidden_state of its own bf16 y, and its codes and
    scales equal quantize_activations of its own h bit for bit."""
    return bf16_round(gelu(bf16_round(np.asarray(y_up, dtype=np.float64))))


def gelu_requantize(y_up, smooth_inv_down, g_a_down, L1_down):
    """The down projection's activation pass on the hidden state of y_up [M, F]: (codes [M, F],
    E4M3 scales [M, F/16], U = h_hat L1_down [M, r])."""
    h = hidden_state(y_up)
    codes, scales = svdq.quantize_activations(h, smooth_inv_down, g_a_down)
    return codes, scales, svdq.lowrank_down(h, smooth_inv_down, L1_down)
