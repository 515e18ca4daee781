"""Seeded synthetic workloads shared by the tests, the benchmark and the CPU oracle.

This package only draws random numbers and prepares the layer's stored
parameters the way an offline exporter would (smoothing factors, rank-32
decomposition, residual, AWQ min/max quantization).  It holds none of the
runtime arithmetic that is under test (no NVFP4 quantizer, no GEMM, no
dequantization) and imports neither the oracle nor the CUDA product package.
"""

from .inputs import (  # noqa: F401
    SvdqWorkload,
    AwqWorkload,
    svdq_workload,
    awq_workload,
    bf16_bits,
    bf16_from_bits,
    to_bf16,
)
