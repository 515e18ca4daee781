"""CPU oracle for the SVDQuant W4A4 (NVFP4) linear layer and the AWQ W4A16 linear layer.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (the CUDA library and its Python binding) never imports
it, and nothing here imports the product package.

Everything is plain NumPy in float64, written from the definitions:

* ``formats``  E2M1 and E4M3 code tables built from their bit fields, and exact
  round-to-nearest-even quantizers onto those grids.
* ``nvfp4``    the NVFP4 block format: one E4M3 scale per 16 contiguous K
  elements, a power-of-two per-tensor scale, E2M1 codes; pack/unpack of nibbles.
* ``svdq``     the SVDQuant forward  y = Q4(X diag(lambda)^-1) Q4(R)^T
  + (X diag(lambda)^-1 L1) L2 + b.
* ``awq``      the AWQ-style W4A16 group-64 dequantize-then-matmul forward.
* ``int4``     the svdq_w4a4 int4 / group-64 row: signed 4-bit codes with a bf16 scale
  (amax / 7, rounded once) per 64 K elements on both operands, the same low-rank branch.
* ``qkv_epilogue``  the QKV projection's epilogue (per-head RMSNorm and RoPE of q and k),
  the definition a fused epilogue kernel is to match.
* ``mlp_epilogue``  the MLP up-projection's epilogue: GELU of the stored output, then the
  down projection's activation pass (NVFP4 codes, scales, low-rank U) on the hidden state.

Sources: "Nunchaku Lite" (Hugging Face Diffusers documentation), section
"Supported quantization types" (method table: svdq_w4a4 / nvfp4 / group 16,
svdq_w4a4 / int4 / 64, awq_w4a16 / int4 / 64) and section
"NunchakuLiteQuantizationConfig" (rank 32); the Indonesian article "Memangkas VRAM
Model Diffusi ... Lewat Nunchaku Lite", section on what happens when a diffusion
model is quantized (outliers moved into a 16-bit low-rank branch, W4A4 for the
rest; awq_w4a16 for adaptive-normalisation layers).  The pages never define E2M1
or E4M3; the tables follow the public OCP 8-bit floating point (E4M3 "FN": no
infinities, NaN at S.1111.111) and OCP microscaling (E2M1) definitions.

Parity status: every function here is pinned by tests under ``tests/`` against
code tables built independently, torch's float8_e4m3fn cast, brute-force
nearest-value search, exact rational arithmetic on tiny shapes, exact
reconstruction of representable blocks, and the low-rank decomposition identity.
No worked numeric example exists on the pages, so parity with the pages' own
kernels is unpinned beyond those invariants.
"""

from . import formats, nvfp4, svdq, awq, int4  # noqa: F401
