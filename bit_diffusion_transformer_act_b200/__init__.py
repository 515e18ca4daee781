"""SVDQuant W4A4 (NVFP4) and AWQ W4A16 linear layers for NVIDIA B200 (sm_100a).

The compute path is libsvdq.so (hand-written CUDA for sm_100a behind a C ABI,
``include/svdq.h``); this package is its ctypes binding.  Importing fails if
the library has not been built (``python bit_diffusion_transformer_act_b200/build.py``).
``torch_ops`` registers the device calls as ``torch.ops.svdq.*`` custom operators (with
fake implementations for tracing) and provides the nn.Module layers.
"""

from .ops import (  # noqa: F401
    RANK,
    SvdqError,
    EXPORTED,
    LIB,
    svdq_packed_weight_bytes,
    svdq_act_scale_bytes,
    svdq_pack_weights,
    svdq_unswizzle_scales,
    svdq_swizzle_scales,
    svdq_device_status,
    svdq_quantize_act_lowrank_down,
    svdq_w4a4_nvfp4_linear,
    svdq_w4a4_nvfp4_linear_qkv,
    svdq_w4a4_nvfp4_linear_gelu_quant,
    svdq_gelu_quant_workspace_bytes,
    svdq_gelu_table_fill,
    svdq_int4_pack_weights,
    int4_padded_rows,
    svdq_int4_quantize_act_lowrank_down,
    svdq_w4a4_int4_linear,
    awq_w4a16_linear,
    svdq_act_amax,
    svdq_act_amax_noalloc,
    svdq_quantize_act_lowrank_down_dyn,
    svdq_w4a4_nvfp4_linear_dyn,
    SvdqW4A4Linear,
    AwqW4A16Linear,
)
from .torch_ops import AwqLinear, SvdqLinear, swap_linears  # noqa: F401,E402
