"""Routed-expert MoE layer (router + top-k, permutation, grouped SwiGLU
experts in BF16 / AWQ W4A16 g32 / NVFP4 W4A4, combine) and RAZOR Refill-RMS
expert scoring for NVIDIA B200 (sm_100a).

The compute path is the C ABI of libmoe_b200.so (include/moe.h), bound
function-for-function in `abi`; `MoELayer` chains those calls into a layer.
`synth` draws the seeded synthetic inputs.
"""

from . import abi, synth  # noqa: F401
from .abi import (  # noqa: F401
    moe_awq_dequant_g32,
    moe_combine,
    moe_device_status,
    moe_grouped_swiglu_awq_g32,
    moe_grouped_swiglu_bf16,
    moe_grouped_swiglu_nvfp4,
    moe_nvfp4_quantize,
    moe_permute,
    moe_route_topk,
    moe_workspace_size,
    razor_refill_rms_accumulate,
    razor_select,
)
from .layer import MoELayer  # noqa: F401
