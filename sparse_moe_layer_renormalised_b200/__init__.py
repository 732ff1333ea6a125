"""Stable LatentMoE layer forward pass for NVIDIA B200 (sm_100a).

The compute path is the CUDA library built from ``csrc/`` (``libmoe_b200.so``);
this package is its ctypes binding.  See ``include/moe.h`` for the ABI.
"""
from ._binding import (  # noqa: F401
    EXPORTED,
    LIB_PATH,
    MOE_BF16,
    MOE_ERR_CUDA,
    MOE_ERR_DEVICE,
    MOE_ERR_INVALID_ARG,
    MOE_ERR_UNSUPPORTED,
    MOE_F32,
    MOE_MXFP4,
    MOE_NUM_STAGES,
    STAGE_NAMES,
    MOE_OK,
    Dims,
    MoeLibraryMissing,
    check,
    lib,
    make_aux,
    make_weights,
    moe_aux,
    moe_combine,
    moe_device_error,
    moe_dims,
    moe_expert_ffn,
    moe_last_launch_count,
    moe_layer_forward,
    moe_permute,
    moe_permute_noalloc,
    moe_qb_bias_update,
    MOE_PERMUTE_NOALLOC_SCRATCH_BYTES,
    moe_router_topk,
    moe_status_str,
    moe_weights,
    moe_workspace_size,
)
from .layer import MoeLayer  # noqa: F401
