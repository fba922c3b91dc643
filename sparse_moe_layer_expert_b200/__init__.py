"""B200 (sm_100a) FP8 DeepSeekMoE layer forward.

The layer ("DeepSeek-V3 Technischer Bericht", Methode section 2, and the FP8
recipe of its Kernideen section) runs in the CUDA kernels of libmoefp8.so
behind the C ABI in include/moe_fp8.h; this package is its thin Python
binding.  Importing it raises ImportError when the library has not been built
(`python sparse_moe_layer_expert_b200/build.py`); there is no fallback.
"""
from ._binding import (  # noqa: F401
    EXPORTS, LIB_PATH, MOE_PROFILE_EVENTS, MOE_PROFILE_BWD_EVENTS, MOE_ROUTE_NOALLOC_SCRATCH_BYTES, PROFILE_STAGES,
    PROFILE_BWD_STAGES, MOE_DTYPE_BF16, MOE_DTYPE_F32, MOE_DEVERR_BAD_INDEX, MOE_DEVERR_TIMEOUT, MOE_ERR_CUDA,
    MOE_ERR_DEVICE, MOE_ERR_INVALID_ARG, MOE_ERR_NO_DEVICE, MOE_ERR_NOT_IMPLEMENTED, MOE_ERR_TIMEOUT,
    MOE_ERR_UNSUPPORTED_SHAPE, MOE_ERR_WORKSPACE_TOO_SMALL, MOE_OK, MOE_SCALE_AMAX, MOE_SCALE_POW2, MoeConfig, MoeWeights,
    MoeError, config, config_from,
    fp8_blockscaled_gemm, fp8_quant_128x128, fp8_quant_1x128, lib, moe_bias_update, moe_check_device_error,
    moe_forward, moe_profile_events, moe_route, moe_route_noalloc, moe_route_workspace_size, moe_selftest_wait_timeout,
    moe_seq_balance_loss, moe_set_gemm_variant, moe_gemm_kernel_for, moe_workspace_layout, MOE_GEMM_AUTO, MOE_GEMM_PAIR,
    MOE_GEMM_SINGLE, MOE_GEMM_BLOCK_SCALED, MOE_GEMM_TALL,
    moe_workspace_size, new_err_flag, weights_struct, ws_view, moe_ep_row_bytes, moe_ep_dispatch, moe_ep_experts,
    moe_ep_combine, moe_transpose_weights, moe_backward, moe_backward_workspace_layout,
)
from .layer import MoeLayer  # noqa: F401
