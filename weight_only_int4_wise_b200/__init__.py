"""B200-native (sm_100a) INT4 group-wise weight-only GEMM (W4A16).

The product path is the C-ABI CUDA library `libw4a16.so` (see include/w4a16.h);
this package only builds it (`build.build()`) and binds it (`_lib`).
"""
from ._lib import (  # noqa: F401
    EXPORTED, MAX_EXPERTS, MAX_TOPK, LaunchInfo, W4A16Error, device_status, gemm, grouped_gemm, load, moe_layer,
    pack, prepare_weights, quantize, repack, status_string, unpack, w4a16_device_status, w4a16_gemm,
    w4a16_gemm_launch_info, w4a16_grouped_gemm, w4a16_grouped_gemm_act, w4a16_grouped_launch_info,
    w4a16_moe_combine, w4a16_moe_dispatch, w4a16_moe_gather, w4a16_moe_layer, w4a16_moe_route,
    w4a16_moe_workspace_size, w4a16_pack, w4a16_quantize, w4a16_repack, w4a16_set_fault_injection,
    w4a16_set_static_weights, w4a16_tiled_bytes, w4a16_unpack, w4a16_get_valid_tactics, w4a16_tactic_launch_info,
    w4a16_set_tactic, w4a16_get_tactic, w4a16_clear_tactics, w4a16_autotune, w8a16_tiled_bytes, w8a16_repack,
    w8a16_gemm, w8a16_gemm_launch_info, repack_w8, gemm_w8, w4a16_moe_layer_static, w4a16_moe_static_scratch_bytes,
    w4a16_gemm_ex, FLAG_STATIC_WEIGHTS, w8a16_quantize, quantize_w8,
)
from ._lib import (  # noqa: F401
    ACT_GELU_ERF, ACT_GELU_TANH, ACT_IDENTITY, ACT_RELU, ERR_BAD_OFFSETS, ERR_BAD_ROUTING, ERR_CUDA,
    ERR_INVALID_ARG, ERR_MISALIGNED, ERR_SCRATCH_TOO_SMALL, ERR_TIMEOUT, ERR_UNSUPPORTED, OK,
)
