"""B200-native (sm_100a) INT4 group-wise weight-only GEMM (W4A16).

The product path is the C-ABI CUDA library `libw4a16.so` (see include/w4a16.h);
this package only builds it (`build.build()`) and binds it (`_lib`).
"""
from ._lib import (  # noqa: F401
    EXPORTED, MAX_EXPERTS, LaunchInfo, W4A16Error, device_status, gemm, grouped_gemm, load, pack,
    prepare_weights, quantize, repack, status_string, unpack, w4a16_device_status, w4a16_gemm,
    w4a16_gemm_launch_info, w4a16_grouped_gemm, w4a16_grouped_launch_info, w4a16_pack, w4a16_quantize,
    w4a16_repack, w4a16_set_fault_injection, w4a16_set_static_weights, w4a16_tiled_bytes, w4a16_unpack,
)
from ._lib import (  # noqa: F401
    ERR_BAD_OFFSETS, ERR_CUDA, ERR_INVALID_ARG, ERR_MISALIGNED, ERR_TIMEOUT, ERR_UNSUPPORTED, OK,
)
