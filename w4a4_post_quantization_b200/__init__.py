"""B200-native KroQuant online activation quantizer.

Kronecker-structured 32x32 block transform followed by MXFP4 (E8M0 scale +
E2M1 codes), as hand-written sm_100a CUDA behind the C ABI in ``include/kq.h``.
This package is the thin Python binding over that library.
"""
from ._lib import (  # noqa: F401
    KQ_IMPL_AUTO, KQ_IMPL_DIRECT, KQ_IMPL_MMA, KQ_IMPL_PANEL, KQ_IMPL_TMA, KQ_IMPL_WARP, KQ_OUT_BF16, KQ_OUT_F32, KQError, LIB_PATH, dequantize,
    device_status, fold_weight, gemm_mxfp4, gemm_mxfp4_tiled, host_workspace_bytes, inverse_transform, lib, load_library, quantize,
    adam_step, params_grad_workspace_bytes, quantize_adaln, quantize_adaln_tiled, quantize_hadamard, residual,
    residual_workspace_bytes, scales_to_tiled, transform_params_grad, quantize_host, quantize_host_static, quantize_smooth, quantize16, quantize16_tiled, quantize_weight16, quantize_weight16_tiled, fold_weight16,
    gemm_mxfp4_16_tiled, quantize_tiled, quantize_weight, quantize_weight_tiled, transform,
    transform16, transform_adaln)

BLOCK = 32
