"""ConvRot W8A8 / W4A4 quantized linear layer for NVIDIA B200 (sm_100a).

The compute lives in ``libconvrot.so`` (hand-written CUDA, C ABI in
``include/convrot.h``); this package is its thin Python binding.
"""
from .binding import (  # noqa: F401
    CLIP_ABSMAX, CLIP_MSE, ConvRotError, QuantizedLinear, convrot_device_status, convrot_gemm_w4a4,
    convrot_gemm_w8a8, convrot_linear_gemm, convrot_linear_quant_act, convrot_linear_w4a4, convrot_linear_w8a8,
    convrot_linear_w8a8_noalloc, convrot_quantize_weight, convrot_quantize_weight_tensorwise,
    convrot_rotate_quant_act, convrot_tensorwise_workspace_bytes,
    convrot_linear_workspace_bytes, convrot_version, convrot_workspace_bytes, load_library,
)
from ._build import build  # noqa: F401
