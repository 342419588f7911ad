"""B200-native forward pass of a top-k routed mixture-of-experts SwiGLU FFN layer.

The layer runs in libmoe.so (CUDA kernels for sm_100a behind the C ABI in
include/moe.h); this package is its thin Python binding plus the seeded
synthetic input generators. There is no CPU path: calls fail loudly when the
library or a CUDA device is missing.
"""
from . import _lib
from ._lib import (MOE_BF16, MOE_F32, MOE_NUM_KERNELS, KERNEL_NAMES, MoeError, moe_capacity,
                   moe_forward, moe_forward_host_io, moe_get_device_status, moe_workspace_layout,
                   moe_workspace_size, make_dims, status_string)
from .layer import (Workspace, dequantize_fp8, dequantize_mxfp4, forward, quantize_fp8,
                    quantize_mxfp4, routing_views)

__all__ = ["forward", "routing_views", "quantize_fp8", "dequantize_fp8", "quantize_mxfp4",
           "dequantize_mxfp4", "Workspace",
           "moe_forward", "moe_forward_host_io", "moe_workspace_size", "moe_workspace_layout", "moe_capacity", "moe_get_device_status",
           "make_dims", "status_string", "MoeError", "MOE_BF16", "MOE_F32", "MOE_NUM_KERNELS",
           "KERNEL_NAMES"]
