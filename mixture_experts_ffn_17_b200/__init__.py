"""B200-native forward pass of a DeepSeek-V3-style mixture-of-experts FFN layer.

The computation lives in libmoe.so (CUDA for sm_100a behind the C ABI in
include/moe.h); `binding` marshals torch tensors to it.  `layer` wraps one
layer's weights and workspace for convenience.
"""
from .binding import (MOE_BF16, MOE_E4M3, MOE_F32, MOE_ROUTE_SIGMOID_GROUP, MOE_ROUTE_TOPK_SOFTMAX, MoeError,
                      MoeShape, make_shape, shape_of)

__all__ = ["MoeError", "MoeShape", "make_shape", "shape_of", "MOE_BF16", "MOE_E4M3", "MOE_F32",
           "MOE_ROUTE_TOPK_SOFTMAX", "MOE_ROUTE_SIGMOID_GROUP"]
