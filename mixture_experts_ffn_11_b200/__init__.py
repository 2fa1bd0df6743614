"""B200-native (sm_100a) sparse mixture-of-experts feed-forward layer.

The CUDA library ``libmoe.so`` (C-ABI in ``include/moe.h``) does all the work; this package is its thin
Python binding (``_native``) plus a layer object that owns buffers and calls the entry points in order
(``layer.MoEFFN``). Importing the package loads the library and fails if it has not been built.
"""
from . import _native
from ._native import (MoEError, ROUTE_MODES, get_device_error, grouped_gemm_down, grouped_gemm_gateup, permute,
                      permute_workspace_size, route_topk, topk_from_logits, unpermute_combine)
from .layer import MoEFFN

__all__ = ["MoEFFN", "MoEError", "ROUTE_MODES", "route_topk", "topk_from_logits", "permute",
           "permute_workspace_size", "grouped_gemm_gateup", "grouped_gemm_down", "unpermute_combine",
           "get_device_error"]
