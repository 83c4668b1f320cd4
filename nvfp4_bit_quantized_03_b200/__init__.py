"""NVFP4 training hot path on B200 (sm_100a): quantizers and block-scaled FP4 GEMMs for the
three GEMMs of a linear layer, behind the C ABI of libnvfp4.so (include/nvfp4.h).

The Python surface is the ctypes binding in ``binding``; it loads the in-tree
``libnvfp4.so`` on first use and raises if the library is missing.
"""
from . import binding
from .binding import (AMAX_GIVEN, BLOCK2D, COLWISE, OUT_BF16, OUT_F32, ROWWISE, SR,
                      DEVSTAT_BOUNDS, DEVSTAT_NONFINITE, DEVSTAT_TIMEOUT, NVFP4Error,
                      QuantizedTensor, bounds_checked, gemm,
                      linear_dgrad, linear_fprop, linear_wgrad, quantize, rht_quantize,
                      sign_mask_from_seed)

__all__ = ["binding", "AMAX_GIVEN", "BLOCK2D", "COLWISE", "OUT_BF16", "OUT_F32", "ROWWISE", "SR",
           "DEVSTAT_BOUNDS", "DEVSTAT_NONFINITE", "DEVSTAT_TIMEOUT", "NVFP4Error",
           "QuantizedTensor", "bounds_checked", "gemm",
           "linear_dgrad", "linear_fprop", "linear_wgrad", "quantize", "rht_quantize",
           "sign_mask_from_seed"]
