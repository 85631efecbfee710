"""B200 (sm_100a) SVDQuant-style NVFP4 W4A4 linear layer.

The computation runs in ``libsvdq.so`` (C ABI in ``include/svdq.h``); this
package is its Python binding.  The library is loaded on first use, and any
call fails with ImportError if it has not been built
(``python -m bit_w4a4_quantized_svdq_b200.build``): there is no fallback.
With SVDQ_DEBUG=1 the debug build ``libsvdq_debug.so`` is loaded instead.
"""
from . import _lib
from ._lib import SvdqError
from .ops import (linear_score_workspace_bytes, mxfp8_sf_bytes, score_workspace_bytes, sf_bytes,
                  svdq_bits_lost, svdq_calib_lambda, svdq_calib_lambda_stored_w, svdq_device_error, svdq_lambda_grid, svdq_linear,
                  svdq_linear_mxfp8, svdq_linear_score, svdq_quantize_act, svdq_quantize_mxfp8, svdq_residual,
                  svdq_score_lambda, svdq_score_lambda_static)
from .layer import SVDQW4A4Linear, alpha_grid, lowrank_factors_device, search_lambda


def load():
    """Load the library (raises ImportError if it is missing) and return the ctypes handle."""
    return _lib.load()


__all__ = [
    "svdq_calib_lambda", "svdq_calib_lambda_stored_w", "svdq_quantize_act", "svdq_linear", "svdq_linear_score", "svdq_score_lambda",
    "svdq_score_lambda_static", "linear_score_workspace_bytes", "svdq_bits_lost", "svdq_lambda_grid",
    "svdq_quantize_mxfp8", "svdq_linear_mxfp8", "mxfp8_sf_bytes",
    "svdq_residual", "svdq_device_error", "sf_bytes", "score_workspace_bytes", "SVDQW4A4Linear",
    "lowrank_factors_device", "alpha_grid", "search_lambda", "load", "SvdqError",
]
