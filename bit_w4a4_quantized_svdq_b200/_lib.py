"""ctypes view of ``libsvdq.so`` (the C ABI declared in ``include/svdq.h``).

With the environment variable ``SVDQ_DEBUG=1`` the debug build
``libsvdq_debug.so`` is loaded instead (pointer checks on the host, store bounds
checks in the kernels); the binding then also checks the device error word and
the guard bands of the outputs it allocated after every call.  Loading fails
loudly when the library is missing: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, Structure, c_char_p, c_int, c_int64, c_size_t, c_uint32, c_void_p

from .build import DEBUG_LIB_PATH, LIB_PATH

DEBUG = os.environ.get("SVDQ_DEBUG", "0") not in ("", "0")

SVDQ_OK = 0
SVDQ_ERR_INVALID_ARG = 1
SVDQ_ERR_UNSUPPORTED = 2
SVDQ_ERR_MISALIGNED = 3
SVDQ_ERR_CUDA = 4
SVDQ_ERR_TIMEOUT = 5
SVDQ_ERR_NO_DEVICE = 6
SVDQ_ERR_SCRATCH_TOO_SMALL = 7
SVDQ_ERR_BOUNDS = 8


class SvdqSeg(Structure):
    _fields_ = [("begin", c_int64), ("end", c_int64)]


class SvdqError(RuntimeError):
    def __init__(self, call: str, status: int, text: str, code: int = 0):
        super().__init__(f"{call} failed: {text} (status {status})")
        self.status = status
        self.code = code          # the device error word's code, where one was read


# name -> (restype, argtypes); mirrors include/svdq.h
SIGNATURES = {
    "svdq_status_string": (c_char_p, [c_int]),
    "svdq_version": (c_int, []),
    "svdq_sf_bytes": (c_size_t, [c_int64, c_int64]),
    "svdq_calib_lambda": (c_int, [c_void_p, c_int64, c_int64, c_int64, POINTER(SvdqSeg), c_int,
                                  c_void_p, c_int64, c_int64,
                                  c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "svdq_calib_lambda_stored_w": (c_int, [c_void_p, c_int64, c_int64, c_int64, POINTER(SvdqSeg), c_int, c_void_p,
                                           c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "svdq_quantize_act": (c_int, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p,
                                  c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "svdq_linear": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                            c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                            c_void_p, c_int64, c_int, c_int64, c_int64, c_int64, c_void_p]),
    "svdq_score_workspace_bytes": (c_size_t, [POINTER(SvdqSeg), c_int, c_int64]),
    "svdq_score_lambda": (c_int, [c_void_p, c_void_p, c_int64, c_int64, c_int64, POINTER(SvdqSeg), c_int,
                                  c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "svdq_score_static_max_bytes": (c_size_t, []),
    "svdq_score_lambda_static": (c_int, [c_void_p, c_void_p, c_int64, c_int64, c_int64, POINTER(SvdqSeg), c_int,
                                         c_void_p, c_void_p, c_void_p, c_void_p]),
    "svdq_residual": (c_int, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p, c_void_p, c_int,
                              c_void_p, c_void_p]),
    "svdq_device_error": (c_int, [c_void_p, POINTER(c_uint32)]),
    "svdq_debug_arm_score_timeout": (c_int, [c_int64, c_int64]),
    "svdq_debug_build": (c_int, []),
    "svdq_debug_limit_extent": (c_int, [c_int, c_int64]),
    "svdq_linear_score": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_void_p,
                                  c_void_p, c_void_p, c_void_p, c_int64, c_void_p, c_int64, POINTER(SvdqSeg), c_int,
                                  c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_int64, c_int64, c_int64,
                                  c_void_p]),
    "svdq_linear_score_workspace_bytes": (c_size_t, [c_int]),
    "svdq_bits_lost": (c_int, [c_void_p, c_int64, c_int, c_void_p, c_int64, c_int, c_int64, c_void_p, c_void_p]),
    "svdq_lambda_grid": (c_int, [c_void_p, c_void_p, c_int64, c_void_p, c_int, c_void_p, c_void_p, c_void_p,
                                 c_void_p]),
    "svdq_mxfp8_sf_bytes": (c_size_t, [c_int64, c_int64]),
    "svdq_quantize_mxfp8": (c_int, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p, c_void_p]),
    "svdq_linear_mxfp8": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int64,
                                  c_int64, c_int64, c_void_p]),
}

_lib = None


def load(path: str = None) -> ctypes.CDLL:
    """Load (once) and return the library with every signature declared."""
    global _lib
    if _lib is not None:
        return _lib
    if path is None:
        path = DEBUG_LIB_PATH if DEBUG else LIB_PATH
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python -m bit_w4a4_quantized_svdq_b200.build` "
            "(the CUDA library is the only implementation; there is no fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_text(status: int) -> str:
    return load().svdq_status_string(status).decode()


def check(call: str, status: int) -> None:
    if status != SVDQ_OK:
        raise SvdqError(call, status, status_text(status))
    if DEBUG:
        _debug_after(call)


# Debug mode: outputs the binding allocates sit between two guard bands of
# _GUARD bytes holding _GUARD_FILL; their bodies start as 0xFF bytes (NaN in
# every float format, so an element a call should write but does not shows).
_GUARD = 4096
_GUARD_FILL = 0xA5
_guarded = []


def out_empty(shape, dtype, device):
    """Output buffer of a call: torch.empty, or in debug mode a guarded view
    (plain torch.empty while a CUDA graph is being captured)."""
    import torch
    if not DEBUG or torch.cuda.is_current_stream_capturing():
        return torch.empty(shape, dtype=dtype, device=device)
    shape = (shape,) if isinstance(shape, int) else tuple(shape)
    n = 1
    for d in shape:
        n *= int(d)
    n *= torch.empty((), dtype=dtype).element_size()
    buf = torch.full((n + 2 * _GUARD,), _GUARD_FILL, dtype=torch.uint8, device=device)
    body = buf[_GUARD:_GUARD + n]
    body.fill_(0xFF)
    _guarded.append(buf)
    return body.view(dtype).view(shape)


def _debug_after(call: str) -> None:
    """After a call in debug mode: wait for it, read (and clear) the device error
    word, and check the guard bands of the outputs allocated since the last call."""
    import torch
    if torch.cuda.is_current_stream_capturing():
        return
    torch.cuda.synchronize()
    code = c_uint32(0)
    st = load().svdq_device_error(None, ctypes.byref(code))
    bufs = list(_guarded)
    _guarded.clear()
    if st != SVDQ_OK:
        raise SvdqError(call, st, f"{status_text(st)} (device code {code.value:#x})", code=int(code.value))
    for b in bufs:
        if not (bool((b[:_GUARD] == _GUARD_FILL).all()) and bool((b[-_GUARD:] == _GUARD_FILL).all())):
            raise SvdqError(call, SVDQ_ERR_BOUNDS, "a guard band around an output was overwritten")


def seg_array(segs):
    """Host array of svdq_seg from [(begin, end), ...]; (None, 0) for None."""
    if segs is None:
        return None, 0
    arr = (SvdqSeg * len(segs))(*[SvdqSeg(int(b), int(e)) for b, e in segs])
    return arr, len(segs)
