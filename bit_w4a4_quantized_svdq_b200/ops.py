"""Python binding of the C ABI, one function per entry point, same names.

Argument marshalling only: torch tensors provide device memory and the
current CUDA stream; every computation runs in ``libsvdq.so``.  bf16 tensors
may be ``torch.bfloat16`` or raw ``int16``/``uint16`` bit patterns.

Every call runs on the device that holds its tensors: all tensor arguments
must share one CUDA device, which is made current for the call (the library
looks up its per-device state -- error word, SM count, static arrays -- on the
current device), and the default stream is that device's current stream.
"""
from __future__ import annotations

import functools
import inspect
from ctypes import byref, c_uint32
from typing import Optional, Sequence, Tuple

import torch

from . import _lib

Segs = Optional[Sequence[Tuple[int, int]]]


def _tensors_in(v):
    if isinstance(v, torch.Tensor):
        yield v
    elif isinstance(v, dict):
        for x in v.values():
            yield from _tensors_in(x)
    elif isinstance(v, (list, tuple)):
        for x in v:
            yield from _tensors_in(x)


def _on_tensor_device(fn):
    """Run ``fn`` with the device of its tensor arguments current.

    Raises ValueError when the tensors sit on more than one device, on a
    non-CUDA device, or when an explicit stream belongs to another device."""
    params = list(inspect.signature(fn).parameters)
    stream_pos = params.index("stream") if "stream" in params else None

    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        devs = {t.device for a in (*args, *kwargs.values()) for t in _tensors_in(a)}
        if not devs:
            return fn(*args, **kwargs)
        if len(devs) > 1:
            names = ", ".join(sorted(str(d) for d in devs))
            raise ValueError(f"{fn.__name__}: tensor arguments are on different devices ({names})")
        dev = devs.pop()
        if dev.type != "cuda":
            raise ValueError(f"{fn.__name__}: tensor arguments must be CUDA tensors, got {dev}")
        stream = kwargs.get("stream")
        if stream is None and stream_pos is not None and len(args) > stream_pos:
            stream = args[stream_pos]
        if stream is not None and stream.device != dev:
            raise ValueError(f"{fn.__name__}: stream is on {stream.device}, tensors on {dev}")
        with torch.cuda.device(dev):
            return fn(*args, **kwargs)

    return wrapper


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check_bf16(t: torch.Tensor, name: str) -> None:
    if t.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise TypeError(f"{name} must be bf16 (or its 16-bit pattern), got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


_BF16_TYPES = (torch.bfloat16, torch.int16, torch.uint16)


def _check_dense(t: Optional[torch.Tensor], dtypes, min_numel: int, name: str, optional: bool = False) -> None:
    """A dense (contiguous) tensor of one of `dtypes` holding at least `min_numel`
    elements: the kernels read such arguments through a bare pointer, so a wrong
    type or a short buffer is refused here rather than read past its end."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if t.dtype not in dtypes:
        want = " or ".join(str(d) for d in dtypes)
        raise TypeError(f"{name} must be {want}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() < min_numel:
        raise ValueError(f"{name} holds {t.numel()} elements, the call reads {min_numel}")


def _check_matrix(t: Optional[torch.Tensor], dtypes, rows: int, cols: int, name: str) -> None:
    """A contiguous [rows, cols] tensor of one of `dtypes` (None passes)."""
    if t is None:
        return
    _check_dense(t, dtypes, 0, name)
    if tuple(t.shape) != (rows, cols):
        raise ValueError(f"{name} must be [{rows}, {cols}], got {list(t.shape)}")


def _row_stride(t: torch.Tensor, name: str) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be a row-major 2-D tensor")
    return t.stride(0)


def sf_bytes(rows: int, k: int) -> int:
    return int(_lib.load().svdq_sf_bytes(rows, k))


@_on_tensor_device
def svdq_calib_lambda(x: torch.Tensor, segs: Segs = None, w: Optional[torch.Tensor] = None,
                      stream=None) -> dict:
    """Per-channel absmax, lambda, 1/lambda and the static tensor scale (device tensors)."""
    lib = _lib.load()
    _check_bf16(x, "x")
    m, k = x.shape
    ldx = _row_stride(x, "x")
    dev = x.device
    ax = _lib.out_empty(k, torch.float32, dev)
    aw = _lib.out_empty(k, torch.float32, dev) if w is not None else None
    lam = _lib.out_empty(k, torch.float32, dev)
    inv = _lib.out_empty(k, torch.float32, dev)
    s_g = _lib.out_empty(1, torch.float32, dev)
    if w is not None:
        _check_bf16(w, "w")
        n, ldw = w.shape[0], _row_stride(w, "w")
    else:
        n, ldw = 0, 0
    arr, n_seg = _lib.seg_array(segs)
    _lib.check("svdq_calib_lambda", lib.svdq_calib_lambda(
        _ptr(x), m, k, ldx, arr, n_seg, _ptr(w), n, ldw,
        _ptr(ax), _ptr(aw), _ptr(lam), _ptr(inv), _ptr(s_g), _stream(stream)))
    return dict(amax_x=ax, amax_w=aw, lam=lam, inv_lam=inv, s_g=s_g)


@_on_tensor_device
def svdq_calib_lambda_stored_w(x: torch.Tensor, segs: Segs, amax_w: torch.Tensor, stream=None) -> dict:
    """svdq_calib_lambda against a stored weight absmax (fp32 [K] device tensor): reads only x."""
    lib = _lib.load()
    _check_bf16(x, "x")
    m, k = x.shape
    ldx = _row_stride(x, "x")
    if amax_w.dtype != torch.float32 or amax_w.numel() != k or not amax_w.is_contiguous():
        raise ValueError("amax_w must be a contiguous float32 tensor of K values")
    dev = x.device
    ax = _lib.out_empty(k, torch.float32, dev)
    lam = _lib.out_empty(k, torch.float32, dev)
    inv = _lib.out_empty(k, torch.float32, dev)
    s_g = _lib.out_empty(1, torch.float32, dev)
    arr, n_seg = _lib.seg_array(segs)
    _lib.check("svdq_calib_lambda_stored_w", lib.svdq_calib_lambda_stored_w(
        _ptr(x), m, k, ldx, arr, n_seg, _ptr(amax_w), _ptr(ax), _ptr(lam), _ptr(inv), _ptr(s_g), _stream(stream)))
    return dict(amax_x=ax, amax_w=amax_w, lam=lam, inv_lam=inv, s_g=s_g)


@_on_tensor_device
def svdq_quantize_act(x: torch.Tensor, inv_lambda: Optional[torch.Tensor], s_g: torch.Tensor,
                      down: Optional[torch.Tensor] = None, sat_count: Optional[torch.Tensor] = None,
                      out: Optional[dict] = None, stream=None) -> dict:
    """NVFP4 codes, scale bytes (tensor-core layout) and D = x down^T."""
    lib = _lib.load()
    _check_bf16(x, "x")
    m, k = x.shape
    ldx = _row_stride(x, "x")
    r = 0 if down is None else int(down.shape[0])
    _check_dense(inv_lambda, (torch.float32,), k, "inv_lambda", optional=True)
    _check_dense(s_g, (torch.float32,), 1, "s_g")
    _check_matrix(down, _BF16_TYPES, r, k, "down")
    _check_dense(sat_count, (torch.int32, torch.uint32), 1, "sat_count", optional=True)
    dev = x.device
    if out is None:
        out = dict(codes=_lib.out_empty((m, k // 2), torch.uint8, dev),
                   sf=_lib.out_empty(sf_bytes(m, k), torch.uint8, dev),
                   d=_lib.out_empty((m, r), torch.float32, dev) if r else None)
    _check_dense(out["codes"], (torch.uint8,), m * (k // 2), "out['codes']")
    _check_dense(out["sf"], (torch.uint8,), sf_bytes(m, k), "out['sf']")
    _check_dense(out.get("d"), (torch.float32,), m * r, "out['d']", optional=r == 0)
    _lib.check("svdq_quantize_act", lib.svdq_quantize_act(
        _ptr(x), m, k, ldx, _ptr(inv_lambda), _ptr(s_g), _ptr(down), r,
        _ptr(out["codes"]), _ptr(out["sf"]), _ptr(out["d"]), _ptr(sat_count), _stream(stream)))
    return out


def _check_linear_operands(a_codes, a_sf, s_g_act, d, w_codes, w_sf, s_g_w, up, bias):
    """Shapes and types of the NVFP4 linear's operands; returns (m, n, k, r)."""
    if a_codes.dim() != 2 or w_codes.dim() != 2:
        raise ValueError("a_codes and w_codes must be 2-D [rows, K/2] byte tensors")
    m, kh = a_codes.shape
    n = w_codes.shape[0]
    k = 2 * kh
    _check_matrix(a_codes, (torch.uint8,), m, kh, "a_codes")
    _check_matrix(w_codes, (torch.uint8,), n, kh, "w_codes")
    _check_dense(a_sf, (torch.uint8,), sf_bytes(m, k), "a_sf")
    _check_dense(w_sf, (torch.uint8,), sf_bytes(n, k), "w_sf")
    _check_dense(s_g_act, (torch.float32,), 1, "s_g_act")
    _check_dense(s_g_w, (torch.float32,), 1, "s_g_w")
    r = 0 if d is None else int(d.shape[-1])
    if d is not None:
        _check_matrix(d, (torch.float32,), m, r, "d")
    if up is not None:
        _check_matrix(up, _BF16_TYPES, n, r, "up")
    _check_dense(bias, _BF16_TYPES, n, "bias", optional=True)
    return m, n, k, r


@_on_tensor_device
def svdq_linear(a_codes: torch.Tensor, a_sf: torch.Tensor, s_g_act: torch.Tensor, d: Optional[torch.Tensor],
                w_codes: torch.Tensor, w_sf: torch.Tensor, s_g_w: torch.Tensor, up: Optional[torch.Tensor],
                bias: Optional[torch.Tensor], out_dtype: torch.dtype = torch.bfloat16,
                out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Y = s_g_act s_g_w deq(A) deq(W)^T + D up^T + bias."""
    lib = _lib.load()
    m, n, k, r = _check_linear_operands(a_codes, a_sf, s_g_act, d, w_codes, w_sf, s_g_w, up, bias)
    if out is None:
        out = _lib.out_empty((m, n), out_dtype, a_codes.device)
    if out.dtype not in (torch.bfloat16, torch.float32) or out.dim() != 2 or tuple(out.shape) != (m, n):
        raise ValueError(f"out must be a bf16 or float32 [{m}, {n}] tensor")
    ldy = _row_stride(out, "out")
    code = {torch.bfloat16: 0, torch.float32: 1}[out.dtype]
    _lib.check("svdq_linear", lib.svdq_linear(
        _ptr(a_codes), _ptr(a_sf), _ptr(s_g_act), _ptr(d), r, _ptr(w_codes), _ptr(w_sf), _ptr(s_g_w),
        _ptr(up), _ptr(bias), _ptr(out), ldy, code, m, n, k, _stream(stream)))
    return out


def linear_score_workspace_bytes(n_seg: int) -> int:
    return int(_lib.load().svdq_linear_score_workspace_bytes(int(n_seg)))


@_on_tensor_device
def svdq_linear_score(a_codes: torch.Tensor, a_sf: torch.Tensor, s_g_act: torch.Tensor, d: Optional[torch.Tensor],
                      w_codes: torch.Tensor, w_sf: torch.Tensor, s_g_w: torch.Tensor, up: Optional[torch.Tensor],
                      bias: Optional[torch.Tensor], yref: torch.Tensor, segs: Sequence[Tuple[int, int]],
                      out: Optional[torch.Tensor] = None, write_out: bool = True,
                      workspace: Optional[torch.Tensor] = None, stream=None):
    """The bf16 linear and, in the same kernel, its per-segment (num, den, rel) against
    yref.  Returns (out or None, num, den, rel); write_out=False skips the output."""
    lib = _lib.load()
    _check_bf16(yref, "yref")
    m, n, k, r = _check_linear_operands(a_codes, a_sf, s_g_act, d, w_codes, w_sf, s_g_w, up, bias)
    if tuple(yref.shape) != (m, n):
        raise ValueError(f"yref must be [{m}, {n}], got {tuple(yref.shape)}")
    dev = a_codes.device
    if write_out and out is None:
        out = _lib.out_empty((m, n), torch.bfloat16, dev)
    if not write_out:
        out = None
    if out is not None and (out.dtype not in _BF16_TYPES or tuple(out.shape) != (m, n)):
        raise ValueError(f"out must be a bf16 [{m}, {n}] tensor")
    ldy = _row_stride(out, "out") if out is not None else n
    arr, n_seg = _lib.seg_array(segs)
    num = _lib.out_empty(n_seg, torch.float64, dev)
    den = _lib.out_empty(n_seg, torch.float64, dev)
    rel = _lib.out_empty(n_seg, torch.float64, dev)
    if workspace is None:
        workspace = _lib.out_empty(linear_score_workspace_bytes(n_seg), torch.uint8, dev)
    _lib.check("svdq_linear_score", lib.svdq_linear_score(
        _ptr(a_codes), _ptr(a_sf), _ptr(s_g_act), _ptr(d), r, _ptr(w_codes), _ptr(w_sf), _ptr(s_g_w),
        _ptr(up), _ptr(bias), _ptr(out), ldy, _ptr(yref), _row_stride(yref, "yref"), arr, n_seg,
        _ptr(num), _ptr(den), _ptr(rel), _ptr(workspace), workspace.numel() * workspace.element_size(),
        m, n, k, _stream(stream)))
    return out, num, den, rel


def score_workspace_bytes(segs: Sequence[Tuple[int, int]], n: int) -> int:
    arr, n_seg = _lib.seg_array(segs)
    return int(_lib.load().svdq_score_workspace_bytes(arr, n_seg, n))


@_on_tensor_device
def svdq_score_lambda(yq: torch.Tensor, yref: torch.Tensor, segs: Sequence[Tuple[int, int]],
                      workspace: Optional[torch.Tensor] = None, stream=None):
    """Per-segment (num, den, rel) fp64 device tensors."""
    lib = _lib.load()
    _check_bf16(yq, "yq")
    _check_bf16(yref, "yref")
    m, n = yq.shape
    ld = _row_stride(yq, "yq")
    if _row_stride(yref, "yref") != ld:
        raise ValueError("yq and yref must share a row stride")
    arr, n_seg = _lib.seg_array(segs)
    dev = yq.device
    num = _lib.out_empty(n_seg, torch.float64, dev)
    den = _lib.out_empty(n_seg, torch.float64, dev)
    rel = _lib.out_empty(n_seg, torch.float64, dev)
    need = score_workspace_bytes(segs, n)
    if workspace is None:
        workspace = _lib.out_empty(need, torch.uint8, dev)
    _lib.check("svdq_score_lambda", lib.svdq_score_lambda(
        _ptr(yq), _ptr(yref), m, n, ld, arr, n_seg, _ptr(num), _ptr(den), _ptr(rel),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    return num, den, rel


@_on_tensor_device
def svdq_score_lambda_static(yq: torch.Tensor, yref: torch.Tensor, segs: Sequence[Tuple[int, int]], stream=None):
    """svdq_score_lambda without a workspace: partial sums in the library's static array."""
    lib = _lib.load()
    _check_bf16(yq, "yq")
    _check_bf16(yref, "yref")
    m, n = yq.shape
    ld = _row_stride(yq, "yq")
    if _row_stride(yref, "yref") != ld:
        raise ValueError("yq and yref must share a row stride")
    arr, n_seg = _lib.seg_array(segs)
    dev = yq.device
    num = _lib.out_empty(n_seg, torch.float64, dev)
    den = _lib.out_empty(n_seg, torch.float64, dev)
    rel = _lib.out_empty(n_seg, torch.float64, dev)
    _lib.check("svdq_score_lambda_static", lib.svdq_score_lambda_static(
        _ptr(yq), _ptr(yref), m, n, ld, arr, n_seg, _ptr(num), _ptr(den), _ptr(rel), _stream(stream)))
    return num, den, rel


@_on_tensor_device
def svdq_residual(w: torch.Tensor, lam: Optional[torch.Tensor], down: Optional[torch.Tensor],
                  up: Optional[torch.Tensor], stream=None) -> torch.Tensor:
    """R = bf16(W diag(lambda) - (diag(lambda) down^T up^T)^T), computed in fp64."""
    lib = _lib.load()
    _check_bf16(w, "w")
    n, k = w.shape
    r = 0 if down is None else int(down.shape[0])
    _check_dense(lam, (torch.float32,), k, "lam", optional=True)
    _check_matrix(down, _BF16_TYPES, r, k, "down")
    _check_matrix(up, _BF16_TYPES, n, r, "up")
    out = _lib.out_empty((n, k), torch.bfloat16, w.device)
    _lib.check("svdq_residual", lib.svdq_residual(
        _ptr(w), n, k, _row_stride(w, "w"), _ptr(lam), _ptr(down), _ptr(up), r, _ptr(out), _stream(stream)))
    return out


@_on_tensor_device
def svdq_bits_lost(amax_x: torch.Tensor, inv_lambda: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Mean bits lost to the NVFP4 group scale, fp64 [n_cand, n_mod].

    amax_x: fp32 [n_mod, K] (or [K]) per-modality channel absmax; inv_lambda:
    fp32 [n_cand, K] (or [K]) candidate 1/lambda rows, None for lambda = 1."""
    lib = _lib.load()
    ax = amax_x if amax_x.dim() == 2 else amax_x.view(1, -1)
    if ax.dtype != torch.float32 or not ax.is_cuda or ax.stride(1) != 1:
        raise ValueError("amax_x must be a CUDA float32 tensor with unit column stride")
    n_mod, k = ax.shape
    il, n_cand, ld_lam = None, 1, k
    if inv_lambda is not None:
        il = inv_lambda if inv_lambda.dim() == 2 else inv_lambda.view(1, -1)
        if il.dtype != torch.float32 or not il.is_cuda or il.stride(1) != 1 or il.shape[1] != k:
            raise ValueError("inv_lambda must be a CUDA float32 [n_cand, K] tensor with unit column stride")
        n_cand, ld_lam = il.shape[0], il.stride(0)
    bits = _lib.out_empty((n_cand, n_mod), torch.float64, ax.device)
    _lib.check("svdq_bits_lost", lib.svdq_bits_lost(
        _ptr(ax), ax.stride(0), n_mod, _ptr(il), ld_lam, n_cand, k, _ptr(bits), _stream(stream)))
    return bits


@_on_tensor_device
def svdq_lambda_grid(amax_x: torch.Tensor, amax_w: torch.Tensor, alpha: torch.Tensor, stream=None) -> dict:
    """Candidate lambda, 1/lambda [n_alpha, K] and s_g [n_alpha] for every alpha (fp32 device tensors)."""
    lib = _lib.load()
    for t, name in ((amax_x, "amax_x"), (amax_w, "amax_w"), (alpha, "alpha")):
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or t.dim() != 1:
            raise ValueError(f"{name} must be a contiguous 1-D CUDA float32 tensor")
    k = amax_x.numel()
    if amax_w.numel() != k:
        raise ValueError("amax_x and amax_w differ in length")
    n = alpha.numel()
    dev = amax_x.device
    lam = _lib.out_empty((n, k), torch.float32, dev)
    inv = _lib.out_empty((n, k), torch.float32, dev)
    s_g = _lib.out_empty(n, torch.float32, dev)
    _lib.check("svdq_lambda_grid", lib.svdq_lambda_grid(
        _ptr(amax_x), _ptr(amax_w), k, _ptr(alpha), n, _ptr(lam), _ptr(inv), _ptr(s_g), _stream(stream)))
    return dict(lam=lam, inv_lam=inv, s_g=s_g)


def mxfp8_sf_bytes(rows: int, k: int) -> int:
    return int(_lib.load().svdq_mxfp8_sf_bytes(rows, k))


@_on_tensor_device
def svdq_quantize_mxfp8(x: torch.Tensor, out: Optional[dict] = None, stream=None) -> dict:
    """bf16 [M, K] -> dict(codes u8 [M, K] E4M3, sf u8 E8M0 scales in the tensor-core layout)."""
    lib = _lib.load()
    _check_bf16(x, "x")
    m, k = x.shape
    nbytes = mxfp8_sf_bytes(m, k)
    if nbytes == 0:
        raise ValueError("K must be a positive multiple of 128")
    if out is None:
        out = dict(codes=_lib.out_empty((m, k), torch.uint8, x.device),
                   sf=_lib.out_empty(nbytes, torch.uint8, x.device))
    _check_dense(out["codes"], (torch.uint8,), m * k, "out['codes']")
    _check_dense(out["sf"], (torch.uint8,), nbytes, "out['sf']")
    _lib.check("svdq_quantize_mxfp8", lib.svdq_quantize_mxfp8(
        _ptr(x), m, k, _row_stride(x, "x"), _ptr(out["codes"]), _ptr(out["sf"]), _stream(stream)))
    return out


@_on_tensor_device
def svdq_linear_mxfp8(a_codes: torch.Tensor, a_sf: torch.Tensor, w_codes: torch.Tensor, w_sf: torch.Tensor,
                      bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """Y bf16 [M, N] = dequant(A) dequant(W)^T + bias on the MXFP8 tensor-core path."""
    lib = _lib.load()
    if a_codes.dim() != 2 or w_codes.dim() != 2:
        raise ValueError("a_codes and w_codes must be 2-D [rows, K] byte tensors")
    m, k = a_codes.shape
    n = w_codes.shape[0]
    _check_matrix(a_codes, (torch.uint8,), m, k, "a_codes")
    _check_matrix(w_codes, (torch.uint8,), n, k, "w_codes")
    _check_dense(a_sf, (torch.uint8,), mxfp8_sf_bytes(m, k), "a_sf")
    _check_dense(w_sf, (torch.uint8,), mxfp8_sf_bytes(n, k), "w_sf")
    _check_dense(bias, _BF16_TYPES, n, "bias", optional=True)
    if out is None:
        out = _lib.out_empty((m, n), torch.bfloat16, a_codes.device)
    if out.dtype not in _BF16_TYPES or tuple(out.shape) != (m, n):
        raise ValueError(f"out must be a bf16 [{m}, {n}] tensor")
    _lib.check("svdq_linear_mxfp8", lib.svdq_linear_mxfp8(
        _ptr(a_codes), _ptr(a_sf), _ptr(w_codes), _ptr(w_sf), _ptr(bias), _ptr(out), _row_stride(out, "out"),
        m, n, k, _stream(stream)))
    return out


def svdq_device_error(stream=None) -> int:
    """Synchronise and return (then clear) the device error word: 0 = nothing
    recorded, 1..6 = a bounded wait ran out, 0x100 + site = a store the debug
    library found outside its output."""
    code = c_uint32(0)
    st = _lib.load().svdq_device_error(_stream(stream), byref(code))
    if st not in (_lib.SVDQ_OK, _lib.SVDQ_ERR_TIMEOUT, _lib.SVDQ_ERR_BOUNDS):
        _lib.check("svdq_device_error", st)
    return int(code.value)
