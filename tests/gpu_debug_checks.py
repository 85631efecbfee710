"""The debug library's checks, made to fire without any store leaving its buffer.

These run only against the debug build (SVDQ_DEBUG=1: ``libsvdq_debug.so``,
and the binding reads the device error word and the guard bands of the outputs
it allocated after every call).  The file name keeps it out of the default
collection; test_gpu_debug_build.py names it explicitly in a child process.  For each output a test lowers the extent the kernel checks its stores
against (``svdq_debug_limit_extent``, one call) and checks that
  - the call reports SVDQ_ERR_BOUNDS with that output's code (0x100 + site),
  - where the test owns the output buffer: nothing at or past the lowered
    extent was written, and what lies below it equals an unarmed call's result.
The lowered extent is always inside the real buffer, so a store the check
failed to stop would still land in memory the test owns.
"""
import os

import numpy as np
import pytest
import torch

import synthetic as S
from gpu_util import dev_bits, dev_f32, requires_cuda

pytestmark = [pytest.mark.gpu, requires_cuda,
              pytest.mark.skipif(os.environ.get("SVDQ_DEBUG", "0") in ("", "0"),
                                 reason="debug-library checks: run with SVDQ_DEBUG=1")]

M, K, N, R = 300, 320, 384, 32          # ragged rows, K % 64, N % 128: several tiles, partial ones

SITE = dict(calib_zero=1, calib_amax=2, calib_lambda=3, codes=4, sf=5, d=6, linear_box=7, linear_f32=8,
            linear_score=9, score_part=10, score_out=11, residual=12, grid=13, bits=14, mx_codes=15, mx_sf=16)


@pytest.fixture(scope="module")
def P():
    import bit_w4a4_quantized_svdq_b200 as P
    assert P.load().svdq_debug_build() == 1, "the debug library must be the one loaded"
    return P


@pytest.fixture(scope="module")
def layer(P):
    x = dev_bits(S.random_bf16((M, K), 901, 1.0))
    w = dev_bits(S.random_bf16((N, K), 902, 0.05))
    bias = dev_bits(S.random_bf16((N,), 903, 0.1))
    down = dev_bits(S.random_bf16((R, K), 904, 0.05))
    up = dev_bits(S.random_bf16((N, R), 905, 0.05))
    cal = P.svdq_calib_lambda(x, None, w)
    res = P.svdq_residual(w, cal["lam"], down, up)
    wc = P.svdq_calib_lambda(res, None, None)
    wq = P.svdq_quantize_act(res, None, wc["s_g"])
    q = P.svdq_quantize_act(x, cal["inv_lam"], cal["s_g"], down)
    return dict(x=x, w=w, bias=bias, down=down, up=up, cal=cal, wq=wq, wsg=wc["s_g"], q=q)


def _armed(P, site, extent, fn):
    """Arm `site` at `extent`, run `fn`; the call must raise SVDQ_ERR_BOUNDS naming the site."""
    assert P.load().svdq_debug_limit_extent(site, extent) == 0
    with pytest.raises(P.SvdqError) as e:
        fn()
    assert e.value.status == P._lib.SVDQ_ERR_BOUNDS, str(e.value)
    assert e.value.code == 0x100 + site, hex(e.value.code)


def _filled(t):
    """Every byte 0xFF (the pattern a skipped store leaves)."""
    t.view(torch.uint8).fill_(0xFF)
    return t


def _bytes(t):
    return t.contiguous().view(torch.uint8).reshape(-1).cpu().numpy()


def _check_prefix(got, want, limit_bytes):
    """Bytes below the limit equal the unarmed result; bytes from it on were never written."""
    g, w = _bytes(got), _bytes(want)
    assert np.array_equal(g[:limit_bytes], w[:limit_bytes])
    assert np.all(g[limit_bytes:] == 0xFF), "a store past the lowered extent was made"


def test_calibration_sites(P, layer):
    x, w = layer["x"], layer["w"]
    _armed(P, SITE["calib_zero"], 0, lambda: P.svdq_calib_lambda(x, None, w))
    _armed(P, SITE["calib_amax"], K // 2, lambda: P.svdq_calib_lambda(x, None, w))
    _armed(P, SITE["calib_lambda"], K // 2, lambda: P.svdq_calib_lambda(x, None, w))
    P.svdq_calib_lambda(x, None, w)                     # unarmed: no report


def test_quantiser_sites(P, layer):
    x, cal, down = layer["x"], layer["cal"], layer["down"]
    want = P.svdq_quantize_act(x, cal["inv_lam"], cal["s_g"], down)

    def fresh():
        return dict(codes=_filled(torch.empty_like(want["codes"])), sf=_filled(torch.empty_like(want["sf"])),
                    d=_filled(torch.empty_like(want["d"])))

    for key, site, limit_elems, elem in (("codes", "codes", (M // 2) * (K // 2), 1),
                                         ("sf", "sf", want["sf"].numel() // 2, 1),
                                         ("d", "d", (M // 2) * R, 4)):
        out = fresh()
        _armed(P, SITE[site], limit_elems,
               lambda: P.svdq_quantize_act(x, cal["inv_lam"], cal["s_g"], down, out=out))
        _check_prefix(out[key], want[key], limit_elems * elem)


def _linear_args(L):
    q, wq = L["q"], L["wq"]
    return (q["codes"], q["sf"], L["cal"]["s_g"], q["d"], wq["codes"], wq["sf"], L["wsg"], L["up"], L["bias"])


def test_linear_sites(P, layer):
    args = _linear_args(layer)
    want = P.svdq_linear(*args)
    y = _filled(torch.empty_like(want))
    # Y's TMA boxes: columns from N / 2 on are not stored
    _armed(P, SITE["linear_box"], N // 2, lambda: P.svdq_linear(*args, out=y))
    g, wb = y.view(torch.int16).cpu().numpy(), want.view(torch.int16).cpu().numpy()
    assert np.array_equal(g[:, :N // 2], wb[:, :N // 2]) and np.all(g[:, N // 2:] == -1)
    # fp32 output: rows from M / 2 on are not stored
    want32 = P.svdq_linear(*args, out_dtype=torch.float32)
    y32 = _filled(torch.empty_like(want32))
    _armed(P, SITE["linear_f32"], (M // 2) * N, lambda: P.svdq_linear(*args, out_dtype=torch.float32, out=y32))
    _check_prefix(y32, want32, (M // 2) * N * 4)


def test_fused_and_standalone_scoring_sites(P, layer):
    args = _linear_args(layer)
    y = P.svdq_linear(*args)
    yref = dev_bits(S.random_bf16((M, N), 906, 0.5))
    segs = [(0, 100), (100, 300)]
    _armed(P, SITE["linear_score"], 0, lambda: P.svdq_linear_score(*args, yref=yref, segs=segs, write_out=False))
    _armed(P, SITE["score_part"], 0, lambda: P.svdq_score_lambda(y, yref, segs))
    _armed(P, SITE["score_out"], 1, lambda: P.svdq_score_lambda(y, yref, segs))
    # strided rows take the other scoring kernel
    big = dev_bits(np.zeros((M, N + 8), np.uint16))
    ys = big[:, :N]
    _armed(P, SITE["score_part"], 0, lambda: P.svdq_score_lambda(ys, ys, segs))


def test_weight_and_search_sites(P, layer):
    w, cal, down, up = layer["w"], layer["cal"], layer["down"], layer["up"]
    _armed(P, SITE["residual"], (N // 2) * K, lambda: P.svdq_residual(w, cal["lam"], down, up))
    alphas = dev_f32(np.array([0.3, 0.5, 0.7], np.float32))
    _armed(P, SITE["grid"], K, lambda: P.svdq_lambda_grid(cal["amax_x"], cal["amax_w"], alphas))
    g = P.svdq_lambda_grid(cal["amax_x"], cal["amax_w"], alphas)
    ax = torch.stack([cal["amax_x"], cal["amax_x"]])
    _armed(P, SITE["bits"], 1, lambda: P.svdq_bits_lost(ax, g["inv_lam"]))


def test_mxfp8_sites(P, layer):
    x = layer["x"][:, :256].contiguous()          # K % 128
    want = P.svdq_quantize_mxfp8(x)
    for key, site, limit in (("codes", "mx_codes", (M // 2) * 256), ("sf", "mx_sf", want["sf"].numel() // 2)):
        out = dict(codes=_filled(torch.empty_like(want["codes"])), sf=_filled(torch.empty_like(want["sf"])))
        _armed(P, SITE[site], limit, lambda: P.svdq_quantize_mxfp8(x, out=out))
        _check_prefix(out[key], want[key], limit)


def test_host_pointer_is_refused_before_launch(P, layer):
    """A host buffer where device memory is required: the debug build's pointer
    check refuses the call before anything is launched (the release build would
    hand the pointer to the kernel)."""
    raw = P.load()
    assert raw.svdq_debug_build() == 1
    q, cal = layer["q"], layer["cal"]
    raw_host = np.zeros(M * (K // 2) + 256, np.uint8)
    skip = (-raw_host.ctypes.data) % 256                 # 256-byte aligned: only the pointer check can refuse it
    host_codes = raw_host[skip:skip + M * (K // 2)]
    st = raw.svdq_quantize_act(layer["x"].data_ptr(), M, K, K, cal["inv_lam"].data_ptr(), cal["s_g"].data_ptr(),
                               None, 0, host_codes.ctypes.data, q["sf"].data_ptr(), None, None, None)
    assert st == P._lib.SVDQ_ERR_INVALID_ARG
    assert not host_codes.any()


def test_guard_band_check_reports_an_overwrite(P, layer):
    """The binding's guard-band check itself: an output whose guard band no
    longer holds its fill byte is reported after the call that allocated it."""
    from bit_w4a4_quantized_svdq_b200 import _lib
    orig = _lib.out_empty

    def spoiled(shape, dtype, device):
        t = orig(shape, dtype, device)
        _lib._guarded[-1][-1] = 0        # the last byte of the trailing guard band
        return t

    _lib.out_empty = spoiled
    try:
        with pytest.raises(P.SvdqError, match="guard band"):
            P.svdq_calib_lambda(layer["x"], None, None)
    finally:
        _lib.out_empty = orig
    P.svdq_calib_lambda(layer["x"], None, None)
