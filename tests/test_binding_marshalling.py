"""The Python binding's marshalling, on CPU: each op's body runs against a
recording stand-in for the library, with the argument forms the layer and the
GPU tests use, and the C call must receive the right pointers, sizes and
strides in the order ``include/svdq.h`` declares.  Only the size functions of
the real library are called (host code); nothing is launched.
"""
import numpy as np
import pytest
import torch

import synthetic as S
from bit_w4a4_quantized_svdq_b200 import _lib, ops

_HOST_CALLS = ("svdq_sf_bytes", "svdq_mxfp8_sf_bytes", "svdq_score_workspace_bytes",
               "svdq_linear_score_workspace_bytes", "svdq_status_string")


class _Recorder:
    """Stands in for the loaded library: records every entry-point call."""

    def __init__(self, real):
        self.real = real
        self.calls = []

    def __getattr__(self, name):
        if name in _HOST_CALLS:
            return getattr(self.real, name)

        def call(*args):
            self.calls.append((name, args))
            return _lib.SVDQ_OK
        return call


@pytest.fixture
def rec(monkeypatch):
    r = _Recorder(_lib.load())
    monkeypatch.setattr(_lib, "load", lambda path=None: r)
    monkeypatch.setattr(_lib, "out_empty", lambda shape, dtype, device: torch.empty(shape, dtype=dtype))
    monkeypatch.setattr(ops, "_stream", lambda stream: None)

    def check_bf16_host(t, name):            # the dtype part of the check; the device part needs a GPU
        if t.dtype not in ops._BF16_TYPES:
            raise TypeError(name)
    monkeypatch.setattr(ops, "_check_bf16", check_bf16_host)
    return r


def _bits(shape, seed, scale=1.0):
    return torch.from_numpy(np.ascontiguousarray(S.random_bf16(shape, seed, scale)).view(np.int16))


def _p(t):
    return t.data_ptr()


def test_quantize_act_arguments(rec):
    m, k, r = 130, 128, 16
    x, down = _bits((m, k), 1), _bits((r, k), 2)
    inv, s_g, sat = torch.ones(k), torch.ones(1), torch.zeros(1, dtype=torch.int32)
    q = ops.svdq_quantize_act.__wrapped__(x, inv, s_g, down, sat_count=sat)
    name, a = rec.calls[-1]
    assert name == "svdq_quantize_act"
    assert a == (_p(x), m, k, k, _p(inv), _p(s_g), _p(down), r, _p(q["codes"]), _p(q["sf"]), _p(q["d"]), _p(sat),
                 None)
    assert q["codes"].shape == (m, k // 2) and q["sf"].numel() == 256 * k // 16 and q["d"].shape == (m, r)
    # a row of a candidate grid as 1/lambda and a 0-dim tensor scale (the lambda search's forms),
    # rows with a stride above K, and the caller's own output buffers
    grid_inv, grid_sg = torch.ones((3, k)), torch.ones(3)
    wide = torch.zeros((m, k + 64), dtype=torch.int16)
    ops.svdq_quantize_act.__wrapped__(wide[:, :k], grid_inv[1], grid_sg[1], None, out=dict(q, d=None))
    _, a = rec.calls[-1]
    assert a[1:4] == (m, k, k + 64) and a[4] == _p(grid_inv[1]) and a[7] == 0 and a[10] is None
    # refused before any call: down over another K, a float64 scale, a short 1/lambda, short outputs
    n_calls = len(rec.calls)
    for args, kw, err in (((x, inv, s_g, _bits((r, k + 64), 3)), {}, ValueError),
                          ((x, inv, torch.ones(1, dtype=torch.float64), down), {}, TypeError),
                          ((x, torch.ones(k - 1), s_g, down), {}, ValueError),
                          ((x, inv, s_g, down), {"out": dict(q, sf=q["sf"][:-1])}, ValueError),
                          ((x, inv, s_g, down), {"out": dict(q, d=None)}, ValueError)):
        with pytest.raises(err):
            ops.svdq_quantize_act.__wrapped__(*args, **kw)
    assert len(rec.calls) == n_calls


def _linear_operands(m, n, k, r):
    sfa, sfw = ops.sf_bytes(m, k), ops.sf_bytes(n, k)
    return (torch.zeros((m, k // 2), dtype=torch.uint8), torch.zeros(sfa, dtype=torch.uint8), torch.ones(1),
            torch.zeros((m, r)) if r else None, torch.zeros((n, k // 2), dtype=torch.uint8),
            torch.zeros(sfw, dtype=torch.uint8), torch.ones(1), _bits((n, r), 4) if r else None, _bits((n,), 5))


@pytest.mark.parametrize("r", [0, 32])
def test_linear_arguments(rec, r):
    m, n, k = 300, 384, 320
    args = _linear_operands(m, n, k, r)
    for dtype, code in ((torch.bfloat16, 0), (torch.float32, 1)):
        y = ops.svdq_linear.__wrapped__(*args, out_dtype=dtype)
        name, a = rec.calls[-1]
        assert name == "svdq_linear" and y.dtype == dtype and y.shape == (m, n)
        assert a == (_p(args[0]), _p(args[1]), _p(args[2]), _p(args[3]) if r else None, r, _p(args[4]),
                     _p(args[5]), _p(args[6]), _p(args[7]) if r else None, _p(args[8]), _p(y), n, code, m, n, k, None)
    # an output that is a column slice of a wider buffer: its row stride goes to the call
    big = torch.empty((m, n + 128), dtype=torch.bfloat16)
    ops.svdq_linear.__wrapped__(*args, out=big[:, :n])
    assert rec.calls[-1][1][11] == n + 128
    with pytest.raises(ValueError):
        ops.svdq_linear.__wrapped__(*args, out=torch.empty((m, n), dtype=torch.float16))


def test_linear_score_arguments(rec):
    m, n, k, r = 300, 512, 512, 16
    args = _linear_operands(m, n, k, r)
    yref = _bits((m, n), 6)
    segs = [(0, 7), (7, 290), (290, 300)]
    out, num, den, rel = ops.svdq_linear_score.__wrapped__(*args, yref=yref, segs=segs, write_out=False)
    name, a = rec.calls[-1]
    assert name == "svdq_linear_score" and out is None
    assert a[10] is None and a[11] == n                      # no output, its stride unused
    assert a[12] == _p(yref) and a[13] == n and a[15] == 3
    assert [(s.begin, s.end) for s in a[14]] == segs
    assert a[16:19] == (_p(num), _p(den), _p(rel)) and a[20] == ops.linear_score_workspace_bytes(3)
    assert a[21:] == (m, n, k, None)
    y = torch.empty((m, n), dtype=torch.bfloat16)
    out, *_ = ops.svdq_linear_score.__wrapped__(*args, yref=yref, segs=segs, out=y)
    assert out is y and rec.calls[-1][1][10] == _p(y)


def test_residual_and_mxfp8_arguments(rec):
    n, k, r = 256, 384, 32
    w, lam, down, up = _bits((n, k), 7), torch.ones(k), _bits((r, k), 8), _bits((n, r), 9)
    res = ops.svdq_residual.__wrapped__(w, lam, down, up)
    assert rec.calls[-1] == ("svdq_residual", (_p(w), n, k, k, _p(lam), _p(down), _p(up), r, _p(res), None))
    with pytest.raises(ValueError):
        ops.svdq_residual.__wrapped__(w, lam, down, _bits((n, 16), 10))        # up's rank differs from down's
    m = 200
    x = _bits((m, k), 11)
    qa = ops.svdq_quantize_mxfp8.__wrapped__(x)
    assert rec.calls[-1] == ("svdq_quantize_mxfp8", (_p(x), m, k, k, _p(qa["codes"]), _p(qa["sf"]), None))
    qw = ops.svdq_quantize_mxfp8.__wrapped__(w)
    bias = _bits((n,), 12)
    y = ops.svdq_linear_mxfp8.__wrapped__(qa["codes"], qa["sf"], qw["codes"], qw["sf"], bias)
    assert rec.calls[-1] == ("svdq_linear_mxfp8", (_p(qa["codes"]), _p(qa["sf"]), _p(qw["codes"]), _p(qw["sf"]),
                                                   _p(bias), _p(y), n, m, n, k, None))
    with pytest.raises(ValueError):
        ops.svdq_linear_mxfp8.__wrapped__(qa["codes"], qa["sf"], qw["codes"], qw["sf"][:-16], bias)  # W's scales short
