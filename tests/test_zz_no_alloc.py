"""The scoring entry point that allocates nothing (svdq_score_lambda_static).

It exists for callers that cannot allocate device memory while they score --
a framework whose memory pool forbids side allocations, a launch sequence
whose buffers were fixed beforehand, a plugin handed only its input and output
tensors.  Its partial sums live in a fixed array inside the library, so its
results must equal those of svdq_score_lambda with a caller workspace bit for
bit (both run the same kernels in the same reduction order), call after call,
whatever an earlier call left in the shared array -- on the streaming path
(rows back to back) and on the per-block path (padded rows).

This file is named to be collected last: a run that stops at the first failure
has then already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import synthetic as S
from bit_w4a4_quantized_svdq_b200 import _lib
from gpu_util import dev_bits, requires_cuda


def _call_static(lib, yq, yref, segs, n=None):
    m, ld = yq.shape
    n = ld if n is None else n
    arr, n_seg = _lib.seg_array(segs)
    out = [torch.empty(n_seg, dtype=torch.float64, device="cuda") for _ in range(3)]
    st = lib.svdq_score_lambda_static(yq.data_ptr(), yref.data_ptr(), m, n, ld, arr, n_seg,
                                      out[0].data_ptr(), out[1].data_ptr(), out[2].data_ptr(),
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == _lib.SVDQ_OK, _lib.status_text(st)
    return [t.cpu().numpy() for t in out]


def _call_workspace(lib, yq, yref, segs, n=None):
    m, ld = yq.shape
    n = ld if n is None else n
    arr, n_seg = _lib.seg_array(segs)
    ws = torch.empty(max(256, lib.svdq_score_workspace_bytes(arr, n_seg, n)), dtype=torch.uint8, device="cuda")
    out = [torch.empty(n_seg, dtype=torch.float64, device="cuda") for _ in range(3)]
    st = lib.svdq_score_lambda(yq.data_ptr(), yref.data_ptr(), m, n, ld, arr, n_seg,
                               out[0].data_ptr(), out[1].data_ptr(), out[2].data_ptr(),
                               ws.data_ptr(), ws.numel(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == _lib.SVDQ_OK, _lib.status_text(st)
    return [t.cpu().numpy() for t in out]


def _pair(m, n, seed):
    yref = S.random_bf16((m, n), seed, 1.0)
    noise = S.random_bf16((m, n), seed + 1, 0.05)
    yq = S.f32_to_bf16_bits(S.bf16_bits_to_f32(yref) + S.bf16_bits_to_f32(noise))
    return dev_bits(yq), dev_bits(yref)


@pytest.mark.gpu
@requires_cuda
def test_static_scratch_score_matches_workspace_score_on_consecutive_calls():
    lib = _lib.load()
    # first call: a larger problem fills many slots of the shared array
    yq, yref = _pair(4096, 1024, 31)
    segs1 = [(0, 29), (29, 4068), (4068, 4096)]
    a = _call_static(lib, yq, yref, segs1)
    b = _call_workspace(lib, yq, yref, segs1)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    # second call right after: a smaller problem must not see the first call's partial sums
    yq2, yref2 = _pair(300, 512, 77)
    segs2 = [(0, 100), (100, 300)]
    a2 = _call_static(lib, yq2, yref2, segs2)
    b2 = _call_workspace(lib, yq2, yref2, segs2)
    for x, y in zip(a2, b2):
        assert np.array_equal(x, y)
    assert np.all(a2[2] > 0.01) and np.all(a2[2] < 0.2)
    # third: padded rows (row stride 504 > 500 columns) take the per-block kernel and its
    # final sum, again right after a larger call left the array full of other sums
    _call_static(lib, yq, yref, segs1)
    yq3, yref3 = _pair(600, 504, 91)
    segs3 = [(0, 7), (7, 590), (590, 600)]
    a3 = _call_static(lib, yq3, yref3, segs3, n=500)
    b3 = _call_workspace(lib, yq3, yref3, segs3, n=500)
    for x, y in zip(a3, b3):
        assert np.array_equal(x, y)
    assert np.all(a3[2] > 0.01) and np.all(a3[2] < 0.2)


def test_static_scratch_rejects_problems_beyond_its_size():
    """Checked before anything touches a device: no GPU needed."""
    lib = _lib.load()
    p = ctypes.c_void_p(0x10000)
    n = 16384
    rows = (lib.svdq_score_static_max_bytes() // 16 + 1)     # one block of 16384 elements per row
    arr, n_seg = _lib.seg_array([(0, rows)])
    st = lib.svdq_score_lambda_static(p, p, rows, n, n, arr, n_seg, p, p, p, None)
    assert st == _lib.SVDQ_ERR_SCRATCH_TOO_SMALL
    assert b"static scratch" in lib.svdq_status_string(st)
