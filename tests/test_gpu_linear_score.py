"""The linear with its scoring fused into the epilogue (svdq_linear_score).

The output must be the one svdq_linear writes, bit for bit, and the scores
those of the scoring definition ("MiniMax-H3 NVFP4 -- what the smoothing scale
should be calibrated on", section "The metric that picks the winner also hides
the cost") applied to that output: the oracle's fp64 scoring of the GPU's own
bf16 output is the reference, and the standalone scoring kernel agrees with it
to the rounding of its fp64 additions.
"""
import numpy as np
import pytest
import torch

import synthetic as S
from oracle import svdq_oracle as O
from gpu_util import dev_bits, dev_f32, host_bits, requires_cuda

pytestmark = [pytest.mark.gpu, requires_cuda]


@pytest.fixture(scope="module")
def lib():
    import bit_w4a4_quantized_svdq_b200 as P
    return P


def _operands(lib, x, w, bias, rank):
    """Quantised operands of the layer (oracle conversion, GPU activation quantisation)."""
    c = O.calib(x, None, w)
    conv = O.convert_weight(w, c["lam"], rank)
    s_ga = dev_f32(np.array([c["s_g"]]))
    s_gw = dev_f32(np.array([conv["s_g"]]))
    q = lib.svdq_quantize_act(dev_bits(x), dev_f32(c["inv_lam"]), s_ga, dev_bits(conv["down"]) if rank else None)
    wq_codes = torch.from_numpy(O.pack_codes(conv["codes"])).cuda()
    wq_sf = torch.from_numpy(O.sf_to_mma_layout(conv["sf"])).cuda()
    return (q["codes"], q["sf"], s_ga, q["d"], wq_codes, wq_sf, s_gw,
            dev_bits(conv["up"]) if rank else None, dev_bits(bias) if bias is not None else None)


def _rel_close(a, b, rtol=1e-12):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return np.all(np.abs(a - b) <= rtol * np.maximum(np.abs(b), 1e-300))


CASES = [
    # m, n, k, r, segments (half-open; overlapping, empty, tile-crossing, ragged tail)
    (300, 512, 512, 16, [(0, 7), (7, 290), (290, 300)]),
    (1, 256, 256, 0, [(0, 1)]),
    (513, 768, 1024, 32, [(0, 128), (100, 400), (400, 400), (450, 513)]),
    (4096, 1024, 512, 32, [(0, 29), (29, 4068), (4068, 4096)]),
    # several tiles per CTA, one 256-channel stage: the epilogue, not the main
    # loop, sets the pace, so the reference-strip ring turns over as fast as it can
    (2048, 5120, 256, 32, [(0, 1000), (1000, 2048)]),
    (4000, 5120, 256, 16, [(0, 4000), (17, 3001), (3001, 3001), (3500, 4000)]),
    (1536, 4096, 1024, 0, [(0, 1536)]),
    # ragged: N % 256 == 128 (the last tile's second column half lies past N) and
    # K % 256 == 64 (a last partial channel stage)
    (700, 1152, 1344, 32, [(0, 350), (350, 700)]),
]


@pytest.mark.parametrize("m,n,k,r,segs", CASES)
def test_output_and_scores(lib, m, n, k, r, segs):
    x = S.random_bf16((m, k), m + k, 1.0)
    w = S.random_bf16((n, k), n + k + 1, 0.02)
    bias = S.random_bf16((n,), 5, 0.02)
    args = _operands(lib, x, w, bias, r)
    # a reference output near the quantised one, as a bf16 layer output is
    noise = S.bf16_bits_to_f32(S.random_bf16((m, n), 7 * m + n, 0.01))
    yref_bits = S.f32_to_bf16_bits(S.bf16_bits_to_f32(host_bits(lib.svdq_linear(*args))) + noise)
    yref = dev_bits(yref_bits)

    y_sep = lib.svdq_linear(*args)
    y, num, den, rel = lib.svdq_linear_score(*args, yref=yref, segs=segs)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_sep.view(torch.int16)), "fused output differs from svdq_linear"

    # the oracle's exact fp64 scoring of this very output: fp32 differences and
    # squares summed in groups of 8, fp64 beyond, so each sum is within a relative
    # 1e-6 (2^-24 per operation over 8-term fp32 partials)
    n64, d64, r64 = O.score(host_bits(y), yref_bits, segs)
    np.testing.assert_allclose(num.cpu().numpy(), n64, rtol=1e-6, atol=0)
    np.testing.assert_allclose(den.cpu().numpy(), d64, rtol=1e-6, atol=0)
    np.testing.assert_allclose(rel.cpu().numpy(), r64, rtol=1e-6, atol=0)

    # the standalone scoring kernel on the written output: the same fp32 groups of
    # 8; the fused kernel adds a row's groups as exact fp32 pairs (within a few
    # units of 2^-48) and the rest in fp64, so the sums agree to ~1e-13
    sn, sd, sr = lib.svdq_score_lambda(y, yref, segs)
    assert _rel_close(num.cpu().numpy(), sn.cpu().numpy())
    assert _rel_close(den.cpu().numpy(), sd.cpu().numpy())

    # without writing the output: the same scores, bit for bit
    none, num2, den2, rel2 = lib.svdq_linear_score(*args, yref=yref, segs=segs, write_out=False)
    assert none is None
    assert torch.equal(num2, num) and torch.equal(den2, den) and torch.equal(rel2, rel)
    assert lib.svdq_device_error() == 0, "a bounded wait ran out"


def test_repeatable(lib):
    m, n, k, r = 640, 512, 512, 32
    x = S.random_bf16((m, k), 11, 1.0)
    w = S.random_bf16((n, k), 12, 0.02)
    args = _operands(lib, x, w, None, r)
    yref = dev_bits(S.random_bf16((m, n), 13, 0.5))
    segs = [(0, 100), (100, 640)]
    first = lib.svdq_linear_score(*args, yref=yref, segs=segs, write_out=False)
    for _ in range(3):
        again = lib.svdq_linear_score(*args, yref=yref, segs=segs, write_out=False)
        assert all(torch.equal(a, b) for a, b in zip(first[1:], again[1:]))
    assert lib.svdq_device_error() == 0


def test_repeatable_many_tiles(lib):
    # 40 x 20 tiles over the SMs, written and score-only calls alternating: every
    # call's scores and output are the same, and no bounded wait runs out
    m, n, k, r = 5120, 5120, 256, 32
    x = S.random_bf16((m, k), 31, 1.0)
    w = S.random_bf16((n, k), 32, 0.02)
    args = _operands(lib, x, w, None, r)
    yref = dev_bits(S.random_bf16((m, n), 33, 0.5))
    segs = [(0, 2500), (2500, 5120)]
    y0 = lib.svdq_linear(*args)
    first = lib.svdq_linear_score(*args, yref=yref, segs=segs)
    assert torch.equal(first[0].view(torch.int16), y0.view(torch.int16))
    for i in range(6):
        again = lib.svdq_linear_score(*args, yref=yref, segs=segs, write_out=bool(i & 1))
        assert all(torch.equal(a, b) for a, b in zip(first[1:], again[1:]))
        if i & 1:
            assert torch.equal(again[0].view(torch.int16), y0.view(torch.int16))
    assert lib.svdq_device_error() == 0


@pytest.mark.parametrize("k", [256, 512])
def test_plain_linear_repeatable_many_tiles(lib, k):
    """The plain linear, bf16 and fp32 output, at one and two 256-channel stages
    per tile (ring slots and scale slots reused at the fastest rate): twenty
    calls are bitwise equal.  A ring slot released while loads from it are still
    in flight shows up here as a 32-row block of one call that differs."""
    m, n, r = 5120, 5120, 32
    x = S.random_bf16((m, k), 41, 1.0)
    w = S.random_bf16((n, k), 42, 0.02)
    args = _operands(lib, x, w, S.random_bf16((n,), 43, 0.1), r)
    for out_dtype in (torch.bfloat16, torch.float32):
        y0 = lib.svdq_linear(*args, out_dtype=out_dtype)
        for _ in range(20):
            y = lib.svdq_linear(*args, out_dtype=out_dtype)
            assert torch.equal(y.view(torch.int32 if out_dtype == torch.float32 else torch.int16),
                               y0.view(torch.int32 if out_dtype == torch.float32 else torch.int16))
    assert lib.svdq_device_error() == 0


def test_rejects_bad_arguments(lib):
    m, n, k = 128, 256, 256
    x = S.random_bf16((m, k), 21, 1.0)
    w = S.random_bf16((n, k), 22, 0.02)
    args = _operands(lib, x, w, None, 0)
    yref = dev_bits(S.random_bf16((m, n), 23, 0.5))
    with pytest.raises(lib._lib.SvdqError):
        lib.svdq_linear_score(*args, yref=yref, segs=[(0, m + 1)])          # segment past M
    with pytest.raises(lib._lib.SvdqError):
        lib.svdq_linear_score(*args, yref=yref, segs=[(0, m)],
                              workspace=torch.empty(8, dtype=torch.uint8, device="cuda"))   # workspace too small
