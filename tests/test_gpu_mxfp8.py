"""The MXFP8 W8A8 variant on the GPU against the oracle (reading R19).

"MiniMax-H3 -- MXFP8 (weight-quantized, vLLM-Omni native layout)", section
"Quant format": E4M3 elements, one E8M0 scale per 32 elements, symmetric
round-to-nearest, activations quantised dynamically per 32.  Codes and scale
bytes are bit-exact (the scaling is by a power of two, so one E4M3 rounding of
an exact value decides each code); the linear is within the GEMM tolerances.
"""
import numpy as np
import pytest
import torch

import synthetic as S
from oracle import svdq_oracle as O
from gpu_util import check_linear_bf16, check_sf, dev_bits, host_bits, requires_cuda

pytestmark = [pytest.mark.gpu, requires_cuda]


@pytest.fixture(scope="module")
def lib():
    import bit_w4a4_quantized_svdq_b200 as P
    return P


def _x(m, k, seed, std=1.0):
    x = S.bf16_bits_to_f32(S.random_bf16((m, k), seed, std)).astype(np.float32)
    rng = np.random.default_rng(seed)
    if m > 3 and k >= 128:
        x[0, :32] = 0.0                                       # an all-zero block
        x[1, 32:64] *= np.float32(2.0 ** 100)                 # large exponents
        x[2, 64:96] *= np.float32(2.0 ** -130)                # subnormal block maximum: exponent -127
        x[3, :] = rng.choice([16.0, 17.0, 19.0, -17.0, 448.0, 480.0, -0.0], size=k)   # ties and saturation
    return S.f32_to_bf16_bits(x)


def _check_quant(q, x_bits):
    m, k = x_bits.shape
    codes, sc = O.mx_quantize(x_bits)
    got = q["codes"].cpu().numpy()
    mism = np.argwhere(got != codes)
    assert mism.size == 0, f"{len(mism)} code mismatches, first {mism[:4].tolist()}"
    check_sf(q["sf"], sc, m, (k // 32) * 16)                 # K / 32 scale columns (the helper counts 16 per scale)
    return codes, sc


@pytest.mark.parametrize("m,k", [(1, 128), (300, 640), (129, 384), (4096, 5120)])
def test_quantize_matches_oracle(lib, m, k):
    x_bits = _x(m, k, m + k)
    q = lib.svdq_quantize_mxfp8(dev_bits(x_bits))
    torch.cuda.synchronize()
    _check_quant(q, x_bits)


def test_quantize_strided_rows(lib):
    x_bits = _x(200, 768, 9)
    wide = torch.zeros((200, 1024), dtype=torch.int16, device="cuda")
    wide[:, :768] = dev_bits(x_bits)
    q = lib.svdq_quantize_mxfp8(wide[:, :768])
    _check_quant(q, x_bits)


@pytest.mark.parametrize("m,n,k", [(128, 256, 128), (300, 512, 640), (1000, 768, 1024), (4096, 1024, 5120)])
def test_linear_matches_oracle(lib, m, n, k):
    x_bits = _x(m, k, 3 * m + k)
    w_bits = S.random_bf16((n, k), n + k, 0.02)
    bias = S.random_bf16((n,), 7, 0.02)
    qa = lib.svdq_quantize_mxfp8(dev_bits(x_bits))
    qw = lib.svdq_quantize_mxfp8(dev_bits(w_bits))
    y = lib.svdq_linear_mxfp8(qa["codes"], qa["sf"], qw["codes"], qw["sf"], dev_bits(bias))
    torch.cuda.synchronize()
    a_c, a_s = _check_quant(qa, x_bits)
    w_c, w_s = _check_quant(qw, w_bits)
    y64 = O.mx_linear(a_c, a_s, w_c, w_s, bias)
    check_linear_bf16(host_bits(y), y64)
    # without a bias
    y0 = lib.svdq_linear_mxfp8(qa["codes"], qa["sf"], qw["codes"], qw["sf"], None)
    check_linear_bf16(host_bits(y0), O.mx_linear(a_c, a_s, w_c, w_s, None))
    assert lib.svdq_device_error() == 0


def test_linear_large_sampled(lib):
    # the attention-projection shape in the bench's launch configuration: every
    # row and column computed, the oracle on a sample of rows
    L = S.make_layer(1)
    qa = lib.svdq_quantize_mxfp8(dev_bits(L.x))
    qw = lib.svdq_quantize_mxfp8(dev_bits(L.w))
    y = lib.svdq_linear_mxfp8(qa["codes"], qa["sf"], qw["codes"], qw["sf"], dev_bits(L.bias))
    rows = np.random.default_rng(0).choice(L.x.shape[0], 96, replace=False)
    a_c, a_s = O.mx_quantize(L.x[rows])
    w_c, w_s = O.mx_quantize(L.w)
    np.testing.assert_array_equal(qa["codes"].cpu().numpy()[rows], a_c)
    check_linear_bf16(host_bits(y)[rows], O.mx_linear(a_c, a_s, w_c, w_s, L.bias))
    assert lib.svdq_device_error() == 0


def test_linear_repeatable_many_tiles(lib):
    """One 128-channel stage per tile (ring and scale slots reused at the fastest
    rate), many tiles per CTA: twenty calls are bitwise equal."""
    m, n, k = 5120, 5120, 128
    qa = lib.svdq_quantize_mxfp8(dev_bits(_x(m, k, 51)))
    qw = lib.svdq_quantize_mxfp8(dev_bits(S.random_bf16((n, k), 52, 0.02)))
    bias = dev_bits(S.random_bf16((n,), 53, 0.02))
    y0 = lib.svdq_linear_mxfp8(qa["codes"], qa["sf"], qw["codes"], qw["sf"], bias)
    for _ in range(20):
        y = lib.svdq_linear_mxfp8(qa["codes"], qa["sf"], qw["codes"], qw["sf"], bias)
        assert torch.equal(y.view(torch.int16), y0.view(torch.int16))
    assert lib.svdq_device_error() == 0
