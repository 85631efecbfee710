"""Pins of the oracle's MXFP8 path (reading R19) against closed forms and torch.

"MiniMax-H3 -- MXFP8 (weight-quantized, vLLM-Omni native layout)", section
"Quant format": E4M3 elements, one E8M0 scale per 32 elements, symmetric
round-to-nearest, activations quantised dynamically per 32.
"""
import numpy as np
import torch

import synthetic as S
from oracle import svdq_oracle as O


def _bits(v):
    return S.f32_to_bf16_bits(np.asarray(v, np.float32))


def test_shared_exponent_closed_forms():
    amax = np.array([1.0, 448.0, 256.0, 255.0, 511.0, 512.0, 0.0, 2.0 ** -130, 2.0 ** 127, 3.0 * 2 ** -20])
    # floor(log2): 0, 8, 8, 7, 8, 9, -, -130, 127, -19
    assert O.mx_shared_exponent(amax).tolist() == [-8, 0, 0, -1, 0, 1, -127, -127, 119, -27]


def test_element_codes_match_torch_float8():
    # every value torch can convert without saturating: torch's own float8 rounding
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.uniform(-448, 448, 200000), rng.uniform(-1, 1, 100000) * 2.0 ** -6,
                        np.float32(np.arange(-448, 449, 0.25))]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(v), ref)


def test_saturation_sign_and_zero():
    assert O.e4m3_encode(np.float32([500.0, -1e6, 448.0, 464.0])).tolist() == [0x7E, 0xFE, 0x7E, 0x7E]
    assert O.e4m3_encode(np.float32([-0.0, 0.0, -2.0 ** -12])).tolist() == [0x80, 0x00, 0x80]
    # ties go to the even code: 17 lies halfway between 16 (0x58) and 18 (0x59)
    assert O.e4m3_encode(np.float32([17.0, 19.0])).tolist() == [0x58, 0x5A]


def test_representable_blocks_are_lossless():
    rng = np.random.default_rng(1)
    grid = O.e4m3_decode(np.arange(0x00, 0x7F, dtype=np.uint8))       # every finite magnitude
    for s in (-20, -3, 0, 5):
        v = rng.choice(grid, size=(4, 64)) * rng.choice([-1.0, 1.0], size=(4, 64))
        v[:, 0] = 448.0          # each block's amax is 448, so its exponent is s exactly
        v[:, 32] = -448.0
        x = v * 2.0 ** s
        codes, sc = O.mx_quantize(_bits(x))
        assert np.all(sc == s + 127)
        np.testing.assert_array_equal(O.mx_dequantize(codes, sc), x)


def test_rounding_error_bound():
    x = S.bf16_bits_to_f32(S.random_bf16((64, 256), 3, 2.0)).astype(np.float64)
    x[5, :32] = 0.0                                   # an all-zero block
    codes, sc = O.mx_quantize(_bits(x))
    assert np.all(sc[5, 0] == 0) and np.all(codes[5, :32] == 0)
    y = O.mx_dequantize(codes, sc)
    scale = np.repeat(np.exp2(sc.astype(np.float64) - 127.0), 32, axis=1)
    # a block's amax / 2^e lies in [256, 512): values above 448 saturate to exactly 448 * 2^e
    sat = np.abs(x) / scale > 448.0
    assert sat.any()
    np.testing.assert_array_equal(y[sat], np.sign(x[sat]) * 448.0 * scale[sat])
    # the rest: half an ulp of 3 mantissa bits in the normal range, half the subnormal step below it
    bound = np.maximum(np.abs(x) * 2.0 ** -4, scale * 2.0 ** -10)
    assert np.all(np.abs(y - x)[~sat] <= bound[~sat])


def test_linear_on_representable_inputs_is_a_plain_matmul():
    rng = np.random.default_rng(4)
    # magnitudes up to 28 = 1.75 * 2^4 and one 16 per block: the block exponent is -4 and
    # every value times 2^4 is an E4M3 value of at most 448, so nothing saturates or rounds
    grid = O.e4m3_decode(np.arange(0x20, 0x5F, dtype=np.uint8))
    a = rng.choice(grid, size=(24, 128)) * rng.choice([-1.0, 1.0], size=(24, 128))
    w = rng.choice(grid, size=(40, 128)) * rng.choice([-1.0, 1.0], size=(40, 128)) * 2.0 ** -7
    a[:, ::32] = 16.0
    w[:, ::32] = -16.0 * 2.0 ** -7
    a_c, a_s = O.mx_quantize(_bits(a))
    w_c, w_s = O.mx_quantize(_bits(w))
    np.testing.assert_array_equal(O.mx_linear(a_c, a_s, w_c, w_s, None), a @ w.T)
    b = _bits(rng.standard_normal(40))
    np.testing.assert_array_equal(O.mx_linear(a_c, a_s, w_c, w_s, b), a @ w.T + O.bf16_to_f64(b)[None, :])


def _golden_mx_blocks():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "mxfp8_blocks.txt")
    rows = []
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        vals, scale, codes = (part.split() for part in line.split("|"))
        parse = lambda t: float.fromhex(t) if "0x" in t else float(t)
        rows.append((np.array([parse(t) for t in vals], dtype=np.float32), int(scale[0], 16),
                     np.array([int(c, 16) for c in codes], dtype=np.uint8)))
    return rows


def test_golden_hand_worked_blocks():
    rows = _golden_mx_blocks()
    assert len(rows) == 4
    for x, scale, codes in rows:
        bits = S.f32_to_bf16_bits(x)
        np.testing.assert_array_equal(S.bf16_bits_to_f32(bits).astype(np.float32), x)   # the values are exact bf16
        got_codes, got_scale = O.mx_quantize(bits[None, :])
        assert int(got_scale[0, 0]) == scale
        np.testing.assert_array_equal(got_codes[0], codes)
