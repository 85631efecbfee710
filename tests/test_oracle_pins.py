"""Pins that hold the CPU oracle to something other than itself (CPU only).

Each test checks an oracle function against an independent fact: a generic
float-format rounding rule, torch's float8 conversion, exact rational brute
force, exactly representable inputs, full-rank reconstruction, or a reduction
identity.  A plausible slip anywhere in the oracle (wrong tie rule, dropped
term, transposed operand, wrong sign, wrong group index) fails one of them.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import svdq_oracle as O
import synthetic as S


def _f32_bits_range(lo: float, hi: float, stride: int) -> np.ndarray:
    a = np.float32(lo).view(np.uint32)
    b = np.float32(hi).view(np.uint32)
    return np.arange(a, b + 1, stride, dtype=np.uint32).view(np.float32)


def _neighbourhoods(points, ulps=300):
    out = []
    for p in points:
        c = np.float32(p).view(np.uint32).astype(np.int64)
        r = np.arange(max(c - ulps, 0), c + ulps + 1, dtype=np.int64).astype(np.uint32)
        out.append(r.view(np.float32))
    return np.concatenate(out)


# --------------------------------------------------------------------------
# E2M1
# --------------------------------------------------------------------------

def _e2m1_generic_round(q: np.ndarray) -> np.ndarray:
    """Round |q| in a float format with one mantissa bit and minimum exponent 0.

    Spacing in binade [2^e, 2^(e+1)) is 2^(e-1); below 1 the (subnormal)
    spacing is 0.5.  np.rint rounds halves to even, i.e. ties go to an even
    mantissa.  Results above the largest finite value (6) saturate.
    """
    mag = np.minimum(np.abs(q.astype(np.float64)), 8.0)   # anything above 8 saturates anyway
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(mag > 0, mag, 1.0)))
    e = np.maximum(e, 0.0)
    spacing = np.exp2(e - 1.0)
    r = np.rint(mag / spacing) * spacing
    return np.minimum(r, 6.0)


def test_e2m1_decode_closed_form():
    for code in range(16):
        s, e, m = code >> 3, (code >> 1) & 3, code & 1
        v = 0.5 * m if e == 0 else 2.0 ** (e - 1) * (1 + 0.5 * m)
        assert O.e2m1_decode(np.array([code], np.uint8))[0] == (-v if s else v)


def test_e2m1_encode_matches_generic_format_rounding():
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0, 0.5, 1.0, 2.0, 3.0, 4.0]
    q = np.concatenate([_f32_bits_range(0.0, 16.0, 97), _neighbourhoods(mids),
                        np.array([0.0, 6.0, 1e30, np.inf, 1e-45], np.float32)])
    q = np.concatenate([q, -q])
    codes = O.e2m1_encode(q)
    got = np.abs(O.e2m1_decode(codes))
    want = _e2m1_generic_round(q)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (q[bad[:5]], got[bad[:5]], want[bad[:5]])
    # the sign bit follows the sign of the input, zero included (reading R1)
    assert np.array_equal(codes >> 3, np.signbit(q).astype(np.uint8))


def test_e2m1_ties_go_to_even_codes():
    q = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    assert O.e2m1_encode(q).tolist() == [0, 2, 2, 4, 4, 6, 6]
    assert O.e2m1_encode(-np.float32(0.1)[None]).tolist() == [8]


# --------------------------------------------------------------------------
# E4M3
# --------------------------------------------------------------------------

def _torch_e4m3(t: np.ndarray) -> np.ndarray:
    return torch.from_numpy(t.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_decode_matches_torch():
    codes = np.arange(127, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    assert np.array_equal(O.e4m3_decode(codes), want.astype(np.float64))


def test_e4m3_encode_matches_torch_float8_conversion():
    vals = O.E4M3_VALUES
    mids = list((vals[1:] + vals[:-1]) / 2) + list(vals)
    t = np.concatenate([_f32_bits_range(0.0, 448.0, 211), _neighbourhoods(mids, 40),
                        np.array([0.0, 2.0 ** -10, 2.0 ** -9, 448.0], np.float32)])
    t = t[(t >= 0) & (t <= 448)]
    assert np.array_equal(O.e4m3_encode_nonneg(t), _torch_e4m3(t))


def test_e4m3_saturates_above_448():
    t = np.array([448.0001, 464.0, 480.0, 1e6, np.inf], np.float32)
    assert np.all(O.e4m3_encode_nonneg(t) == 0x7E)


# --------------------------------------------------------------------------
# Block quantisation: exact rational brute force on tiny blocks
# --------------------------------------------------------------------------

def _brute_block(xs: np.ndarray, s_g: np.float32):
    """Quantise one 16-block by exhaustive search in exact rational arithmetic.

    The fp32 steps of the block scale (t, S, 1/S, xs * 1/S) follow the stated
    op sequence with numpy float32; every nearest-value decision enumerates
    all candidates with exact Fractions.
    """
    a = np.float32(np.max(np.abs(xs)))
    d = np.float32(np.float32(6) * s_g)
    t = np.float32(a / d)
    t_eff = Fraction(float(min(t, np.float32(448))))
    best = None
    for c in range(127):
        v = O.E4M3_VALUES[c]
        dist = abs(t_eff - Fraction(v))
        key = (dist, c % 2)          # smaller distance, then even code
        if best is None or key < best[0]:
            best = (key, c)
    sf = best[1]
    scale = np.float32(np.float32(O.E4M3_VALUES[sf]) * s_g)
    rs = np.float32(0) if scale == 0 else np.float32(np.float32(1) / scale)
    codes = []
    for x in xs:
        q = np.float32(x * rs)
        mag = Fraction(min(abs(float(q)), 6.0))
        bestc = None
        for c in range(8):
            key = (abs(mag - Fraction(O.E2M1_MAGNITUDES[c])), c % 2)
            if bestc is None or key < bestc[0]:
                bestc = (key, c)
        codes.append(bestc[1] | (8 if math.copysign(1.0, float(q)) < 0 else 0))
    return codes, sf


def _adversarial_blocks(rng):
    blocks = []
    blocks.append(np.full(16, 1.0))                       # all equal
    one = np.zeros(16); one[5] = -3.25; blocks.append(one)  # single non-zero
    blocks.append(np.zeros(16))                           # all zero
    # values sitting on E2M1 midpoints once scaled by the block max
    blocks.append(np.array([6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -0.25, -0.75,
                            -1.25, -1.75, -2.5, -3.5, -5, 0.1]) * 0.125)
    blocks.append(np.array([1e-3] * 8 + [-2e-3] * 8))     # tiny: subnormal / zero scales
    blocks.append(np.array([5e4] + [1.0] * 15))           # scale saturates at 448
    for _ in range(20):
        blocks.append(rng.standard_normal(16) * np.exp(rng.uniform(-6, 6)))
    return [S.f32_to_bf16_bits(np.asarray(b, np.float32)) for b in blocks]


@pytest.mark.parametrize("s_g", [1.0 / 448, 0.01, 3.7, 2.0 ** -12])
def test_quantize_blocks_bruteforce(s_g):
    rng = np.random.default_rng(7)
    s_g = np.float32(s_g)
    for bits in _adversarial_blocks(rng):
        codes, sf, _ = O.quantize_blocks(bits[None, :], None, s_g)
        want_codes, want_sf = _brute_block(S.bf16_bits_to_f32(bits), s_g)
        assert int(sf[0, 0]) == want_sf
        assert codes[0].tolist() == want_codes


def test_elements_are_multiplied_by_the_rounded_reciprocal():
    # Reading R4: q = RN32(x * RN32(1/S)), not RN32(x / S).  At s_g = 0.76333332
    # the block maximum 34.5 sets the scale byte 0x4F (7.5), S = RN32(7.5 s_g); for
    # 7.15625, 14.3125 and 28.625 the product lands one fp32 ulp above the E2M1
    # midpoints 1.25, 2.5 and 5 and rounds up (codes 3, 5, 7), while the quotient
    # rounds to the midpoint itself and would tie to the even codes 2, 4, 6.
    s_g = np.float32(0.7633333206176758)
    x = np.zeros(16, np.float32)
    x[:4] = [34.5, 7.15625, 14.3125, 28.625]
    bits = S.f32_to_bf16_bits(x)
    assert np.array_equal(S.bf16_bits_to_f32(bits), x)
    codes, sf, _ = O.quantize_blocks(bits[None, :], None, s_g)
    assert int(sf[0, 0]) == 0x4F and O.E4M3_VALUES[0x4F] == 7.5
    assert codes[0, 1:4].tolist() == [3, 5, 7]
    scale = np.float32(np.float32(7.5) * s_g)
    assert [int(O.e2m1_encode(np.array([np.float32(v / scale)]))[0]) for v in x[1:4]] == [2, 4, 6]
    want_codes, want_sf = _brute_block(x, s_g)
    assert codes[0].tolist() == want_codes and want_sf == 0x4F


def test_quantize_uses_the_group_of_16_consecutive_channels():
    # one large value per group: every group gets its own scale
    x = np.zeros((1, 64), np.float32)
    x[0, [3, 20, 40, 63]] = [1.0, 2.0, 4.0, 8.0]
    s_g = np.float32(0.25)
    codes, sf, _ = O.quantize_blocks(S.f32_to_bf16_bits(x), None, s_g)
    d = np.float32(6) * s_g
    want = _torch_e4m3(np.array([1.0, 2.0, 4.0, 8.0], np.float32) / d)
    assert sf[0].tolist() == want.tolist() and len(set(want.tolist())) == 4
    assert codes[0, 3] == 7 and codes[0, 20] == 7 and codes[0, 40] == 7 and codes[0, 63] == 7


def test_saturation_count():
    x = np.ones((2, 32), np.float32)
    x[1, 17] = 1e4          # second block of row 1 needs a scale above 448 at s_g = 1
    _, sf, n_sat = O.quantize_blocks(S.f32_to_bf16_bits(x), None, np.float32(1.0))
    assert n_sat == 1 and sf[1, 1] == 0x7E
    # a block whose scale is exactly 448 (absmax 2688 = 6 * 448 at s_g = 1) is not
    # saturated; the next bf16 value, 2704, needs 450.67 and is
    y = np.ones((1, 32), np.float32)
    y[0, 3], y[0, 20] = 2688.0, 2704.0
    _, sf, n_sat = O.quantize_blocks(S.f32_to_bf16_bits(y), None, np.float32(1.0))
    assert n_sat == 1 and sf[0].tolist() == [0x7E, 0x7E]


# --------------------------------------------------------------------------
# Exactly representable inputs: quantisation is lossless
# --------------------------------------------------------------------------

def _representable(rng, rows, k, s_g):
    """Rows whose 16-blocks are v_i * S exactly, with max |v_i| = 6 in each block."""
    v = O.E2M1_MAGNITUDES[rng.integers(0, 8, size=(rows, k))] * rng.choice([-1.0, 1.0], size=(rows, k))
    v = v.reshape(rows, k // 16, 16)
    v[:, :, 0] = np.where(v[:, :, 0] >= 0, 6.0, -6.0)     # force max |v| = 6 in every block
    sf = rng.integers(0x30, 0x58, size=(rows, k // 16)).astype(np.uint8)  # normal E4M3 scales
    scale = O.E4M3_VALUES[sf] * float(s_g)
    x = (v * scale[:, :, None]).reshape(rows, k)
    return x, sf


def test_exactly_representable_blocks_requantise_losslessly():
    rng = np.random.default_rng(3)
    s_g = np.float32(2.0 ** -5)
    x, sf_true = _representable(rng, 8, 128, s_g)
    bits = S.f32_to_bf16_bits(x)
    assert np.array_equal(S.bf16_bits_to_f32(bits).astype(np.float64), x)
    codes, sf, n_sat = O.quantize_blocks(bits, None, s_g)
    assert n_sat == 0 and np.array_equal(sf, sf_true)
    assert np.array_equal(O.dequantize(codes, sf) * float(s_g), x)


def test_linear_on_representable_inputs_equals_fp64_matmul():
    rng = np.random.default_rng(11)
    m, n, k = 24, 40, 96           # non-square, so a transposed operand cannot pass
    s_a, s_w = np.float32(2.0 ** -4), np.float32(2.0 ** -9)
    x, _ = _representable(rng, m, k, s_a)
    w, _ = _representable(rng, n, k, s_w)
    xb, wb = S.f32_to_bf16_bits(x), S.f32_to_bf16_bits(w)
    bias = S.random_bf16((n,), 5, 0.1)
    ca, sa, _ = O.quantize_blocks(xb, None, s_a)
    cw, sw, _ = O.quantize_blocks(wb, None, s_w)
    y = O.linear(ca, sa, s_a, cw, sw, s_w, bias_bits=bias)
    want = x @ w.T + S.bf16_bits_to_f32(bias).astype(np.float64)[None, :]
    assert np.array_equal(y, want)


# --------------------------------------------------------------------------
# Smoothing identity (page 1 "Why": the kernel sees X / lambda, the weight W * lambda)
# --------------------------------------------------------------------------

def test_smoothing_identity_with_blockwise_power_of_two_lambda():
    rng = np.random.default_rng(5)
    m, n, k = 16, 32, 128
    x = rng.standard_normal((m, k)).astype(np.float32)
    w = (0.02 * rng.standard_normal((n, k))).astype(np.float32)
    e = rng.integers(-2, 3, size=k // 16)
    lam = np.repeat(2.0 ** e, 16).astype(np.float32)       # constant within each group
    xb, wb = S.f32_to_bf16_bits(x), S.f32_to_bf16_bits(w)
    wl = S.f32_to_bf16_bits(w * lam[None, :])               # exact: power-of-two scaling
    # global scales chosen so every block scale stays a normal E4M3 value (no
    # saturation, no subnormal), the condition under which the identity is exact
    s_a, s_w = np.float32(0.01), np.float32(1e-3)
    ca0, sa0, _ = O.quantize_blocks(xb, None, s_a)
    cw0, sw0, _ = O.quantize_blocks(wb, None, s_w)
    ca1, sa1, _ = O.quantize_blocks(xb, (1 / lam).astype(np.float32), s_a)
    cw1, sw1, _ = O.quantize_blocks(wl, None, s_w)
    assert np.array_equal(ca0, ca1) and np.array_equal(cw0, cw1)
    y0 = O.linear(ca0, sa0, s_a, cw0, sw0, s_w)
    y1 = O.linear(ca1, sa1, s_a, cw1, sw1, s_w)
    assert np.array_equal(y0, y1)
    # exact-arithmetic identity on the unquantised path
    xf, wf = S.bf16_bits_to_f32(xb).astype(np.float64), S.bf16_bits_to_f32(wb).astype(np.float64)
    assert np.array_equal(xf @ wf.T, (xf / lam) @ (wf * lam).T)


def test_lambda_varying_inside_a_group_changes_the_codes():
    rng = np.random.default_rng(9)
    x = S.f32_to_bf16_bits(rng.standard_normal((4, 64)).astype(np.float32))
    lam = np.ones(64, np.float32)
    lam[1::2] = 4.0
    c0, s0, _ = O.quantize_blocks(x, None, np.float32(0.01))
    c1, s1, _ = O.quantize_blocks(x, (1 / lam).astype(np.float32), np.float32(0.01))
    assert not np.array_equal(c0, c1)


# --------------------------------------------------------------------------
# Low-rank branch and residual (page 3, opening section)
# --------------------------------------------------------------------------

def test_full_rank_branch_reconstructs_the_layer():
    rng = np.random.default_rng(21)
    m, n, k = 32, 48, 64
    x = S.f32_to_bf16_bits(rng.standard_normal((m, k)).astype(np.float32))
    w = S.f32_to_bf16_bits((0.02 * rng.standard_normal((n, k))).astype(np.float32))
    b = S.random_bf16((n,), 3, 0.02)
    c = O.calib(x, None, w)
    y_ref = O.reference_linear(x, w, b)
    rel = {}
    for r in (0, n):
        conv = O.convert_weight(w, c["lam"], r)
        y, _ = O.layer_forward(x, c["inv_lam"], c["s_g"], conv["down"] if r else None, conv, b)
        rel[r] = np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref)
    assert rel[n] < 2e-2 and rel[0] > 3 * rel[n]


def test_weight_tensor_scale_closed_form():
    # Reading R3 for weights: s_gW = max|R| / (6 * 448) of the 4-bit weight R; at
    # rank 0, R = W diag(lambda).  The largest |W lambda| is 10.5 * 2 = 21, so
    # s_gW = 21 / 2688 = 2^-7; that element's block scale is then exactly 448
    # (byte 0x7E, S = 3.5) and the element itself the largest E2M1 value, 6.
    rng = np.random.default_rng(4)
    w = (0.02 * rng.standard_normal((16, 32))).astype(np.float32)
    w[5, 7] = 10.5
    lam = np.ones(32, np.float32)
    lam[7] = 2.0
    conv = O.convert_weight(S.f32_to_bf16_bits(w), lam, 0)
    assert conv["s_g"] == np.float32(2.0 ** -7)
    assert conv["sf"][5, 0] == 0x7E and conv["codes"][5, 7] == 7


def test_lowrank_down_folds_lambda():
    rng = np.random.default_rng(4)
    x = S.f32_to_bf16_bits(rng.standard_normal((6, 32)).astype(np.float32))
    w = S.f32_to_bf16_bits((0.02 * rng.standard_normal((16, 32))).astype(np.float32))
    lam = np.float32(2.0) ** rng.integers(-2, 3, size=32).astype(np.float32)
    down, up = O.lowrank_factors(w, lam, 16)
    d = O.lowrank_down(x, down)
    xf = S.bf16_bits_to_f32(x).astype(np.float64)
    # (X / lambda) L1 with L1 = diag(lambda) down^T
    l1 = lam.astype(np.float64)[:, None] * S.bf16_bits_to_f32(down).astype(np.float64).T
    assert np.allclose(d, (xf / lam.astype(np.float64)) @ l1, rtol=0, atol=1e-12)


def test_residual_of_an_exactly_low_rank_weight_is_zero():
    rng = np.random.default_rng(8)
    n, k = 16, 32
    down = S.f32_to_bf16_bits(rng.choice([0.5, 1.0, -2.0, 0.25], size=(1, k)).astype(np.float32))
    up = S.f32_to_bf16_bits(rng.choice([1.0, -0.5, 2.0], size=(n, 1)).astype(np.float32))
    lam = np.float32(2.0) ** rng.integers(-2, 3, size=k).astype(np.float32)
    w = S.bf16_bits_to_f32(up).astype(np.float64) @ S.bf16_bits_to_f32(down).astype(np.float64)
    r = O.residual(S.f32_to_bf16_bits(w.astype(np.float32)), lam, down, up)
    assert np.all(S.bf16_bits_to_f32(r) == 0)


def test_zero_activations_give_zero_codes_and_bias_output():
    x = np.zeros((4, 64), np.uint16)
    codes, sf, n_sat = O.quantize_blocks(x, None, np.float32(0.3))
    assert not codes.any() and not sf.any() and n_sat == 0
    w = S.random_bf16((8, 64), 2, 0.02)
    cw, sw, _ = O.quantize_blocks(w, None, np.float32(1e-4))
    b = S.random_bf16((8,), 1, 0.1)
    y = O.linear(codes, sf, 0.3, cw, sw, 1e-4, bias_bits=b)
    assert np.array_equal(y, np.broadcast_to(S.bf16_bits_to_f32(b).astype(np.float64), y.shape))


# --------------------------------------------------------------------------
# Calibration (page 1 "Calibration"; page 2 "The activation scale bound held")
# --------------------------------------------------------------------------

def test_calib_lambda_closed_forms():
    x = np.zeros((3, 4), np.float32)
    w = np.zeros((2, 4), np.float32)
    x[:, 0] = [1, -16, 2]; w[:, 0] = [1, -0.5]           # 16 / 1  -> lambda 4
    x[:, 1] = [2, 0, 0];  w[:, 1] = [1, 0]               # 2 / 1   -> sqrt(2)
    x[:, 2] = 0;          w[:, 2] = [3, 1]               # zero activation column -> 1
    x[:, 3] = [0, 9, 0];  w[:, 3] = 0                    # zero weight column -> 1
    c = O.calib(S.f32_to_bf16_bits(x), None, S.f32_to_bf16_bits(w))
    assert c["lam"].tolist() == [4.0, np.float32(math.sqrt(2.0)), 1.0, 1.0]
    assert c["ax"].tolist() == [16.0, 2.0, 0.0, 9.0]
    assert c["inv_lam"][0] == 0.25
    # s_g = max(ax / lambda) / (6 * 448): max(4, 2/sqrt2, 0, 9) = 9, not max(ax) = 16
    assert c["s_g"] == np.float32(np.float32(9.0) / np.float32(2688.0))


def test_calib_row_segments_and_permutation():
    rng = np.random.default_rng(2)
    x = S.f32_to_bf16_bits(rng.standard_normal((50, 32)).astype(np.float32))
    w = S.random_bf16((8, 32), 3, 0.02)
    segs = [(0, 10), (30, 45)]
    c = O.calib(x, segs, w)
    sub = np.concatenate([x[0:10], x[30:45]])
    c2 = O.calib(sub[rng.permutation(len(sub))], None, w)
    for key in ("ax", "lam", "inv_lam"):
        assert np.array_equal(c[key], c2[key])
    assert c["s_g"] == c2["s_g"]


# --------------------------------------------------------------------------
# Scoring (page 1: rel-L2 against bf16 by row set)
# --------------------------------------------------------------------------

def test_score_identities():
    yref = S.random_bf16((40, 24), 6, 1.0)
    segs = [(0, 10), (10, 33), (33, 40)]
    num, den, rel = O.score(yref, yref, segs)
    assert np.all(num == 0) and np.all(rel == 0)
    twice = S.f32_to_bf16_bits(2 * S.bf16_bits_to_f32(yref))   # exact doubling
    num, den, rel = O.score(twice, yref, segs)
    assert np.array_equal(num, den) and np.all(rel == 1.0)
    n2, d2, r2 = O.score(twice, yref, segs[::-1])
    assert np.array_equal(n2[::-1], num) and np.array_equal(d2[::-1], den)


def test_score_closed_form_per_segment():
    # Yref = 1 everywhere; segment s adds d_s to every element of its rows (exact in
    # bf16), so num_s = rows_s * N * d_s^2, den_s = rows_s * N and rel_s = d_s.  A
    # segment that took a row of its neighbour, or lost one, changes its sums.
    n = 8
    segs = [(0, 3), (3, 7), (7, 12), (12, 12)]
    d = [0.5, 0.25, 2.0]
    yref = np.ones((12, n), np.float32)
    yq = yref.copy()
    for (b, e), ds in zip(segs, d):
        yq[b:e] += np.float32(ds)
    num, den, rel = O.score(S.f32_to_bf16_bits(yq), S.f32_to_bf16_bits(yref), segs)
    rows = [e - b for b, e in segs[:3]]
    assert num[:3].tolist() == [r * n * ds * ds for r, ds in zip(rows, d)]
    assert den[:3].tolist() == [float(r * n) for r in rows]
    assert rel[:3].tolist() == d
    # an empty segment: nothing to compare, rel 0 (both sums 0)
    assert (num[3], den[3], rel[3]) == (0.0, 0.0, 0.0)
    # a segment whose reference is all zero but whose output is not: rel is +inf
    z = np.zeros((2, n), np.float32)
    _, _, r_inf = O.score(S.f32_to_bf16_bits(z + 1), S.f32_to_bf16_bits(z), [(0, 2)])
    assert r_inf[0] == math.inf


# --------------------------------------------------------------------------
# Storage layouts
# --------------------------------------------------------------------------

def test_pack_codes_low_nibble_first():
    codes = np.array([[1, 2, 15, 8]], np.uint8)
    assert O.pack_codes(codes).tolist() == [[0x21, 0x8F]]
    assert np.array_equal(O.unpack_codes(O.pack_codes(codes)), codes)


def test_sf_layout_is_a_padded_bijection():
    m, k = 200, 320
    g = k // 16
    nat = (np.arange(m * g) % 251 + 1).astype(np.uint8).reshape(m, g)
    flat = O.sf_to_mma_layout(nat)
    assert flat.size == 256 * g
    assert np.array_equal(O.sf_from_mma_layout(flat, m, k), nat)
    offs = O.sf_layout_offsets(m, k)
    assert len(np.unique(offs)) == m * g
    # pad rows 200..255 stay zero
    assert np.count_nonzero(flat) == m * g
    # atom placement: row r of a 128-row block at (r%32)*16 + (r//32)*4, groups of 4 along K first
    assert offs[0, 0] == 0 and offs[1, 0] == 16 and offs[32, 0] == 4 and offs[0, 1] == 1
    assert offs[0, 4] == 512 and offs[128, 0] == (k // 64) * 512


# --------------------------------------------------------------------------
# Hand-worked blocks (tests/golden/nvfp4_blocks.txt)
# --------------------------------------------------------------------------

def _golden_blocks():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_blocks.txt")
    cases = []
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            s_g, xs, sf, codes = [p.strip() for p in line.split("|")]
            cases.append((float(s_g), [float(v) for v in xs.split()], int(sf, 16),
                          [int(c, 16) for c in codes.split()]))
    return cases


@pytest.mark.parametrize("case", _golden_blocks())
def test_golden_hand_worked_blocks(case):
    s_g, xs, sf, codes = case
    bits = S.f32_to_bf16_bits(np.array(xs, np.float32))[None, :]
    c, s, _ = O.quantize_blocks(bits, None, np.float32(s_g))
    assert int(s[0, 0]) == sf
    assert c[0].tolist() == codes
