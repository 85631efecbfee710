"""GPU parity: every kernel against the CPU oracle on the same seeded inputs.

Integer and byte results (absmax, lambda, tensor scales, packed codes, scale
bytes, the bf16 residual) must match bit for bit; floating-point outputs (D,
the layer output, scores) within the stated tolerances.
"""
import numpy as np
import pytest
import torch

import synthetic as S
from oracle import svdq_oracle as O
from gpu_util import (check_codes, check_d, check_linear_bf16, check_linear_f32, check_sf, dev_bits, dev_f32,
                      host_bits, requires_cuda, rel_l2)

pytestmark = [pytest.mark.gpu, requires_cuda]


@pytest.fixture(scope="module")
def lib():
    import bit_w4a4_quantized_svdq_b200 as P
    return P


# ---------------------------------------------------------------------------
# Config 0 (tiny W4A4 linear), full pipeline piece by piece
# ---------------------------------------------------------------------------

@pytest.fixture(scope="module")
def cfg0():
    L = S.make_layer(0)
    segs = L.seg_ranges(L.calib_sets["all"])
    c = O.calib(L.x, segs, L.w)
    conv = O.convert_weight(L.w, c["lam"], L.rank)
    return L, segs, c, conv


def test_calib_cfg0_bit_exact(lib, cfg0):
    L, segs, c, _ = cfg0
    g = lib.svdq_calib_lambda(dev_bits(L.x), segs, dev_bits(L.w))
    for key, gk in (("ax", "amax_x"), ("aw", "amax_w"), ("lam", "lam"), ("inv_lam", "inv_lam")):
        assert np.array_equal(g[gk].cpu().numpy(), c[key]), key
    assert g["s_g"].item() == float(c["s_g"])


@pytest.mark.parametrize("segs", [[(0, 0), (5, 9), (100, 256)], [(255, 256)], [(0, 256)], [(10, 10)]])
def test_calib_row_segments(lib, segs):
    x = S.random_bf16((256, 512), 12, 3.0)
    w = S.random_bf16((64, 512), 13, 0.02)
    c = O.calib(x, segs, w)
    g = lib.svdq_calib_lambda(dev_bits(x), segs, dev_bits(w))
    assert np.array_equal(g["amax_x"].cpu().numpy(), c["ax"])
    assert np.array_equal(g["lam"].cpu().numpy(), c["lam"])
    assert g["s_g"].item() == float(c["s_g"])


@pytest.mark.parametrize("segs", [None, [(0, 0), (5, 9), (100, 1000)], [(999, 1000)]])
def test_calib_stored_weight_absmax_equals_reading_the_weight(lib, segs):
    """The weight's absmax kept from one call over W gives the same lambda, 1/lambda
    and s_g as reading W again, bit for bit, and as the oracle."""
    x = S.random_bf16((1000, 1280), 31, 2.0)
    w = S.random_bf16((300, 1280), 32, 0.02)
    w_bits = w.copy()
    w_bits[:, 5] = 0                                   # a zero weight channel: lambda = 1 there
    c = O.calib(x, segs, w_bits)
    xd, wd = dev_bits(x), dev_bits(w_bits)
    full = lib.svdq_calib_lambda(xd, segs, wd)
    stored = lib.svdq_calib_lambda_stored_w(xd, segs, full["amax_w"])
    for key, gk in (("ax", "amax_x"), ("lam", "lam"), ("inv_lam", "inv_lam")):
        assert np.array_equal(stored[gk].cpu().numpy(), c[key]), key
        assert torch.equal(stored[gk], full[gk]), key
    assert stored["s_g"].item() == float(c["s_g"]) == full["s_g"].item()


@pytest.mark.parametrize("m,k", [(1, 8), (3, 72), (1000, 264)])
def test_calib_ragged_and_without_weight(lib, m, k):
    x = S.random_bf16((m, k), 21, 1.0)
    c = O.calib(x, None, None)
    g = lib.svdq_calib_lambda(dev_bits(x), None, None)
    assert np.array_equal(g["amax_x"].cpu().numpy(), c["ax"])
    assert np.all(g["lam"].cpu().numpy() == 1.0)
    assert g["s_g"].item() == float(c["s_g"])


def test_calib_all_zero_rows_give_unit_scales(lib):
    x = np.zeros((300, 1024), dtype=np.uint16)
    x[:, 7] = 0x8000                                   # negative zeros only
    w = S.random_bf16((64, 1024), 5, 0.02)
    c = O.calib(x, None, w)
    g = lib.svdq_calib_lambda(dev_bits(x), None, dev_bits(w))
    assert np.all(g["lam"].cpu().numpy() == 1.0) and np.all(c["lam"] == 1.0)
    assert g["s_g"].item() == 1.0 == float(c["s_g"])


def test_calib_wide_k_many_strips_and_repeated_calls(lib):
    """K = 20480 (the FFN down-projection width): 80 channel strips; two calls
    into recycled output memory must agree with the oracle both times."""
    x = S.random_bf16((300, 20480), 41, 2.0)
    w = S.random_bf16((96, 20480), 42, 0.02)
    segs = [(0, 7), (50, 299)]
    c = O.calib(x, segs, w)
    for _ in range(2):
        g = lib.svdq_calib_lambda(dev_bits(x), segs, dev_bits(w))
        for key, gk in (("ax", "amax_x"), ("aw", "amax_w"), ("lam", "lam"), ("inv_lam", "inv_lam")):
            assert np.array_equal(g[gk].cpu().numpy(), c[key]), key
        assert g["s_g"].item() == float(c["s_g"])
        del g


def test_quantize_cfg0_bit_exact(lib, cfg0):
    L, segs, c, conv = cfg0
    codes, sf, n_sat = O.quantize_blocks(L.x, c["inv_lam"], c["s_g"])
    sat = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = lib.svdq_quantize_act(dev_bits(L.x), dev_f32(c["inv_lam"]), dev_f32(np.array([c["s_g"]])),
                              dev_bits(conv["down"]), sat_count=sat)
    check_codes(q["codes"], codes)
    check_sf(q["sf"], sf, L.m, L.k)
    assert int(sat.item()) == n_sat
    d64 = O.lowrank_down(L.x, conv["down"])
    check_d(q["d"].cpu().numpy(), d64, L.x, conv["down"])


def _outlier_x(m, k, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((m, k)).astype(np.float32)
    x[:, rng.choice(k, size=max(1, k // 64), replace=False)] *= 40.0
    return S.f32_to_bf16_bits(x)


@pytest.mark.parametrize("m,k,r", [(1, 64, 0), (1, 64, 16), (129, 320, 32), (200, 512, 16), (300, 1024, 0),
                                   (128, 64, 32), (77, 1280, 32), (513, 4096, 16)])
def test_quantize_shapes(lib, m, k, r):
    x = _outlier_x(m, k, m * 7 + k)
    rng = np.random.default_rng(k)
    lam = np.exp(rng.uniform(-1.5, 1.5, size=k)).astype(np.float32)
    inv = (np.float32(1) / lam).astype(np.float32)
    s_g = np.float32(0.004)
    codes, sf, n_sat = O.quantize_blocks(x, inv, s_g)
    down = S.random_bf16((r, k), 5, 0.05) if r else None
    sat = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = lib.svdq_quantize_act(dev_bits(x), dev_f32(inv), dev_f32(np.array([s_g])),
                              dev_bits(down) if r else None, sat_count=sat)
    check_codes(q["codes"], codes)
    check_sf(q["sf"], sf, m, k)
    assert int(sat.item()) == n_sat
    if r:
        d64 = O.lowrank_down(x, down)
        check_d(q["d"].cpu().numpy(), d64, x, down)


def test_quantize_ties_saturation_and_signed_zero(lib):
    # Rows of hand-built groups: E2M1 midpoints, tiny groups (zero / subnormal
    # scales), saturating groups and signed zeros, at several tensor scales.
    base = np.array([6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5, -0.0],
                    np.float32)
    rows = []
    for e in range(-12, 10, 3):
        rows.append(np.concatenate([base * np.float32(2.0 ** e), -base * np.float32(2.0 ** e),
                                    np.full(16, np.float32(1e-30)), np.array([-0.0] * 16, np.float32)]))
    x = S.f32_to_bf16_bits(np.stack(rows))
    k = x.shape[1]
    for s_g in (np.float32(2.0 ** -8), np.float32(1 / 448), np.float32(1e-6), np.float32(3.0)):
        codes, sf, n_sat = O.quantize_blocks(x, None, s_g)
        sat = torch.zeros(1, dtype=torch.int32, device="cuda")
        q = lib.svdq_quantize_act(dev_bits(x), None, dev_f32(np.array([s_g])), None, sat_count=sat)
        check_codes(q["codes"], codes)
        check_sf(q["sf"], sf, x.shape[0], k)
        assert int(sat.item()) == n_sat


def _e4m3_boundaries():
    """The finite positive E4M3 values' rounding midpoints, and 448 (saturation)."""
    vals = sorted({float(O.e4m3_decode(np.array([b], np.uint8))[0]) for b in range(0x7F)})
    mids = [(a + b) / 2 for a, b in zip(vals[:-1], vals[1:])]
    return mids + [448.0]


def test_quantize_scale_near_every_e4m3_boundary(lib):
    """Group absmax a with a / (6 s_g) within +-4 fp32 ulps of each E4M3
    rounding midpoint and of 448: the scale byte, the codes and the saturation
    count must match the oracle's exact quotient bit for bit."""
    for s_g in (np.float32(1.0), np.float32(0.0123), np.float32(3.7e-5)):
        d = np.float64(np.float32(np.float32(6.0) * s_g))
        targets = []
        for m in _e4m3_boundaries():
            a0 = np.float32(m * d)
            bits = int(a0.view(np.uint32))
            targets += [np.uint32(bits + j).view(np.float32) for j in range(-4, 5)]   # +-4 fp32 steps
        g = len(targets)
        k = (g * 16 + 63) // 64 * 64
        inv = np.ones(k, np.float32)
        x = np.zeros((2, k), np.float32)
        for i, t in enumerate(targets):
            inv[16 * i] = t                      # xs = RN(1 * t) = t: the group's absmax
            x[0, 16 * i] = 1.0
            x[1, 16 * i] = -1.0
            x[:, 16 * i + 1] = 0.5               # a second, smaller element in every group
        xb = S.f32_to_bf16_bits(x)
        codes, sf, n_sat = O.quantize_blocks(xb, inv, s_g)
        sat = torch.zeros(1, dtype=torch.int32, device="cuda")
        q = lib.svdq_quantize_act(dev_bits(xb), dev_f32(inv), dev_f32(np.array([s_g])), None, sat_count=sat)
        check_codes(q["codes"], codes)
        check_sf(q["sf"], sf, 2, k)
        assert int(sat.item()) == n_sat


def test_quantize_repeatable_at_scale(lib):
    """Many CTAs, long rings: eight calls on a 20480 x 5120 input (with and
    without 1/lambda and the low-rank branch) give bitwise identical codes,
    scales and D, equal to the oracle on sampled rows.  Guards the ring's
    hand-over between quantiser teams, whose races show up only now and then."""
    m, k = 20480, 5120
    x = _outlier_x(m, k, 99)
    rng = np.random.default_rng(5)
    inv = (np.float32(1) / np.exp(rng.uniform(-1.0, 1.0, size=k)).astype(np.float32)).astype(np.float32)
    s_g = np.float32(0.02)
    down = S.random_bf16((32, k), 6, 0.05)
    rows = np.unique(np.concatenate([np.arange(0, m, 331), [m - 1]]))
    xd = dev_bits(x)
    for use_il, dn in ((False, None), (True, down)):
        il = dev_f32(inv) if use_il else None
        codes, sf, _ = O.quantize_blocks(x[rows], inv if use_il else None, s_g)
        first = None
        for _ in range(8):
            q = lib.svdq_quantize_act(xd, il, dev_f32(np.array([s_g])), dev_bits(dn) if dn is not None else None)
            got = (q["codes"].clone(), q["sf"].clone(), None if q["d"] is None else q["d"].clone())
            if first is None:
                first = got
                check_codes(q["codes"], codes, rows=rows)
                assert np.array_equal(O.sf_from_mma_layout(q["sf"].cpu().numpy(), m, k)[rows], sf)
            else:
                for a, b in zip(got, first):
                    assert (a is None and b is None) or torch.equal(a, b)


def test_quantize_zero_rows(lib):
    x = np.zeros((130, 128), np.uint16)
    q = lib.svdq_quantize_act(dev_bits(x), None, dev_f32(np.array([1.0])), dev_bits(S.random_bf16((16, 128), 1)))
    assert not q["codes"].any().item() and not q["sf"].any().item()
    assert not q["d"].any().item()


# ---------------------------------------------------------------------------
# Weight conversion: residual and its encoding
# ---------------------------------------------------------------------------

def test_residual_cfg0_bit_exact(lib, cfg0):
    L, _, c, conv = cfg0
    r = lib.svdq_residual(dev_bits(L.w), dev_f32(c["lam"]), dev_bits(conv["down"]), dev_bits(conv["up"]))
    got = host_bits(r)
    assert np.array_equal(got, conv["residual"])


def test_weight_encoding_cfg0_bit_exact(lib, cfg0):
    L, _, c, conv = cfg0
    rt = dev_bits(conv["residual"])
    wc = lib.svdq_calib_lambda(rt, None, None)
    assert wc["s_g"].item() == float(conv["s_g"])
    q = lib.svdq_quantize_act(rt, None, wc["s_g"])
    check_codes(q["codes"], conv["codes"])
    check_sf(q["sf"], conv["sf"], L.n, L.k)


# ---------------------------------------------------------------------------
# The fused W4A4 linear
# ---------------------------------------------------------------------------

def _linear_case(lib, x, w, bias, rank, seed=0):
    """Oracle conversion + forward; GPU forward from the same quantised operands."""
    c = O.calib(x, None, w)
    conv = O.convert_weight(w, c["lam"], rank)
    y64, parts = O.layer_forward(x, c["inv_lam"], c["s_g"], conv["down"] if rank else None, conv, bias)
    s_ga = dev_f32(np.array([c["s_g"]]))
    s_gw = dev_f32(np.array([conv["s_g"]]))
    q = lib.svdq_quantize_act(dev_bits(x), dev_f32(c["inv_lam"]), s_ga, dev_bits(conv["down"]) if rank else None)
    check_codes(q["codes"], parts["codes"])
    wq = dict(codes=torch.from_numpy(O.pack_codes(conv["codes"])).cuda(),
              sf=torch.from_numpy(O.sf_to_mma_layout(conv["sf"])).cuda())
    args = (q["codes"], q["sf"], s_ga, q["d"], wq["codes"], wq["sf"], s_gw,
            dev_bits(conv["up"]) if rank else None, dev_bits(bias) if bias is not None else None)
    y_bf = lib.svdq_linear(*args, out_dtype=torch.bfloat16)
    y_f32 = lib.svdq_linear(*args, out_dtype=torch.float32)
    return y64, host_bits(y_bf), y_f32.cpu().numpy()


def test_linear_cfg0(lib, cfg0):
    L = cfg0[0]
    y64, yb, yf = _linear_case(lib, L.x, L.w, L.bias, L.rank)
    check_linear_f32(yf, y64, tight_rel=1e-4)
    check_linear_bf16(yb, y64)


@pytest.mark.parametrize("m,n,k,r,bias", [
    (128, 256, 256, 0, True), (1, 256, 512, 16, True), (200, 512, 768, 32, False), (384, 256, 1024, 32, True),
    (300, 768, 512, 16, True), (129, 512, 2048, 0, False),
    (3200, 1024, 256, 32, True),      # 100 whole tiles: a last wave too full to split into half tiles
    # several tiles per CTA, each closed by its low-rank stage in the operand ring:
    # 2, 3, 4 and 12 ring positions per tile against the ring's 4 slots, and an odd
    # number of K stages (the last scale batch half past K)
    (8192, 2048, 256, 32, True), (2048, 4608, 512, 16, True), (1536, 6144, 768, 32, False),
    (2560, 4096, 2816, 32, True),
    # ragged N (a multiple of 128, not of 256) and K (a multiple of 64, not of 256)
    (300, 384, 320, 32, True), (129, 640, 576, 16, True), (2048, 1152, 1344, 32, False)])
def test_linear_shapes(lib, m, n, k, r, bias):
    x = _outlier_x(m, k, 3 * m + k)
    w = S.random_bf16((n, k), n + k, 0.02)
    b = S.random_bf16((n,), 4, 0.02) if bias else None
    y64, yb, yf = _linear_case(lib, x, w, b, r)
    check_linear_f32(yf, y64, tight_rel=1e-4)
    check_linear_bf16(yb, y64)


# ---------------------------------------------------------------------------
# Scoring
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("m,n", [(300, 512), (7, 264), (4096, 768)])
def test_score_matches_oracle(lib, m, n):
    yref = S.random_bf16((m, n), m + n, 1.0)
    noise = S.random_bf16((m, n), m * n, 0.05)
    yq = S.f32_to_bf16_bits(S.bf16_bits_to_f32(yref) + S.bf16_bits_to_f32(noise))
    segs = [(0, m // 3), (m // 3, m // 3), (m // 3, m), (0, m)]
    num, den, rel = O.score(yq, yref, segs)
    g = lib.svdq_score_lambda(dev_bits(yq), dev_bits(yref), segs)
    # fp32 differences/squares summed in groups of 8, fp64 beyond: relative error
    # of each sum well under 1e-6 (2^-24 per operation, 8-term fp32 partials)
    for a, b in zip(g, (num, den, rel)):
        np.testing.assert_allclose(a.cpu().numpy(), b, rtol=1e-6, atol=0)
    g2 = lib.svdq_score_lambda(dev_bits(yq), dev_bits(yref), segs)
    for a, b in zip(g, g2):
        assert torch.equal(a, b)      # fixed reduction order: bitwise reproducible


def test_score_row_strided_and_odd_width(lib):
    """Rows with a stride wider than N take the per-chunk kernel, back-to-back
    rows the streaming one; both reduce each chunk in the same order, so the
    results agree bit for bit.  N % 8 != 0 (scalar path, rows strided) against the oracle."""
    m, n, ld = 1000, 512, 576
    yref = S.random_bf16((m, ld), 17, 1.0)
    yq = S.f32_to_bf16_bits(S.bf16_bits_to_f32(yref) + S.bf16_bits_to_f32(S.random_bf16((m, ld), 18, 0.05)))
    segs = [(0, 13), (13, 990), (990, 1000)]
    wide_q, wide_r = dev_bits(yq), dev_bits(yref)
    strided = lib.svdq_score_lambda(wide_q[:, :n], wide_r[:, :n], segs)
    packed = lib.svdq_score_lambda(wide_q[:, :n].contiguous(), wide_r[:, :n].contiguous(), segs)
    for a, b in zip(strided, packed):
        assert torch.equal(a, b)
    num, den, rel = O.score(np.ascontiguousarray(yq[:, :n]), np.ascontiguousarray(yref[:, :n]), segs)
    np.testing.assert_allclose(packed[2].cpu().numpy(), rel, rtol=1e-6, atol=0)
    odd = 100                                 # rows stay 16-byte aligned through the stride
    g = lib.svdq_score_lambda(wide_q[:, :odd], wide_r[:, :odd], segs)
    q2, r2 = np.ascontiguousarray(yq[:, :odd]), np.ascontiguousarray(yref[:, :odd])
    for a, b in zip(g, O.score(q2, r2, segs)):
        np.testing.assert_allclose(a.cpu().numpy(), b, rtol=1e-6, atol=0)


def test_score_identities(lib):
    yref = S.random_bf16((64, 256), 3, 1.0)
    twice = S.f32_to_bf16_bits(2 * S.bf16_bits_to_f32(yref))
    num, den, rel = lib.svdq_score_lambda(dev_bits(yref), dev_bits(yref), [(0, 64)])
    assert num.item() == 0.0 and rel.item() == 0.0
    num, den, rel = lib.svdq_score_lambda(dev_bits(twice), dev_bits(yref), [(0, 32), (32, 64)])
    assert torch.equal(num, den) and torch.all(rel == 1.0)


# ---------------------------------------------------------------------------
# Config 1 (DiT attention projection) at full size
# ---------------------------------------------------------------------------

@pytest.fixture(scope="module")
def cfg1():
    L = S.make_layer(1)
    segs = L.seg_ranges(L.calib_sets["all"])
    c = O.calib(L.x, segs, L.w)
    sketch = S.power_iteration_sketch(L.n, L.rank)
    conv = O.convert_weight(L.w, c["lam"], L.rank, sketch=sketch)
    return L, segs, c, conv


def test_config1_calib_quantize_full(lib, cfg1):
    L, segs, c, conv = cfg1
    g = lib.svdq_calib_lambda(dev_bits(L.x), segs, dev_bits(L.w))
    assert np.array_equal(g["lam"].cpu().numpy(), c["lam"])
    assert g["s_g"].item() == float(c["s_g"])
    codes, sf, n_sat = O.quantize_blocks(L.x, c["inv_lam"], c["s_g"])
    sat = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = lib.svdq_quantize_act(dev_bits(L.x), g["inv_lam"], g["s_g"], dev_bits(conv["down"]), sat_count=sat)
    check_codes(q["codes"], codes)
    check_sf(q["sf"], sf, L.m, L.k)
    assert int(sat.item()) == n_sat
    rows = np.arange(0, L.m, 61)
    d64 = O.lowrank_down(L.x[rows], conv["down"])
    check_d(q["d"].cpu().numpy()[rows], d64, L.x[rows], conv["down"])


def test_config1_residual_and_linear_sampled(lib, cfg1):
    L, segs, c, conv = cfg1
    r = lib.svdq_residual(dev_bits(L.w), dev_f32(c["lam"]), dev_bits(conv["down"]), dev_bits(conv["up"]))
    assert np.array_equal(host_bits(r), conv["residual"])
    s_ga = dev_f32(np.array([c["s_g"]]))
    wc = lib.svdq_calib_lambda(r, None, None)
    assert wc["s_g"].item() == float(conv["s_g"])
    wq = lib.svdq_quantize_act(r, None, wc["s_g"])
    check_codes(wq["codes"], conv["codes"])
    q = lib.svdq_quantize_act(dev_bits(L.x), dev_f32(c["inv_lam"]), s_ga, dev_bits(conv["down"]))
    args = (q["codes"], q["sf"], s_ga, q["d"], wq["codes"], wq["sf"], wc["s_g"], dev_bits(conv["up"]),
            dev_bits(L.bias))
    yb = host_bits(lib.svdq_linear(*args))
    yf = lib.svdq_linear(*args, out_dtype=torch.float32).cpu().numpy()
    rows = np.unique(np.concatenate([np.arange(0, L.m, 97), [0, 28, 29, 4067, 4068, L.m - 1]]))
    codes, sf, _ = O.quantize_blocks(L.x[rows], c["inv_lam"], c["s_g"])
    d64 = O.lowrank_down(L.x[rows], conv["down"])
    y64 = O.linear(codes, sf, c["s_g"], conv["codes"], conv["sf"], conv["s_g"], d64, conv["up"], L.bias)
    check_linear_f32(yf[rows], y64, tight_rel=1e-4)
    check_linear_bf16(yb[rows], y64)


def test_no_device_wait_timed_out(lib):
    assert lib.svdq_device_error() == 0


# ---------------------------------------------------------------------------
# The product's own offline conversion (device factorisation + library kernels)
# ---------------------------------------------------------------------------

def test_product_conversion_quality(lib, cfg0):
    """The layer built by SVDQW4A4Linear.convert is as good as the oracle's pipeline.

    Its low-rank factors come from a randomized range finder on the device, so
    they are not bit-identical to the oracle's exact SVD; what must hold is
    that the rank-r residual is near-optimal and the layer's error against the
    unquantised fp64 output is no worse than the oracle pipeline's.
    """
    L, segs, c, conv = cfg0
    x, w, b = dev_bits(L.x), dev_bits(L.w), dev_bits(L.bias)
    cal = lib.SVDQW4A4Linear.calibrate(x, w, segs)
    assert np.array_equal(cal["lam"].cpu().numpy(), c["lam"])
    layer = lib.SVDQW4A4Linear.convert(w, b, cal, L.rank)
    y = layer(x, out_dtype=torch.float32).cpu().numpy().astype(np.float64)
    y_ref = O.reference_linear(L.x, L.w, L.bias)
    y_orc, _ = O.layer_forward(L.x, c["inv_lam"], c["s_g"], conv["down"], conv, L.bias)
    rel_gpu, rel_orc = rel_l2(y, y_ref), rel_l2(y_orc, y_ref)
    assert rel_gpu <= 1.10 * rel_orc, (rel_gpu, rel_orc)
    # near-optimal rank-r split: ||W lambda - (lambda down^T up^T)^T||_F vs the SVD tail
    lam = c["lam"].astype(np.float64)
    w_hat = O.bf16_to_f64(L.w) * lam[None, :]
    down = O.bf16_to_f64(host_bits(layer.down))
    up = O.bf16_to_f64(host_bits(layer.up))
    resid = np.linalg.norm(w_hat - up @ (down * lam[None, :]))
    sv = np.linalg.svd(w_hat, compute_uv=False)
    tail = np.sqrt(np.sum(sv[L.rank:] ** 2))
    assert resid <= 1.02 * tail, (resid, tail)
    assert lib.svdq_device_error() == 0
