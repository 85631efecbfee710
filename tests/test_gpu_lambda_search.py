"""The lambda candidate grid (svdq_lambda_grid) and the search over it (search_lambda).

"MiniMax-H3 NVFP4 -- what the smoothing scale should be calibrated on",
sections "Calibration" (lambda picked from a grid of candidates built from
absmax statistics) and "The metric that picks the winner also hides the cost"
(candidates ranked by rel-L2 against bf16 on each modality's rows).

lambda(alpha) goes through fp64 log2 / exp2 on both sides; the two libraries
can part in the last fp64 bit, which moves the fp32 rounding only when the
value sits on a rounding boundary: lambda is compared exactly for almost every
element and within one fp32 ulp for all.  The search at rank 0 (no randomized
factorisation) runs the same chain as the oracle's: calibration, grid,
residual, NVFP4 weight and activation codes are exact, the GEMM within its
tolerance, so every candidate's per-modality rel-L2 matches to 1e-3 relative.
"""
import numpy as np
import pytest
import torch

import synthetic as S
from oracle import svdq_oracle as O
from gpu_util import dev_bits, host_bits, requires_cuda

pytestmark = [pytest.mark.gpu, requires_cuda]


@pytest.fixture(scope="module")
def lib():
    import bit_w4a4_quantized_svdq_b200 as P
    return P


def _stats(k, seed):
    rng = np.random.default_rng(seed)
    ax = rng.lognormal(0.0, 2.5, k).astype(np.float32)
    aw = rng.lognormal(-4.0, 1.0, k).astype(np.float32)
    ax[rng.random(k) < 0.01] = 0.0
    aw[rng.random(k) < 0.01] = 0.0
    return ax, aw


@pytest.mark.parametrize("k", [1, 300, 5120, 20480])
def test_grid_matches_oracle(lib, k):
    ax, aw = _stats(k, k)
    alphas = O.alpha_grid()
    g = lib.svdq_lambda_grid(torch.from_numpy(ax).cuda(), torch.from_numpy(aw).cuda(), torch.from_numpy(alphas).cuda())
    lam = g["lam"].cpu().numpy()
    inv = g["inv_lam"].cpu().numpy()
    s_g = g["s_g"].cpu().numpy()
    lam_o, inv_o, s_g_o = O.lambda_grid(ax, aw, alphas)
    same = lam == lam_o
    assert same.mean() >= 0.9999
    assert np.all(np.abs(lam.astype(np.float64) - lam_o) <= np.spacing(lam_o))
    # 1/lambda is the rounded reciprocal of the lambda written
    assert np.array_equal(inv, (np.float32(1) / lam).astype(np.float32))
    rows = same.all(axis=1)
    assert np.array_equal(s_g[rows], s_g_o[rows])
    assert np.all(np.abs(s_g.astype(np.float64) - s_g_o) <= 2 * np.spacing(s_g_o))


def test_half_is_the_calibration_rule(lib):
    # alpha = 0.5 against svdq_calib_lambda's square root of the same statistics:
    # the calibration rounds ax / aw to fp32 before its square root, the grid
    # does not, so the two part by one ulp where that rounding matters
    L = S.make_layer(1)
    x, w = dev_bits(L.x), dev_bits(L.w)
    cal = lib.svdq_calib_lambda(x, L.seg_ranges(L.calib_sets["all"]), w)
    g = lib.svdq_lambda_grid(cal["amax_x"], cal["amax_w"], torch.tensor([0.5], device="cuda"))
    a, b = g["lam"][0].cpu().numpy(), cal["lam"].cpu().numpy()
    assert np.all(np.abs(a.astype(np.float64) - b) <= np.spacing(b))
    assert (a == b).mean() > 0.75


def test_search_matches_oracle_rank0(lib):
    L = S.make_layer(4, m=768, k=512, n=512)
    segs = [(sg.begin, sg.end) for sg in L.segments]
    calib_segs = L.seg_ranges(L.calib_sets["all"])
    alphas = O.alpha_grid()
    yref_bits = O.f64_to_bf16(O.reference_linear(L.x, L.w, L.bias))
    res = lib.search_lambda(dev_bits(L.x), dev_bits(L.w), dev_bits(L.bias), 0, calib_segs, segs,
                            alphas=torch.from_numpy(alphas), yref=dev_bits(yref_bits))
    rel = res["rel"].cpu().numpy()

    c = O.calib(L.x, calib_segs, L.w)
    lam, inv, s_g = O.lambda_grid(c["ax"], c["aw"], alphas)
    rel_o = np.zeros_like(rel)
    for i in range(len(alphas)):
        conv = O.convert_weight(L.w, lam[i], 0)
        y64, _ = O.layer_forward(L.x, inv[i], s_g[i], None, conv, L.bias)
        rel_o[i] = O.score(O.f64_to_bf16(y64), yref_bits, segs)[2]
    np.testing.assert_allclose(rel, rel_o, rtol=1e-3)
    total = rel_o @ np.ones(len(segs))
    order = np.argsort(total)
    if (total[order[1]] - total[order[0]]) / total[order[0]] > 1e-2:
        assert res["best"] == O.select_candidate(rel_o, np.ones(len(segs)))
    # the weighted pick follows the weights: one modality alone
    for m in range(len(segs)):
        wts = np.eye(len(segs))[m]
        assert O.select_candidate(rel, wts) == int(np.argmin(rel[:, m]))
    ax_mod = np.stack([O.calib(L.x, [s], None)["ax"] for s in segs])
    np.testing.assert_allclose(res["bits"].cpu().numpy(), O.bits_lost(ax_mod, inv), rtol=1e-6, atol=1e-9)
    assert lib.svdq_device_error() == 0


def test_search_rank32_consistent(lib):
    # with the rank-32 branch: the returned layer is the winner, and its output
    # scores what the search recorded for it
    L = S.make_layer(4, m=1536, k=1024, n=1024)
    segs = [(sg.begin, sg.end) for sg in L.segments]
    x, w, bias = dev_bits(L.x), dev_bits(L.w), dev_bits(L.bias)
    alphas = torch.tensor([0.2, 0.35, 0.5, 0.65, 0.8])
    res = lib.search_lambda(x, w, bias, 32, L.seg_ranges(L.calib_sets["all"]), segs, alphas=alphas,
                            weights=[1.0, 2.0, 1.0])
    rel = res["rel"].cpu().numpy()
    assert rel.shape == (5, 3) and np.all(np.isfinite(rel)) and np.all(rel > 0)
    assert res["best"] == int(np.argmin(rel @ np.array([1.0, 2.0, 1.0])))
    yref = x.view(torch.bfloat16) @ w.view(torch.bfloat16).t() + bias.view(torch.bfloat16)
    y = res["layer"](x)
    _, _, rel_best = lib.svdq_score_lambda(y, yref, segs)
    np.testing.assert_allclose(rel_best.cpu().numpy(), rel[res["best"]], rtol=1e-9)
    assert lib.svdq_device_error() == 0
