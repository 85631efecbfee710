"""svdq_bits_lost on the GPU against the oracle's bits-lost proxy.

"MiniMax-H3 NVFP4 -- what the smoothing scale should be calibrated on",
section "Why": log2(group_absmax / channel_absmax) of the statistics the kernel
sees (X / lambda), averaged per modality.  The fp32 smoothed statistics and the
group maxima are exact on both sides; the logarithms (fp64, within an ulp) and
the order of the fp64 sum differ, hence a relative 1e-12.
"""
import numpy as np
import pytest
import torch

import synthetic as S
from oracle import svdq_oracle as O
from gpu_util import dev_bits, requires_cuda

pytestmark = [pytest.mark.gpu, requires_cuda]


@pytest.fixture(scope="module")
def lib():
    import bit_w4a4_quantized_svdq_b200 as P
    return P


def _stats(n_mod, k, seed):
    rng = np.random.default_rng(seed)
    ax = rng.lognormal(0.0, 2.0, size=(n_mod, k)).astype(np.float32)
    ax[rng.random((n_mod, k)) < 0.05] = 0.0               # dead channels
    ax[:, :16] = 0.0                                       # one all-zero group
    return ax


@pytest.mark.parametrize("n_mod,n_cand,k", [(1, 1, 16), (3, 1, 5120), (3, 39, 5120), (2, 7, 20480), (64, 3, 1024)])
def test_matches_oracle(lib, n_mod, n_cand, k):
    ax = _stats(n_mod, k, k + n_mod)
    il = np.random.default_rng(n_cand).uniform(0.05, 20.0, size=(n_cand, k)).astype(np.float32)
    got = lib.svdq_bits_lost(torch.from_numpy(ax).cuda(), torch.from_numpy(il).cuda()).cpu().numpy()
    np.testing.assert_allclose(got, O.bits_lost(ax, il), rtol=1e-12, atol=1e-15)
    if n_cand == 1:
        got1 = lib.svdq_bits_lost(torch.from_numpy(ax).cuda()).cpu().numpy()
        np.testing.assert_allclose(got1, O.bits_lost(ax, None), rtol=1e-12, atol=1e-15)


def test_all_zero_and_strided(lib):
    ax = np.zeros((2, 64), np.float32)
    ax[1, 3] = 2.0
    got = lib.svdq_bits_lost(torch.from_numpy(ax).cuda()).cpu().numpy()
    assert got[0, 0] == 0.0 and got[0, 1] == 0.0
    # rows of a wider buffer (row stride > K)
    wide = torch.from_numpy(_stats(3, 96, 5)).cuda()[:, :64]
    il = torch.from_numpy(np.random.default_rng(6).uniform(0.5, 2, size=(4, 80)).astype(np.float32)).cuda()[:, :64]
    got = lib.svdq_bits_lost(wide, il).cpu().numpy()
    np.testing.assert_allclose(got, O.bits_lost(wide.cpu().numpy(), il.cpu().numpy()), rtol=1e-12, atol=1e-15)


def test_calibration_pass_end_to_end(lib):
    # per-modality statistics from the calibration kernel, lambda from each modality
    # and from all rows: the same chain as the oracle's (calib is bit-exact)
    L = S.make_layer(1)
    x = dev_bits(L.x)
    w = dev_bits(L.w)
    mods = [(sg.begin, sg.end) for sg in L.segments]
    ax_gpu = torch.stack([lib.svdq_calib_lambda(x, [m], None)["amax_x"] for m in mods])
    cands = [lib.svdq_calib_lambda(x, segs, w)["inv_lam"] for segs in (L.seg_ranges(L.calib_sets["all"]), *([m] for m in mods))]
    got = lib.svdq_bits_lost(ax_gpu, torch.stack(cands)).cpu().numpy()
    ax_o = np.stack([O.calib(L.x, [m], None)["ax"] for m in mods])
    il_o = np.stack([O.calib(L.x, segs, L.w)["inv_lam"] for segs in (L.seg_ranges(L.calib_sets["all"]), *([m] for m in mods))])
    np.testing.assert_allclose(got, O.bits_lost(ax_o, il_o), rtol=1e-12, atol=1e-15)
    assert lib.svdq_device_error() == 0
