"""Pins of the oracle's lambda candidate grid and candidate selection.

"MiniMax-H3 NVFP4 -- what the smoothing scale should be calibrated on",
sections "Calibration" (a grid of lambda candidates from absmax statistics)
and "The metric that picks the winner also hides the cost" (candidates ranked
by rel-L2 against bf16, on proportional rows or per modality).
"""
import math

import numpy as np

from oracle import svdq_oracle as O


def _stats(k, seed):
    rng = np.random.default_rng(seed)
    ax = rng.lognormal(0.0, 2.0, k).astype(np.float32)
    aw = rng.lognormal(-3.0, 1.0, k).astype(np.float32)
    ax[3] = 0.0
    aw[7] = 0.0
    return ax, aw


def test_grid_values():
    g = O.alpha_grid()
    assert g.dtype == np.float32 and len(g) == 39
    assert g[0] == np.float32(0.05) and g[-1] == np.float32(0.95) and g[19] == np.float32(0.5)
    assert np.all(np.diff(g.astype(np.float64)) > 0)


def test_endpoints_are_closed_forms():
    ax, aw = _stats(256, 0)
    lam, inv, _ = O.lambda_grid(ax, aw, np.float32([0.0, 1.0]))
    ok = (ax > 0) & (aw > 0)
    # alpha = 1: lambda is the activation absmax; alpha = 0: it is 1 / weight absmax
    assert np.array_equal(lam[1][ok], ax[ok])
    assert np.array_equal(lam[0][ok], (np.float64(1.0) / aw[ok].astype(np.float64)).astype(np.float32))
    assert np.all(lam[:, ~ok] == 1.0)
    assert np.array_equal(inv, (np.float32(1) / lam).astype(np.float32))


def test_half_is_the_square_root_rule():
    # alpha = 0.5 is R8's sqrt(ax / aw): equal up to the one rounding where the two
    # evaluations part (within one fp32 ulp), and mostly bit-equal
    ax, aw = _stats(4096, 1)
    lam, _, _ = O.lambda_grid(ax, aw, np.float32([0.5]))
    ok = (ax > 0) & (aw > 0)
    exact = np.sqrt(ax[ok].astype(np.float64) / aw[ok].astype(np.float64))
    ulp = np.spacing(lam[0][ok])
    assert np.all(np.abs(lam[0][ok].astype(np.float64) - exact) <= ulp)


def test_powers_of_two_are_exact():
    ax = np.float32(2.0) ** np.arange(-8, 8, dtype=np.float32)
    aw = np.float32(2.0) ** np.arange(4, -12, -1, dtype=np.float32)
    lam, _, s_g = O.lambda_grid(ax, aw, np.float32([0.25, 0.75]))
    e_x = np.arange(-8, 8)
    e_w = np.arange(4, -12, -1)
    for i, a in enumerate((0.25, 0.75)):
        expect = np.array([2.0 ** (a * x - (1 - a) * w) for x, w in zip(e_x, e_w)])
        exact = (a * e_x - (1 - a) * e_w) == np.round(a * e_x - (1 - a) * e_w)
        assert np.array_equal(lam[i][exact].astype(np.float64), expect[exact])
        smoothed = ax.astype(np.float64) / lam[i].astype(np.float64)
        assert math.isclose(float(s_g[i]), smoothed.max() / 2688.0, rel_tol=2 ** -22)


def test_monotone_in_alpha():
    ax, aw = _stats(512, 2)
    lam, _, _ = O.lambda_grid(ax, aw, O.alpha_grid())
    ok = (ax > 0) & (aw > 0)
    prod = ax[ok].astype(np.float64) * aw[ok].astype(np.float64)
    d = np.diff(lam[:, ok].astype(np.float64), axis=0)
    # d lambda / d alpha = lambda * ln(ax * aw): the sign of log(ax * aw) for every step
    assert np.all(d[:, prod > 1.001] >= 0) and np.all(d[:, prod < 0.999] <= 0)


def test_selection():
    rel = np.array([[0.10, 0.20, 0.30], [0.12, 0.15, 0.25], [0.09, 0.30, 0.40]])
    assert O.select_candidate(rel, np.array([1.0, 0.0, 0.0])) == 2
    assert O.select_candidate(rel, np.array([1.0, 1.0, 1.0])) == 1
    assert O.select_candidate(np.array([[1.0], [1.0]]), np.array([1.0])) == 0     # ties: the lower index
