"""A bounded device wait that runs out: the kernel returns, the host reads an
error status, and the context stays usable.

Every wait in the library's kernels gives up after a cycle limit, records a
code in the per-device error word, tells the CTA's other roles to stop and
drains the CTA's own copies before returning.  Here the host arms one call of
the calibration stream kernel (no tensor memory, no MMA) so that its first
CTA leaves one ring unit unloaded and waits only ~1 ms: the consumer wait for
that unit runs out.  Nothing is faulted or trapped; the next calls must be
exact again.
"""
import time

import numpy as np
import pytest

import synthetic as S
from gpu_util import dev_bits, requires_cuda
from oracle import svdq_oracle as O

pytestmark = [pytest.mark.gpu, requires_cuda]

WAIT_FULL = 1          # error code: a consumer waited too long for a TMA stage


@pytest.fixture(scope="module")
def lib():
    import bit_w4a4_quantized_svdq_b200 as P
    return P


def _exact(lib, xd, x, w=None, wd=None):
    g = lib.svdq_calib_lambda(xd, None, wd)
    c = O.calib(x, None, w)
    assert np.array_equal(g["amax_x"].cpu().numpy(), c["ax"])
    assert np.array_equal(g["lam"].cpu().numpy(), c["lam"])
    assert np.array_equal(g["inv_lam"].cpu().numpy(), c["inv_lam"])
    assert float(g["s_g"].item()) == float(c["s_g"])


@pytest.mark.parametrize("unit", [0, 2])
def test_calib_wait_runs_out_reports_and_recovers(lib, unit):
    # 4096 x 2048 without a weight: 8 strips x 128 row boxes = 1024 units over at
    # most 148 CTAs, so the first CTA owns about 7 units -- fewer than its 8 ring
    # slots, so its loader never blocks and the consumer wait is the one that runs out.
    m, k = 4096, 2048
    x = S.random_bf16((m, k), 77, 1.0)
    xd = dev_bits(x)
    assert lib.svdq_device_error() == 0
    raw = lib.load()
    assert raw.svdq_debug_arm_calib_timeout(unit, 2_000_000) == 0       # about 1 ms of SM cycles
    t0 = time.perf_counter()
    lib.svdq_calib_lambda(xd, None, None)
    code = lib.svdq_device_error()                                     # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert code == WAIT_FULL
    assert elapsed < 1.0, f"the armed wait should give up after ~1 ms, took {elapsed:.3f} s"
    # the context is usable: the same call, unarmed, is bit-exact, twice, with and without a weight
    _exact(lib, xd, x)
    w = S.random_bf16((512, k), 78, 0.02)
    _exact(lib, xd, x, w, dev_bits(w))
    assert lib.svdq_device_error() == 0


def test_arming_rejects_bad_values(lib):
    raw = lib.load()
    assert raw.svdq_debug_arm_calib_timeout(-1, 2_000_000) == 1
    assert raw.svdq_debug_arm_calib_timeout(0, 10) == 1
