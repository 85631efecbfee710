"""A bounded device wait that runs out: the kernel returns, the host reads an
error status, and the context stays usable.

Every wait in the library's kernels gives up after a cycle limit, records a
code in the per-device error word, tells the CTA's other roles to stop and
drains the CTA's own copies before returning.  Here the host arms one call of
the scoring stream kernel (no tensor memory, no MMA) so that its first CTA
leaves one chunk uncopied and waits only ~1 ms: the consumer wait for that
chunk runs out, and the CTA still meets the others at the kernel's grid
barrier.  Nothing is faulted or trapped; the next calls must be exact again.
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


def _exact(lib, yq, yr, yqd, yrd, segs):
    num, den, rel = lib.svdq_score_lambda(yqd, yrd, segs)
    n64, d64, r64 = O.score(yq, yr, segs)
    assert np.allclose(num.cpu().numpy(), n64, rtol=1e-6, atol=0)
    assert np.allclose(den.cpu().numpy(), d64, rtol=1e-6, atol=0)
    assert np.allclose(rel.cpu().numpy(), r64, rtol=1e-6, atol=0)
    again = lib.svdq_score_lambda(yqd, yrd, segs)
    assert np.array_equal(again[2].cpu().numpy(), rel.cpu().numpy())


@pytest.mark.parametrize("chunk", [1, 3])
def test_score_wait_runs_out_reports_and_recovers(lib, chunk):
    # 4096 x 2048 in 16384-element chunks: 512 chunks over 148 CTAs, so the
    # first CTA owns 4 chunks in a 3-slot ring.  Its loader only waits again on
    # the slot of its first chunk (for its fourth), so with chunk 1, 2 or 3
    # missing the loader never waits on the missing chunk's slot and the
    # consumers' wait is the one that runs out (with chunk 0 missing, the two
    # waits would race).
    m, n = 4096, 2048
    yq = S.random_bf16((m, n), 77, 1.0)
    yr = S.random_bf16((m, n), 78, 1.0)
    yqd, yrd = dev_bits(yq), dev_bits(yr)
    segs = [(0, 1000), (1000, m)]
    assert lib.svdq_device_error() == 0
    raw = lib.load()
    assert raw.svdq_debug_arm_score_timeout(chunk, 2_000_000) == 0      # about 1 ms of SM cycles
    t0 = time.perf_counter()
    lib.svdq_score_lambda(yqd, yrd, segs)
    code = lib.svdq_device_error()                                     # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert code == WAIT_FULL
    assert elapsed < 1.0, f"the armed wait should give up after ~1 ms, took {elapsed:.3f} s"
    # the context is usable: the same call, unarmed, matches the oracle, twice
    _exact(lib, yq, yr, yqd, yrd, segs)
    assert lib.svdq_device_error() == 0


def test_arming_rejects_bad_values(lib):
    raw = lib.load()
    assert raw.svdq_debug_arm_score_timeout(-1, 2_000_000) == 1
    assert raw.svdq_debug_arm_score_timeout(0, 10) == 1
