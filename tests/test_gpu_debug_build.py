"""The GPU parity tests again, against the debug library, plus its own checks.

A child pytest runs with SVDQ_DEBUG=1, so it loads ``libsvdq_debug.so`` (the
same source with every output store bounds-checked in the kernels and every
pointer argument checked on the host) and the binding, after every call,
synchronises, reads the device error word and checks the guard bands around the
outputs it allocated (whose bodies start as 0xFF bytes, so an element a call
should write but does not fails the parity comparison).  Any store a kernel
makes outside its output, on any parity shape, fails the child run.
"""
import os
import re
import subprocess
import sys

import pytest

from gpu_util import requires_cuda

pytestmark = [pytest.mark.gpu, requires_cuda]

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FILES = ["tests/test_gpu_parity.py", "tests/test_gpu_linear_score.py", "tests/test_gpu_mxfp8.py",
         "tests/test_gpu_bits_lost.py", "tests/test_gpu_lambda_search.py", "tests/gpu_debug_checks.py"]


def test_parity_suite_and_checks_under_the_debug_library():
    env = dict(os.environ, SVDQ_DEBUG="1")
    res = subprocess.run([sys.executable, "-m", "pytest", *FILES, "-m", "gpu", "-x", "-q", "-p", "no:cacheprovider",
                          "-rs"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    tail = res.stdout[-6000:] + res.stderr[-3000:]
    assert res.returncode == 0, tail
    passed = re.search(r"(\d+) passed", res.stdout)
    assert passed and int(passed.group(1)) >= 60, tail
    assert "skipped" not in res.stdout.splitlines()[-1], tail
