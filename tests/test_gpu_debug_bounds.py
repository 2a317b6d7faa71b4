"""The debug-bounds build (libmk_debug.so, compiled with MK_DEBUG_BOUNDS):
every task checks the indices of its global and shared-memory accesses
against their buffers and reports a violation as MK_ERR_BOUNDS instead of
performing the access.  The decode cases of tests/bounds_cases.py -- every
execution mode, split boundaries, the batched step, shuffled KV pages, fp8
weights, Llama widths -- must run through it without a violation and still
meet the oracle.  (A violation is never provoked on purpose: the checks are
exercised by valid work only.)"""
import os
import subprocess
import sys

import pytest

from persistent_megakernel_03_b200 import build

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_decode_cases_pass_in_the_debug_bounds_build(cuda_ok):
    lib = build.build(debug_bounds=True)
    env = dict(os.environ, MK_LIBRARY=lib)
    r = subprocess.run([sys.executable, os.path.join(HERE, "bounds_cases.py")], env=env,
                       capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "bounds cases ok" in r.stdout
