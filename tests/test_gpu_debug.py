"""The debug build of the library (needs a B200): copy bounds checks and bounded
waits that run out.

The debug library (libkivi_debug.so: KIVI_DEBUG_BUILD, KIVI_DEBUG_BOUNDS, waits of
about 1 ms) runs in a child process selected with KIVI_LIBRARY, so this process
keeps the regular library.  No GPU is faulted: a wait is made to run out by
telling the decode kernel to expect more bytes than its copies bring, while
every issued copy still lands whole, and the kernel reports the failure in its
status word.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.fixture(scope="module")
def debug_lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from decode_attention_kivi_b200 import build

    return build.build(debug=True)


def _child(lib, what):
    env = dict(os.environ, KIVI_LIBRARY=lib, PYTHONPATH=os.pathsep.join([ROOT, HERE]))
    r = subprocess.run([sys.executable, os.path.join(HERE, "gpu_debug_child.py"), what],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    return r.stdout


def test_parity_under_bounds_checks(debug_lib):
    assert "bounds: ok" in _child(debug_lib, "bounds")


def test_wait_that_runs_out_reports_a_device_error(debug_lib):
    assert "wait: ok" in _child(debug_lib, "wait")
