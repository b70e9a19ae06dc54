"""The checked build (libfathom_checked.so): small parity cases on both scan
kernels, the fallback and the batched launch, with every plane-row, sample
and candidate index bounds-checked on the device.  They must match the
oracle and record no device fault.  Runs in a child process, since the
library to load is chosen when the binding first loads it."""

import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_checked_build_small_cases():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bit_plane_kv_scan_b200 import build
    build.build()
    env = dict(os.environ, FATHOM_LIB="checked")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "checked_cases.py")], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "ok batched" in r.stdout
