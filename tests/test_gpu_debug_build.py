"""The bounds-checking debug build (libradial_debug.so, -DRADIAL_DEBUG) on a
device: small forward and backward parity cases run through it in a child
process.  Every kernel there checks each tile number and work-item index it
reads from the mask's arrays; an out-of-range value would make the parity
tests' radial_device_status() calls raise RADIAL_EDEVICE."""

import os
import subprocess
import sys

import pytest

from block_sparse_attention_csr_b200 import build as build_mod

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parity_through_the_debug_build():
    build_mod.build()
    env = dict(os.environ, RADIAL_LIBRARY=build_mod.OUT_DEBUG)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-m", "gpu",
                        os.path.join(ROOT, "tests", "test_gpu_fwd.py"), os.path.join(ROOT, "tests", "test_gpu_bwd.py"),
                        "-k", "test_small_all_rows or test_small_all_gradients or test_tiny_config"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    # the child really loaded the debug build
    check = subprocess.run([sys.executable, "-c", "import block_sparse_attention_csr_b200._binding as B; print(B.lib_path)"],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=120)
    assert check.stdout.strip() == build_mod.OUT_DEBUG
