"""Build step: compile libradial.so (sm_100a) in-tree with nvcc.

Usage: ``python -m block_sparse_attention_csr_b200.build [--force]``.
"""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "libradial.so")
# Same sources with -DRADIAL_DEBUG: every index the kernels read from the
# mask's arrays is range-checked on the device (see sm100_primitives.cuh).
OUT_DEBUG = os.path.join(HERE, "libradial_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
    "-I", os.path.join(ROOT, "include"),
]


def _sources():
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))
            if f.endswith((".cu", ".cuh", ".h"))] + [os.path.join(ROOT, "include", "radial.h")]


def up_to_date(out=OUT):
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(s) <= t for s in _sources())


def _compile(out, extra, verbose):
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, *NVCC_FLAGS, *extra, "-o", out + ".tmp", os.path.join(CSRC, "radial_lib.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(out + ".tmp", out)


def build(force=False, verbose=False, debug=True):
    """Build libradial.so (and, unless debug=False, libradial_debug.so)."""
    if force or not up_to_date(OUT):
        _compile(OUT, [], verbose)
    if debug and (force or not up_to_date(OUT_DEBUG)):
        _compile(OUT_DEBUG, ["-DRADIAL_DEBUG"], verbose)
    return OUT


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(OUT)
