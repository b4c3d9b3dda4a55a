"""The small parity shapes under the bounds-check build of the library.

libkvq_debug.so is built from the same sources with -DKVQ_DEBUG: its kernels compare every
data-dependent global index (rows and groups found through the length rules or the block
table, window and retained slots, partial rows) with the extent of the buffer it addresses,
and count failures in a record instead of touching memory out of bounds.  This test runs the
parity tests of every small shape (all but the full-size workloads) in a child process that
loads that library; the conftest fixture asserts after each of them that no check failed, and
the parity assertions themselves still hold.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_small_parity_shapes_pass_every_bounds_check():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = os.path.join(ROOT, "mixed_precision_quantized_pack_b200", "libkvq_debug.so")
    assert os.path.exists(lib), "build the bounds-check library: python -m mixed_precision_quantized_pack_b200.build --debug"
    env = dict(os.environ, KVQ_LIBRARY="debug")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_gpu_parity.py"),
                        "-m", "gpu", "-x", "-q", "-p", "no:cacheprovider", "-k", "not full_size"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-30:])
    assert r.returncode == 0, tail
    assert " passed" in r.stdout, tail
