"""The address-checking build (libsparse_attn_bounds.so, -DSA_DEBUG_BOUNDS):
every gather checks that the first row it reads lies inside the slab of its
tensor that the operation means to read (a kv-head's N keys, a query head's
padded rows, a unit's landmarks) and sets status bit 8 when not.  The parity
tests below run against that build in a child process (SPARSE_ATTN_LIB); each
of them asserts that the status word is clear after its calls, so a gather
outside its slab fails them, and they still compare every output with the
oracle."""
from __future__ import annotations

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BOUNDS_LIB = os.path.join(ROOT, "block_sparse_long_landmark_b200", "lib", "libsparse_attn_bounds.so")
FILES = ["test_gpu_parity.py", "test_gpu_select_decode.py", "test_gpu_backward.py", "test_gpu_lsa.py",
         "test_gpu_lsa_tree.py", "test_gpu_varlen.py"]


def test_parity_on_the_address_checking_build():
    if not os.path.exists(BOUNDS_LIB):
        from block_sparse_long_landmark_b200 import build
        build.build(bounds=True)
    env = dict(os.environ, SPARSE_ATTN_LIB=BOUNDS_LIB)
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-m", "gpu"] + \
        [os.path.join(ROOT, "tests", f) for f in FILES]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
