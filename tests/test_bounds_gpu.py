"""The bounds-checked debug build (libentmax_attn_bounds.so, compiled with
-DENTMAX_BOUNDS_CHECK): every shared-memory, tensor-memory and global index
the kernels compute is checked before the access, and a violation sets
ENTMAX_ST_BOUNDS in the status word and skips the access -- the stand-in for a
memory checker, which this environment does not offer.

The small parity suites (ragged N, N = 1, block 64 and 128, causal and not,
head dim 64 and 128, alpha 1.5, 2 and the power path, the fp32 path, the
router) run against that build in a child process.  Each of their cases asserts
that the device status word is 0, so a single out-of-range index fails them;
their outputs must also still match the oracle.
"""

import os
import subprocess
import sys

import pytest

from differentiable_sparse_attention_b200 import build as build_mod

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import os, sys
import pytest
import differentiable_sparse_attention_b200 as dsa
assert dsa.LIB_PATH.endswith("libentmax_attn_bounds.so"), dsa.LIB_PATH
rc = pytest.main(["-q", "-p", "no:cacheprovider", "-m", "gpu", "-x"] + sys.argv[1:])
maps = open("/proc/self/maps").read()
assert "libentmax_attn_bounds.so" in maps and "libentmax_attn.so" not in maps
sys.exit(int(rc))
"""


def test_small_parity_suites_under_the_bounds_checked_build():
    lib = build_mod.build(bounds_check=True)
    env = dict(os.environ, ENTMAX_ATTN_LIB=lib)
    env.pop("PARITY_REPORT", None)
    suites = [os.path.join(ROOT, "tests", f) for f in
              ("test_fwd_gpu.py", "test_bwd_gpu.py", "test_alpha_generic_gpu.py",
               "test_fp32_gpu.py", "test_dash_gpu.py", "test_failure_gpu.py",
               "test_zz_no_alloc.py")]
    run = subprocess.run([sys.executable, "-c", CHILD] + suites, cwd=ROOT,
                         env=env, capture_output=True, text=True, timeout=1200)
    assert run.returncode == 0, (run.stdout[-3000:] + run.stderr[-3000:])
