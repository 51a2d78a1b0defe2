"""Build libentmax_attn.so (sm_100a) in the package directory with nvcc.

    python -m differentiable_sparse_attention_b200.build [--ptxas-verbose] [--bounds-check]

--bounds-check builds the debug variant libentmax_attn_bounds.so instead: every
shared-memory, tensor-memory and global index the kernels compute is checked
before the access, and a violation sets ENTMAX_ST_BOUNDS in the status word
and skips the access (the kernels never trap).  Load it by setting
ENTMAX_ATTN_LIB to its path before importing the package.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "entmax_attn.cu")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libentmax_attn.so")
LIB_BOUNDS = os.path.join(HERE, "libentmax_attn_bounds.so")


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build(ptxas_verbose: bool = False, force: bool = False, bounds_check: bool = False) -> str:
    lib = LIB_BOUNDS if bounds_check else LIB
    deps = [SRC, os.path.join(INCLUDE, "entmax_attn.h"), os.path.abspath(__file__)]
    deps += [os.path.join(HERE, "csrc", f) for f in os.listdir(os.path.join(HERE, "csrc"))]
    if (not force and not ptxas_verbose and os.path.exists(lib)
            and os.path.getmtime(lib) >= max(os.path.getmtime(d) for d in deps)):
        return lib
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
           "-I", INCLUDE, "-o", lib + ".tmp", SRC]
    if bounds_check:
        cmd.insert(1, "-DENTMAX_BOUNDS_CHECK")
    if ptxas_verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed:\n{res.stdout}\n{res.stderr}")
    if ptxas_verbose:
        sys.stderr.write(res.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(ptxas_verbose="--ptxas-verbose" in sys.argv, force=True,
                bounds_check="--bounds-check" in sys.argv))
