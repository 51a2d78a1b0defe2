"""Build libentmax_attn.so (sm_100a) in the package directory with nvcc.

    python -m differentiable_sparse_attention_b200.build [--ptxas-verbose]
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


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build(ptxas_verbose: bool = False, force: bool = False) -> str:
    deps = [SRC, os.path.join(INCLUDE, "entmax_attn.h")]
    deps += [os.path.join(HERE, "csrc", f) for f in os.listdir(os.path.join(HERE, "csrc"))]
    if (not force and not ptxas_verbose and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(d) for d in deps)):
        return LIB
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
           "-I", INCLUDE, "-o", LIB + ".tmp", SRC]
    if ptxas_verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed:\n{res.stdout}\n{res.stderr}")
    if ptxas_verbose:
        sys.stderr.write(res.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(ptxas_verbose="--ptxas-verbose" in sys.argv, force=True))
