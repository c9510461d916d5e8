"""Build libsfa.so in-tree with nvcc for sm_100a.

    python -m sparse_attention_backward_sfa_b200.build
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCES = ["sfa_api.cu", "sfa_prep.cu", "sfa_generic.cu", "fa_generic.cu", "sfa_fused.cu", "sfa_noalloc.cu", "fa_fused.cu",
           "sfa_fwd_fused.cu", "lig_fused.cu", "sfa_pair.cu"]
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
         "-shared", "-Xptxas", "-warn-spills"]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def build(verbose: bool = False) -> str:
    out = os.path.join(HERE, "libsfa.so")
    srcs = [os.path.join(HERE, "csrc", s) for s in SOURCES]
    deps = srcs + glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + [os.path.join(HERE, "..", "include", "sfa.h")]
    if os.path.exists(out) and all(os.path.getmtime(out) >= os.path.getmtime(d) for d in deps):
        return out
    cmd = [nvcc(), *FLAGS, "-o", out + ".tmp", *srcs]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed ({r.returncode}):\n{r.stdout}\n{r.stderr}")
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(verbose=True))
