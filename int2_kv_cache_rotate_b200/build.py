"""Build ``libokv.so`` in-tree with nvcc for sm_100a (no JIT cache, no torch extension).

Usage: ``python -m int2_kv_cache_rotate_b200.build [--verbose-ptxas] [--short-wait]``.
``--short-wait`` builds the test library ``libokv_shortwait.so`` instead: every
bounded wait of the kernels gives up after 64 cycles (the waits of the timeout
paths for work already issued keep their full limit), so that a test can run
the timeout paths.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libokv.so")
SHORT_WAIT_LIB = os.path.join(HERE, "libokv_shortwait.so")
SOURCES = ["okv_api.cu", "append.cu", "decode.cu", "dequant.cu", "prefill.cu", "noalloc.cu", "calib.cpp",
           "rotio.cpp"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def build(verbose_ptxas: bool = False, out: str = LIB, short_wait: bool = False) -> str:
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    defs = ["-DOKV_WAIT_LIMIT_LOG2=6"] if short_wait else []
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", *defs,
           "-Xcompiler", "-fPIC,-fopenmp,-O3", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           "-o", out, *srcs, "-lgomp"]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose_ptxas:
        sys.stderr.write(res.stderr)
    return out


if __name__ == "__main__":
    if "--short-wait" in sys.argv:
        print(build(verbose_ptxas="--verbose-ptxas" in sys.argv, out=SHORT_WAIT_LIB, short_wait=True))
    else:
        print(build(verbose_ptxas="--verbose-ptxas" in sys.argv))
