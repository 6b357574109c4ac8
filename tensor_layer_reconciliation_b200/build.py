"""Compile the CUDA library ``libtp_reconcile.so`` in-tree with nvcc for sm_100a.

One translation unit (csrc/tp_reconcile.cu includes the kernel headers). The
CUDA runtime is linked statically, so the library needs no libcudart at load
time; the driver's TMA-descriptor encoder is looked up at run time through the
runtime's driver entry-point query, so it needs no libcuda at link time either.
No fast-math: bf16 and fp32 subnormals and round-to-nearest-even are kept.
"""

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libtp_reconcile.so")
MAIN = os.path.join(CSRC, "tp_reconcile.cu")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-std=c++17", "-O3", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
         "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared", "-cudart", "static",
         "-I", INCLUDE, "-I", CSRC]


def _sources():
    out = [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    out += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh", ".h"))]
    return out


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(s) for s in _sources())
        if os.path.getmtime(LIB) >= newest:
            return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, MAIN, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
