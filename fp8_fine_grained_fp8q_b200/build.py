"""Build libfp8q.so in-tree for B200 (sm_100a) with nvcc.

No fast-math: the quantisers must reproduce IEEE binary32 division and multiplication exactly
(they also use explicit __fdiv_rn / __fmul_rn).  The CUDA runtime is linked statically and the
driver's TMA-descriptor entry point is fetched at run time, so the library loads on machines
without a GPU driver (every call then returns FP8Q_ERR_CUDA).
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libfp8q.so")
LOG = os.path.join(PKG, "libfp8q.ptxas.txt")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared",
    "-Xptxas", "-v",
    "-cudart", "static",
]


def sources():
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".cu", ".cuh"))]


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + [os.path.join(INCLUDE, "fp8q.h"), os.path.abspath(__file__)]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC,
           os.path.join(CSRC, "fp8q.cu"), "-o", LIB + ".tmp"]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    with open(LOG, "w") as f:
        f.write(" ".join(cmd) + "\n" + proc.stdout + proc.stderr)
    if proc.returncode != 0:
        sys.stderr.write(proc.stdout + proc.stderr)
        raise RuntimeError(f"nvcc failed (exit {proc.returncode}); see {LOG}")
    if verbose:
        sys.stdout.write(proc.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv))
