"""Build libtf.so in-tree with nvcc for sm_100a (B200).

    python row_split_int4_b200/build.py [-v]

Compiles every .cu file under csrc/ into one shared library next to this
file.  The CUDA runtime is linked as a shared library so that the process
uses one runtime instance together with PyTorch.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libtf.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC,-O2",
         "-cudart", "shared", f"-Xlinker=-rpath,{CUDA_HOME}/lib64", f"-I{INCLUDE}"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))) + \
        [os.path.join(INCLUDE, "tf.h"), os.path.abspath(__file__)]


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in deps())


def build(verbose: bool = False, force: bool = False, ptxas_v: bool = False) -> str:
    if not force and not stale():
        return LIB
    nvcc = os.path.join(CUDA_HOME, "bin", "nvcc")
    cmd = [nvcc, *ARCH, *FLAGS, "-shared", *sources(), "-o", LIB + ".tmp"]
    if ptxas_v:
        cmd.insert(1, "-Xptxas=-v")
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed ({r.returncode}):\n{r.stdout}\n{r.stderr}")
    if verbose or ptxas_v:
        print(r.stdout + r.stderr, file=sys.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(verbose="-v" in sys.argv, force=True, ptxas_v="--ptxas" in sys.argv)
    print(LIB)
