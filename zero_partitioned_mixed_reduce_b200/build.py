"""Build libzero_b200.so in-tree for sm_100a.

Kernels: nvcc -gencode arch=compute_100a,code=sm_100a, -O3, --fmad=false (no
multiply-add contraction anywhere in the step), no fast-math (IEEE division
and square root, no flush-to-zero). Host C++: g++ -O2. The CUDA runtime is
linked statically.
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
OUT = os.path.join(PKG, "libzero_b200.so")
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")
NVCC = os.path.join(CUDA_HOME, "bin", "nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", *ARCH, "-lineinfo", "--fmad=false", "-Xptxas", "-v",
              "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC]
CXX_FLAGS = ["-O2", "-std=c++17", "-fPIC", "-Wall", "-Wextra", "-ffp-contract=off",
             "-fno-fast-math", "-I", INCLUDE, "-I", CSRC, "-I", os.path.join(CUDA_HOME, "include")]
# the host AdamW loop is vectorized (target_clones picks AVX-512 / AVX2 / baseline)
CXX_EXTRA = {"cpu_adam.cpp": ["-O3", "-pthread"]}

CU_SOURCES = ["kernels.cu", "noalloc.cu"]
CPP_SOURCES = ["plan.cpp", "capi.cpp", "sched.cpp", "cpu_adam.cpp"]


def _sources():
    return ([os.path.join(CSRC, s) for s in CU_SOURCES + CPP_SOURCES + ["internal.h", "device_common.cuh"]]
            + [os.path.join(INCLUDE, "zero_b200.h")])


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(s) <= t for s in _sources())


def _run(cmd, log=None):
    r = subprocess.run(cmd, capture_output=True, text=True)
    if log is not None:
        with open(log, "w") as f:
            f.write(r.stdout + r.stderr)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"build step failed: {' '.join(cmd[:3])} ...")
    return r


def build(force: bool = False) -> str:
    """Compile the library if it is missing or older than any source."""
    if not force and up_to_date():
        return OUT
    os.makedirs(BUILD, exist_ok=True)
    objs = []
    for s in CU_SOURCES:
        o = os.path.join(BUILD, s + ".o")
        _run([NVCC, *NVCC_FLAGS, "-c", os.path.join(CSRC, s), "-o", o],
             log=os.path.join(BUILD, s + ".ptxas.txt"))
        objs.append(o)
    for s in CPP_SOURCES:
        o = os.path.join(BUILD, s + ".o")
        _run(["g++", *CXX_FLAGS, *CXX_EXTRA.get(s, []), "-c", os.path.join(CSRC, s), "-o", o])
        objs.append(o)
    tmp = OUT + f".tmp{os.getpid()}"
    _run([NVCC, "-shared", *ARCH, "-cudart=static", *objs, "-o", tmp, "-Xcompiler", "-pthread"])
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
