"""Build libzero_b200.so in-tree for sm_100a.

Kernels: nvcc -gencode arch=compute_100a,code=sm_100a, -O3, --fmad=false (no
multiply-add contraction anywhere in the step), no fast-math (IEEE division
and square root, no flush-to-zero). Host C++: g++ -O2. The CUDA runtime is
linked statically.

build(debug=True) makes libzero_b200_debug.so instead: the same sources with
ZERO_DEBUG_BOUNDS defined, so every kernel checks the indices and pointers it
derives before each access, skips a failing access and records it (read back
with zero_debug_bounds). It is a test build, loaded through ZERO_B200_LIB.
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
OUT_DEBUG = os.path.join(PKG, "libzero_b200_debug.so")
BUILD_DEBUG = os.path.join(ROOT, "_build_debug")
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")
NVCC = os.path.join(CUDA_HOME, "bin", "nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", *ARCH, "-lineinfo", "--fmad=false", "-Xptxas", "-v",
              "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC]
CXX_FLAGS = ["-O2", "-std=c++17", "-fPIC", "-Wall", "-Wextra", "-ffp-contract=off",
             "-fno-fast-math", "-I", INCLUDE, "-I", CSRC, "-I", os.path.join(CUDA_HOME, "include")]
# the host AdamW loop is vectorized (target_clones picks AVX-512 / AVX2 / baseline);
# -fno-math-errno drops sqrt's errno branch, which blocks vectorization and
# does not change any result (sqrt is correctly rounded either way)
CXX_EXTRA = {"cpu_adam.cpp": ["-O3", "-pthread", "-fno-math-errno"]}

CU_SOURCES = ["kernels.cu", "noalloc.cu", "norm_slots.cu"]
CPP_SOURCES = ["plan.cpp", "capi.cpp", "sched.cpp", "cpu_adam.cpp", "trace.cpp", "ipc.cpp"]


def _sources():
    return ([os.path.join(CSRC, s) for s in CU_SOURCES + CPP_SOURCES + ["internal.h", "device_common.cuh", "debug_bounds.cuh"]]
            + [os.path.join(INCLUDE, "zero_b200.h")])


def up_to_date(out=OUT) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
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


def build(force: bool = False, debug: bool = False) -> str:
    """Compile the library if it is missing or older than any source."""
    out, bdir = (OUT_DEBUG, BUILD_DEBUG) if debug else (OUT, BUILD)
    if not force and up_to_date(out):
        return out
    os.makedirs(bdir, exist_ok=True)
    extra = ["-DZERO_DEBUG_BOUNDS"] if debug else []
    objs = []
    for s in CU_SOURCES:
        o = os.path.join(bdir, s + ".o")
        _run([NVCC, *NVCC_FLAGS, *extra, "-c", os.path.join(CSRC, s), "-o", o],
             log=os.path.join(bdir, s + ".ptxas.txt"))
        objs.append(o)
    for s in CPP_SOURCES:
        o = os.path.join(bdir, s + ".o")
        _run(["g++", *CXX_FLAGS, *extra, *CXX_EXTRA.get(s, []), "-c", os.path.join(CSRC, s), "-o", o])
        objs.append(o)
    tmp = out + f".tmp{os.getpid()}"
    _run([NVCC, "-shared", *ARCH, "-cudart=static", *objs, "-o", tmp, "-Xcompiler", "-pthread"])
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, debug="--debug" in sys.argv))
