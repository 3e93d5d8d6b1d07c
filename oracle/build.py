"""Build the CPU oracle (test infrastructure) into oracle/liboracle.so.

gcc, -O2 with -ffp-contract=off and no fast-math, so the oracle's float
arithmetic is plain IEEE binary32 with one rounding per operation.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "zero_oracle.c")
OUT = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
          "-fno-fast-math", "-fno-unsafe-math-optimizations", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile the oracle if the library is missing or older than its source."""
    hdr = os.path.join(HERE, "zero_oracle.h")
    if (not force and os.path.exists(OUT)
            and os.path.getmtime(OUT) >= max(os.path.getmtime(SRC), os.path.getmtime(hdr))):
        return OUT
    tmp = OUT + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
