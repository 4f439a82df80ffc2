"""Build the oracle's shared library (plain C, gcc).

Test infrastructure only: this builds the CPU checker, never the product.
`libsvo.so` is compiled with OpenMP so that the same source can also run its
request loop on several host threads (the benchmark's CPU baseline); with
``nthreads=1`` it is the plain single-threaded loop.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "svo.c")
HDR = os.path.join(HERE, "svo.h")
LIB = os.path.join(HERE, "libsvo.so")

CFLAGS = [
    "-O2",
    "-std=c11",
    "-fPIC",
    "-shared",
    "-fopenmp",
    # keep every multiply and add separately rounded, as written
    "-ffp-contract=off",
    "-fno-fast-math",
    "-Wall",
    "-Wno-unused-function",
]


def build(force: bool = False) -> str:
    """Compile oracle/libsvo.so when it is missing or older than its sources."""
    if not force and os.path.exists(LIB):
        lib_t = os.path.getmtime(LIB)
        if lib_t >= os.path.getmtime(SRC) and lib_t >= os.path.getmtime(HDR):
            return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
