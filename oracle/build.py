"""Build the CPU oracle shared library (test infrastructure only).

gcc, -O2, no fast-math and no FP contraction, so the oracle's FP32 steps are
single IEEE operations in source order; OpenMP for the large parity cases.
Concurrent callers (test ranks started together) serialise on a lock file and
write through a per-process temporary, so none can load a half-written file.
"""
import fcntl
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "nvfp4_oracle.c")
LIB = os.path.join(HERE, "libnvfp4_oracle.so")
LOCK = os.path.join(HERE, ".build.lock")

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
          "-std=c11", "-Wall", "-Wextra", "-Wno-unused-parameter"]


def _fresh():
    return os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC)


def build(force: bool = False) -> str:
    if not force and _fresh():
        return LIB
    with open(LOCK, "w") as lk:
        fcntl.flock(lk, fcntl.LOCK_EX)
        if force or not _fresh():
            tmp = f"{LIB}.{os.getpid()}.tmp"
            subprocess.run(["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"], check=True)
            os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
