"""Build libnvfp4.so (sm_100a) in-tree with nvcc.

-gencode arch=compute_100a,code=sm_100a; no fast-math, IEEE division and no
FMA contraction (--fmad=false) so the quantizer's FP32 steps are single
roundings in source order; relocatable device code so the kernels' translation
units share the device error word.  Concurrent callers serialise on a lock
file, so two processes never write the same object or library file.
"""
import fcntl
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libnvfp4.so")
SOURCES = ["amax.cu", "quantize.cu", "gemm.cu", "api.cu", "noalloc.cu"]
HEADERS = ["common.cuh", "kernels.h", "linear.h"]
PUBLIC_HEADER = os.path.join(os.path.dirname(HERE), "include", "nvfp4.h")
LOCK = os.path.join(HERE, ".build.lock")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17", "-rdc=true",
         "--fmad=false", "-prec-div=true", "-ftz=false", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2"]


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [PUBLIC_HEADER, __file__]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force=False, verbose=False):
    if not force and not _stale():
        return LIB
    with open(LOCK, "w") as lk:
        fcntl.flock(lk, fcntl.LOCK_EX)
        if force or _stale():
            _compile(verbose)
    return LIB


def _compile(verbose):
    objs = []
    for src in SOURCES:
        obj = os.path.join(CSRC, src.replace(".cu", ".o"))
        cmd = [NVCC, *FLAGS, "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = f"{LIB}.{os.getpid()}.tmp"
    subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-rdc=true", "-shared", "-Xcompiler",
                    "-fPIC", *objs, "-o", tmp], check=True)
    os.replace(tmp, LIB)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
