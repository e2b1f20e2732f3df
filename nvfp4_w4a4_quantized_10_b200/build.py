"""Build libnvfp4.so (the C-ABI library) for sm_100a with nvcc, in-tree.

    python nvfp4_w4a4_quantized_10_b200/build.py [--force] [--verbose]

Objects go to ``_build/`` next to this file; the shared library lands at
``nvfp4_w4a4_quantized_10_b200/libnvfp4.so``.  Only the CUDA runtime is
linked (the driver's tensor-map encoder is looked up at run time).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC_DIR = os.path.join(HERE, "csrc")
BUILD_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libnvfp4.so")
SOURCES = ["runtime.cu", "quantize.cu", "gemm.cu", "harmonize.cu", "mxfp4.cu", "host_io.cu", "mma_peak.cu"]
HEADERS = ["ptx.cuh", "common.h", "block_quant.cuh", os.path.join("..", "..", "include", "nvfp4.h")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-ftz=false", "-prec-div=true", "-prec-sqrt=true", "-fmad=true"]


def _newer(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD_DIR, exist_ok=True)
    headers = [os.path.normpath(os.path.join(SRC_DIR, h)) for h in HEADERS]
    objs = []
    for src in SOURCES:
        s = os.path.join(SRC_DIR, src)
        o = os.path.join(BUILD_DIR, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _newer(o, [s] + headers):
            cmd = [NVCC] + ARCH + FLAGS + ["-c", s, "-o", o]
            if verbose:
                cmd += ["-Xptxas", "-v"]
                print(" ".join(cmd))
            subprocess.run(cmd, check=True)
    if force or _newer(LIB, objs):
        cmd = [NVCC] + ARCH + ["-shared", "-o", LIB + ".tmp"] + objs + ["-lcudart"]
        subprocess.run(cmd, check=True)
        os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
