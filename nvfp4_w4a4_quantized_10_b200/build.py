"""Build libnvfp4.so (the C-ABI library) for sm_100a with nvcc, in-tree, and
its debug twin libnvfp4_debug.so (the same sources with NVFP4_BOUNDS_CHECK=1:
every global address a kernel computes is checked against its buffer, and a
failed check sets the device error word instead of touching memory).

    python nvfp4_w4a4_quantized_10_b200/build.py [--force] [--verbose] [--no-debug]

Objects go to ``_build/`` (``_build/debug/``) next to this file; the shared
libraries land beside it.  Only the CUDA runtime is linked (the driver's
tensor-map encoder is looked up at run time).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC_DIR = os.path.join(HERE, "csrc")
BUILD_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libnvfp4.so")
DEBUG_LIB = os.path.join(HERE, "libnvfp4_debug.so")
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


def _build_one(lib: str, build_dir: str, defines, force: bool, verbose: bool) -> str:
    os.makedirs(build_dir, exist_ok=True)
    headers = [os.path.normpath(os.path.join(SRC_DIR, h)) for h in HEADERS]
    objs = []
    for src in SOURCES:
        s = os.path.join(SRC_DIR, src)
        o = os.path.join(build_dir, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _newer(o, [s] + headers):
            cmd = [NVCC] + ARCH + FLAGS + defines + ["-c", s, "-o", o]
            if verbose:
                cmd += ["-Xptxas", "-v"]
                print(" ".join(cmd))
            subprocess.run(cmd, check=True)
    if force or _newer(lib, objs):
        cmd = [NVCC] + ARCH + ["-shared", "-o", lib + ".tmp"] + objs + ["-lcudart"]
        subprocess.run(cmd, check=True)
        os.replace(lib + ".tmp", lib)
    return lib


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Build the release library (returned) and, unless debug=False, the
    bounds-checked debug library."""
    _build_one(LIB, BUILD_DIR, [], force, verbose)
    if debug:
        _build_one(DEBUG_LIB, os.path.join(BUILD_DIR, "debug"), ["-DNVFP4_BOUNDS_CHECK=1"], force, verbose)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, debug="--no-debug" not in sys.argv))
