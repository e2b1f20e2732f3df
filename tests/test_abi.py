"""The C-ABI library loads and exports what include/nvfp4.h declares, and
argument validation rejects bad calls before touching the GPU (CPU only)."""
import ctypes

import numpy as np
import pytest

import nvfp4_w4a4_quantized_10_b200 as nv
import oracle


def test_every_declared_symbol_is_exported():
    names = nv.declared_symbols()
    assert len(names) >= 13
    for n in names:
        assert hasattr(nv.lib(), n), n          # ctypes resolves via dlsym
    # the binding offers each one under the same name (helpers excepted)
    for n in names:
        if n in ("nvfp4_status_string", "nvfp4_version"):
            continue
        assert hasattr(nv, n), n


def test_debug_build_exports_the_same_symbols():
    # the bounds-checked twin (NVFP4_DEBUG_BOUNDS=1) is a drop-in replacement
    import os
    path = os.path.join(os.path.dirname(nv.LIB_PATH), "libnvfp4_debug.so")
    assert os.path.exists(path), path
    dbg = ctypes.CDLL(path)
    for n in nv.declared_symbols():
        assert hasattr(dbg, n), n
    dbg.nvfp4_bounds_checked.restype = ctypes.c_int
    assert dbg.nvfp4_bounds_checked() == 1
    assert nv.nvfp4_bounds_checked() == nv.DEBUG_BOUNDS


def test_status_strings_and_version():
    assert nv.version() >= 100
    for s in range(7):
        assert nv.status_string(s) != "unknown status"
    assert nv.status_string(99) == "unknown status"


@pytest.mark.parametrize("rows,K", [(1, 32), (8, 5120), (129, 96), (300, 1088), (12384, 5120)])
def test_scale_bytes_matches_layout_definition(rows, K):
    assert nv.nvfp4_scale_bytes(rows, K, nv.SF_TCGEN05) == oracle.tc_scale_bytes(rows, K)
    assert nv.nvfp4_scale_bytes(rows, K, nv.SF_ROWMAJOR) == rows * K // 16
    assert nv.nvfp4_scale_bytes(0, K) == 0
    assert nv.nvfp4_scale_bytes(rows, 24) == 0


# Validation runs before any CUDA call, so these need no device.  Pointer
# values are never dereferenced on a failing check.
P = ctypes.c_void_p
A16 = P(0x10000)
A1 = P(0x10001)


def q(x=A16, dt=0, M=4, K=64, g=1.0, codes=A16, sc=A16, layout=1, amax=None):
    return nv.lib().nvfp4_quantize(x, dt, M, K, ctypes.c_float(g), codes, sc, layout, amax, None)


def test_quantize_validation():
    assert q(x=None) == nv.ERR_INVALID_ARG
    assert q(M=0) == nv.ERR_INVALID_ARG
    assert q(K=48) == nv.ERR_INVALID_ARG          # K % 32
    assert q(K=16) == nv.ERR_INVALID_ARG
    assert q(g=0.0) == nv.ERR_INVALID_ARG
    assert q(g=-1.0) == nv.ERR_INVALID_ARG
    assert q(g=float("inf")) == nv.ERR_INVALID_ARG
    assert q(g=float("nan")) == nv.ERR_INVALID_ARG
    assert q(dt=7) == nv.ERR_INVALID_ARG
    assert q(layout=5) == nv.ERR_INVALID_ARG
    assert q(x=A1) == nv.ERR_ALIGNMENT
    assert q(codes=A1) == nv.ERR_ALIGNMENT
    assert q(amax=P(0x10002)) == nv.ERR_ALIGNMENT


def g(a=A16, sa=A16, ga=1.0, w=A16, sw=A16, gw=1.0, M=8, N=16, K=64, out=A16, od=0):
    return nv.lib().nvfp4_gemm(a, sa, ctypes.c_float(ga), w, sw, ctypes.c_float(gw), M, N, K, out, od, None)


def test_gemm_validation():
    assert g(a=None) == nv.ERR_INVALID_ARG
    assert g(out=None) == nv.ERR_INVALID_ARG
    assert g(M=0) == nv.ERR_INVALID_ARG
    assert g(N=0) == nv.ERR_INVALID_ARG
    assert g(K=48) == nv.ERR_INVALID_ARG
    assert g(ga=0.0) == nv.ERR_INVALID_ARG
    assert g(gw=float("nan")) == nv.ERR_INVALID_ARG
    assert g(od=3) == nv.ERR_INVALID_ARG
    assert g(w=A1) == nv.ERR_ALIGNMENT
    assert g(out=A1) == nv.ERR_ALIGNMENT


def fused(offs, gs, n_seg=None, M=8, K=64):
    n = len(gs) if n_seg is None else n_seg
    o = (ctypes.c_int64 * len(offs))(*offs)
    s = (ctypes.c_float * max(1, len(gs)))(*gs)
    return nv.lib().nvfp4_fused_proj(A16, A16, ctypes.c_float(1.0), A16, A16, o, s, n, M, K, A16, 0, None)


def test_fused_validation():
    assert fused([0, 8, 8, 16], [1.0, 1.0, 1.0]) == nv.ERR_INVALID_ARG      # empty segment
    assert fused([1, 8, 16], [1.0, 1.0]) == nv.ERR_INVALID_ARG              # does not start at 0
    assert fused([0, 8, 16], [1.0, 0.0]) == nv.ERR_INVALID_ARG              # bad scale
    assert fused([0, 8, 16], [1.0, 1.0], n_seg=0) == nv.ERR_INVALID_ARG
    assert fused(list(range(0, 18 * 8, 8)), [1.0] * 17) == nv.ERR_INVALID_ARG  # too many


def test_other_validation():
    L = nv.lib()
    assert L.nvfp4_amax(None, 0, 4, 64, A16, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_amax(A1, 0, 4, 64, A16, None) == nv.ERR_ALIGNMENT
    assert L.nvfp4_swizzle_scales(A16, 0, 64, A16, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_swizzle_scales(A16, 4, 64, A1, None) == nv.ERR_ALIGNMENT
    assert L.nvfp4_convert_e2m1(A16, A16, 3, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_convert_e4m3(None, A16, 3, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_test_wait_timeout(0, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_test_wait_timeout(11_000_000_000, None) == nv.ERR_INVALID_ARG


def harm(offs, gs, g=1.0, N=16, K=64, layout=1, sc=A16, out=A16, n_seg=None):
    n = len(gs) if n_seg is None else n_seg
    o = (ctypes.c_int64 * len(offs))(*offs)
    s = (ctypes.c_float * max(1, len(gs)))(*gs)
    return nv.lib().nvfp4_harmonize_scales(sc, N, K, layout, o, s, n, ctypes.c_float(g), out, None)


def test_harmonize_and_calibration_validation():
    assert harm([0, 8, 16], [1.0, 2.0], sc=None) == nv.ERR_INVALID_ARG
    assert harm([0, 8, 16], [1.0, 2.0], out=None) == nv.ERR_INVALID_ARG
    assert harm([0, 8, 16], [1.0, 2.0], N=0) == nv.ERR_INVALID_ARG
    assert harm([0, 8, 16], [1.0, 2.0], K=24) == nv.ERR_INVALID_ARG
    assert harm([0, 8, 16], [1.0, 2.0], layout=4) == nv.ERR_INVALID_ARG
    assert harm([0, 8, 16], [1.0, 2.0], g=0.0) == nv.ERR_INVALID_ARG
    assert harm([0, 8, 16], [1.0, 2.0], g=float("nan")) == nv.ERR_INVALID_ARG
    assert harm([0, 8, 16], [1.0, -2.0]) == nv.ERR_INVALID_ARG             # bad segment scale
    assert harm([0, 8, 8], [1.0, 2.0]) == nv.ERR_INVALID_ARG               # empty segment
    assert harm([2, 8, 16], [1.0, 2.0]) == nv.ERR_INVALID_ARG              # does not start at 0
    assert harm([0, 8, 17], [1.0, 2.0]) == nv.ERR_INVALID_ARG              # beyond N
    assert harm([0, 8, 16], [1.0, 2.0], n_seg=0) == nv.ERR_INVALID_ARG
    assert harm(list(range(17)), [1.0] * 17, N=32) == nv.ERR_INVALID_ARG   # too many
    assert harm([0, 8, 16], [1.0, 2.0], sc=A1) == nv.ERR_ALIGNMENT
    assert harm([0, 8, 16], [1.0, 2.0], out=A1) == nv.ERR_ALIGNMENT
    L = nv.lib()
    assert L.nvfp4_amax_accumulate(None, 0, 4, 64, A16, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_amax_accumulate(A16, 0, 4, 64, None, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_amax_accumulate(A16, 0, 0, 64, A16, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_amax_accumulate(A16, 0, 1, 4, A16, None) == nv.ERR_INVALID_ARG   # 8 bytes
    assert L.nvfp4_amax_accumulate(A16, 5, 4, 64, A16, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_amax_accumulate(A1, 0, 4, 64, A16, None) == nv.ERR_ALIGNMENT
    assert L.nvfp4_amax_accumulate(A16, 0, 4, 64, P(0x10002), None) == nv.ERR_ALIGNMENT


def test_mx_validation():
    L = nv.lib()
    assert L.nvfp4_mx_quantize(None, 0, 4, 64, A16, A16, 1, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_mx_quantize(A16, 0, 0, 64, A16, A16, 1, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_mx_quantize(A16, 0, 4, 48, A16, A16, 1, None) == nv.ERR_INVALID_ARG   # K % 32
    assert L.nvfp4_mx_quantize(A16, 3, 4, 64, A16, A16, 1, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_mx_quantize(A16, 0, 4, 64, A16, A16, 2, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_mx_quantize(A1, 0, 4, 64, A16, A16, 1, None) == nv.ERR_ALIGNMENT
    assert L.nvfp4_mx_quantize(A16, 0, 4, 64, A16, A1, 1, None) == nv.ERR_ALIGNMENT
    assert L.nvfp4_mx_gemm(None, A16, A16, A16, 8, 16, 64, A16, 0, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_mx_gemm(A16, A16, A16, A16, 0, 16, 64, A16, 0, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_mx_gemm(A16, A16, A16, A16, 8, 16, 48, A16, 0, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_mx_gemm(A16, A16, A16, A16, 8, 16, 64, A16, 2, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_mx_gemm(A16, A16, A1, A16, 8, 16, 64, A16, 0, None) == nv.ERR_ALIGNMENT


def lin(x=A16, dt=0, M=8, K=64, ga=1.0, w=A16, sw=A16, gw=1.0, N=64, out=A16, od=0, ac=None, asc=None):
    return nv.lib().nvfp4_linear(x, dt, M, K, ctypes.c_float(ga), w, sw, ctypes.c_float(gw), N, out, od, ac, asc,
                                 None)


def test_linear_validation():
    assert lin(x=None) == nv.ERR_INVALID_ARG
    assert lin(w=None) == nv.ERR_INVALID_ARG
    assert lin(out=None) == nv.ERR_INVALID_ARG
    assert lin(M=0) == nv.ERR_INVALID_ARG
    assert lin(N=0) == nv.ERR_INVALID_ARG
    assert lin(K=48) == nv.ERR_INVALID_ARG
    assert lin(dt=3) == nv.ERR_INVALID_ARG
    assert lin(od=3) == nv.ERR_INVALID_ARG
    assert lin(ga=float("inf")) == nv.ERR_INVALID_ARG
    assert lin(gw=0.0) == nv.ERR_INVALID_ARG
    assert lin(x=A1) == nv.ERR_ALIGNMENT
    assert lin(sw=A1) == nv.ERR_ALIGNMENT


def test_linear_host_validation():
    L = nv.lib()

    def lh(xh=A16, dt=0, M=8, K=64, ga=1.0, w=A16, sw=A16, gw=1.0, N=64, oh=A16, od=0, xd=A16, od_=A16):
        return L.nvfp4_linear_host(xh, dt, M, K, ctypes.c_float(ga), w, sw, ctypes.c_float(gw), N, oh, od, xd, None,
                                   None, od_, None)
    assert lh(xh=None) == nv.ERR_INVALID_ARG
    assert lh(oh=None) == nv.ERR_INVALID_ARG
    assert lh(xd=None) == nv.ERR_INVALID_ARG
    assert lh(od_=None) == nv.ERR_INVALID_ARG
    assert lh(M=0) == nv.ERR_INVALID_ARG
    assert lh(K=48) == nv.ERR_INVALID_ARG
    assert lh(dt=2) == nv.ERR_INVALID_ARG
    assert lh(od=2) == nv.ERR_INVALID_ARG
    assert lh(ga=0.0) == nv.ERR_INVALID_ARG
    assert lh(xd=A1) == nv.ERR_ALIGNMENT
    assert lh(od_=A1) == nv.ERR_ALIGNMENT


def test_declare_static_validation():
    L = nv.lib()
    assert L.nvfp4_declare_static(None, 64) == nv.ERR_INVALID_ARG
    assert L.nvfp4_declare_static(A16, 0) == nv.ERR_INVALID_ARG
    assert L.nvfp4_declare_static(A16, 64) == nv.OK
    L.nvfp4_forget_static()


def test_product_package_does_not_import_the_oracle():
    import pathlib
    pkg = pathlib.Path(nv.__file__).parent
    for f in list(pkg.rglob("*.py")) + list(pkg.rglob("*.cu")) + list(pkg.rglob("*.cuh")) + list(pkg.rglob("*.h")):
        text = f.read_text()
        assert "import oracle" not in text and "from oracle" not in text, f
        assert "liboracle" not in text, f
