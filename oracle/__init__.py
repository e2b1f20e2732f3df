"""CPU oracle for the NVFP4 W4A4 linear layer (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
CUDA library and its Python binding never import it, and it imports nothing
from them.  Every function here only marshals numpy arrays into the plain C
implementation in ``nvfp4_oracle.c``; the arithmetic and the citations live
there.

Functions with no independent pin: none (every function is pinned by
``tests/test_oracle_*.py``).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        i64 = ctypes.c_int64
        L.orc_e2m1_decode.restype = ctypes.c_double
        L.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.orc_e2m1_encode.restype = ctypes.c_uint8
        L.orc_e2m1_encode.argtypes = [ctypes.c_float]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_encode.argtypes = [ctypes.c_float]
        L.orc_e2m1_encode_array.argtypes = [f32p, u8p, i64]
        L.orc_e4m3_encode_array.argtypes = [f32p, u8p, i64]
        L.orc_amax.restype = ctypes.c_float
        L.orc_amax.argtypes = [f32p, i64]
        L.orc_global_scale.restype = ctypes.c_float
        L.orc_global_scale.argtypes = [ctypes.c_float]
        L.orc_quantize.argtypes = [f32p, i64, i64, ctypes.c_float, u8p, u8p]
        L.orc_dequantize.argtypes = [u8p, u8p, ctypes.c_float, i64, i64, f64p]
        L.orc_tc_scale_bytes.restype = i64
        L.orc_tc_scale_bytes.argtypes = [i64, i64]
        L.orc_scales_to_tc.argtypes = [u8p, i64, i64, u8p]
        L.orc_scales_from_tc.argtypes = [u8p, i64, i64, u8p]
        L.orc_gemm.argtypes = [u8p, u8p, ctypes.c_float, u8p, u8p, ctypes.c_float,
                               i64, i64, i64, f64p]
        L.orc_fused_proj.argtypes = [u8p, u8p, ctypes.c_float, u8p, u8p, i64p, f32p,
                                     ctypes.c_int, i64, i64, f64p]
        L.orc_gemm_exact.argtypes = [u8p, u8p, u8p, u8p, i64, i64, i64, i64p]
        L.orc_saturation.argtypes = [f32p, i64, i64, ctypes.c_float, i64p]
        L.orc_harmonize_scales.argtypes = [u8p, i64, i64, i64p, f32p, ctypes.c_int,
                                           ctypes.c_float, u8p]
        L.orc_e8m0_decode.restype = ctypes.c_double
        L.orc_e8m0_decode.argtypes = [ctypes.c_uint8]
        L.orc_mx_scale.restype = ctypes.c_uint8
        L.orc_mx_scale.argtypes = [ctypes.c_float]
        L.orc_mx_quantize.argtypes = [f32p, i64, i64, u8p, u8p]
        L.orc_mx_dequantize.argtypes = [u8p, u8p, i64, i64, f64p]
        L.orc_mx_gemm.argtypes = [u8p, u8p, u8p, u8p, i64, i64, i64, f64p]
        L.orc_set_threads.argtypes = [ctypes.c_int]
        L.orc_get_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def get_threads() -> int:
    return int(lib().orc_get_threads())


# ---- scalar codecs -------------------------------------------------------

def e2m1_decode(code: int) -> float:
    return lib().orc_e2m1_decode(code)


def e2m1_encode(v: float) -> int:
    return lib().orc_e2m1_encode(v)


def e4m3_decode(code: int) -> float:
    return lib().orc_e4m3_decode(code)


def e4m3_encode(t: float) -> int:
    return lib().orc_e4m3_encode(t)


def e2m1_encode_array(v):
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e2m1_encode_array(_p(v, ctypes.c_float), _p(out, ctypes.c_uint8), v.size)
    return out


def e4m3_encode_array(v):
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e4m3_encode_array(_p(v, ctypes.c_float), _p(out, ctypes.c_uint8), v.size)
    return out


# ---- tensor-level --------------------------------------------------------

def amax(x) -> np.float32:
    x = _c(x, np.float32)
    return np.float32(lib().orc_amax(_p(x, ctypes.c_float), x.size))


def global_scale(amax_value) -> np.float32:
    return np.float32(lib().orc_global_scale(float(amax_value)))


def quantize(x, g):
    """x: [M, K] float32 (K % 16 == 0). Returns (codes [M,K/2] u8, scales [M,K/16] u8)."""
    x = _c(x, np.float32)
    M, K = x.shape
    assert K % 16 == 0
    codes = np.empty((M, K // 2), np.uint8)
    scales = np.empty((M, K // 16), np.uint8)
    lib().orc_quantize(_p(x, ctypes.c_float), M, K, float(np.float32(g)),
                       _p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8))
    return codes, scales


def dequantize(codes, scales, g):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    M = codes.shape[0]
    K = codes.shape[1] * 2
    out = np.empty((M, K), np.float64)
    lib().orc_dequantize(_p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8),
                         float(np.float32(g)), M, K, _p(out, ctypes.c_double))
    return out


def tc_scale_bytes(R: int, K: int) -> int:
    return int(lib().orc_tc_scale_bytes(R, K))


def scales_to_tc(rowmajor, K: int):
    rowmajor = _c(rowmajor, np.uint8)
    R = rowmajor.shape[0]
    out = np.empty(tc_scale_bytes(R, K), np.uint8)
    lib().orc_scales_to_tc(_p(rowmajor, ctypes.c_uint8), R, K, _p(out, ctypes.c_uint8))
    return out


def scales_from_tc(tc, R: int, K: int):
    tc = _c(tc, np.uint8)
    out = np.empty((R, K // 16), np.uint8)
    lib().orc_scales_from_tc(_p(tc, ctypes.c_uint8), R, K, _p(out, ctypes.c_uint8))
    return out


def gemm(a_codes, a_scales, a_gs, w_codes, w_scales, w_gs):
    """FP64 [M, N] = dequant(A) @ dequant(W)^T."""
    a_codes, a_scales = _c(a_codes, np.uint8), _c(a_scales, np.uint8)
    w_codes, w_scales = _c(w_codes, np.uint8), _c(w_scales, np.uint8)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = w_codes.shape[0]
    assert w_codes.shape[1] * 2 == K
    out = np.empty((M, N), np.float64)
    lib().orc_gemm(_p(a_codes, ctypes.c_uint8), _p(a_scales, ctypes.c_uint8),
                   float(np.float32(a_gs)), _p(w_codes, ctypes.c_uint8),
                   _p(w_scales, ctypes.c_uint8), float(np.float32(w_gs)), M, N, K,
                   _p(out, ctypes.c_double))
    return out


def fused_proj(a_codes, a_scales, a_gs, w_codes, w_scales, seg_offsets, seg_gs):
    a_codes, a_scales = _c(a_codes, np.uint8), _c(a_scales, np.uint8)
    w_codes, w_scales = _c(w_codes, np.uint8), _c(w_scales, np.uint8)
    offs = _c(seg_offsets, np.int64)
    gs = _c(seg_gs, np.float32)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = int(offs[-1])
    assert w_codes.shape[0] == N
    out = np.empty((M, N), np.float64)
    lib().orc_fused_proj(_p(a_codes, ctypes.c_uint8), _p(a_scales, ctypes.c_uint8),
                         float(np.float32(a_gs)), _p(w_codes, ctypes.c_uint8),
                         _p(w_scales, ctypes.c_uint8), _p(offs, ctypes.c_int64),
                         _p(gs, ctypes.c_float), len(gs), M, K, _p(out, ctypes.c_double))
    return out


def gemm_exact(a_codes, a_scales, w_codes, w_scales):
    """Integer S with sum_k e2m1*e4m3*e2m1*e4m3 == S * 2**-20 exactly."""
    a_codes, a_scales = _c(a_codes, np.uint8), _c(a_scales, np.uint8)
    w_codes, w_scales = _c(w_codes, np.uint8), _c(w_scales, np.uint8)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = w_codes.shape[0]
    S = np.empty((M, N), np.int64)
    lib().orc_gemm_exact(_p(a_codes, ctypes.c_uint8), _p(a_scales, ctypes.c_uint8),
                         _p(w_codes, ctypes.c_uint8), _p(w_scales, ctypes.c_uint8),
                         M, N, K, _p(S, ctypes.c_int64))
    return S


# ---- static calibration and offline harmonisation ------------------------

def calibrate_amax(batches) -> np.float32:
    """Largest magnitude over several calibration batches: the running maximum
    of the per-batch amax, the statistic a static global scale is built from
    (anthology record LIT-800, "Key takeaways": calibration-only recipe)."""
    m = np.float32(0.0)
    for b in batches:
        m = max(m, amax(b))
    return np.float32(m)


def saturation(x, g):
    """(blocks with a clipped scale, elements with a clipped code, blocks whose
    scale underflowed to zero) when x is quantized with global scale g."""
    x = _c(x, np.float32)
    M, K = x.shape
    counts = np.zeros(3, np.int64)
    lib().orc_saturation(_p(x, ctypes.c_float), M, K, float(np.float32(g)), _p(counts, ctypes.c_int64))
    return tuple(int(c) for c in counts)


def harmonize_scales(scales, seg_offsets, seg_gs, g):
    """Row-major block scales [R, K/16] of a fused weight rewritten from
    per-segment global scales seg_gs to one common scale g (codes unchanged)."""
    scales = _c(scales, np.uint8)
    R, nb = scales.shape
    offs = _c(seg_offsets, np.int64)
    gs = _c(seg_gs, np.float32)
    out = np.empty_like(scales)
    lib().orc_harmonize_scales(_p(scales, ctypes.c_uint8), R, nb * 16, _p(offs, ctypes.c_int64),
                               _p(gs, ctypes.c_float), len(gs), float(np.float32(g)),
                               _p(out, ctypes.c_uint8))
    return out


# ---- MXFP4 (the contrast format) -------------------------------------------

def e8m0_decode(b: int) -> float:
    return float(lib().orc_e8m0_decode(b))


def mx_scale(amax) -> int:
    return int(lib().orc_mx_scale(float(np.float32(amax))))


def mx_quantize(x):
    """x: [M, K] float32 (K % 32 == 0). Returns (codes [M,K/2] u8, E8M0 scales [M,K/32] u8)."""
    x = _c(x, np.float32)
    M, K = x.shape
    assert K % 32 == 0
    codes = np.empty((M, K // 2), np.uint8)
    scales = np.empty((M, K // 32), np.uint8)
    lib().orc_mx_quantize(_p(x, ctypes.c_float), M, K, _p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8))
    return codes, scales


def mx_dequantize(codes, scales):
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint8)
    M, K = codes.shape[0], codes.shape[1] * 2
    out = np.empty((M, K), np.float64)
    lib().orc_mx_dequantize(_p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8), M, K, _p(out, ctypes.c_double))
    return out


def mx_gemm(a_codes, a_scales, w_codes, w_scales):
    a_codes, a_scales = _c(a_codes, np.uint8), _c(a_scales, np.uint8)
    w_codes, w_scales = _c(w_codes, np.uint8), _c(w_scales, np.uint8)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = w_codes.shape[0]
    out = np.empty((M, N), np.float64)
    lib().orc_mx_gemm(_p(a_codes, ctypes.c_uint8), _p(a_scales, ctypes.c_uint8), _p(w_codes, ctypes.c_uint8),
                      _p(w_scales, ctypes.c_uint8), M, N, K, _p(out, ctypes.c_double))
    return out


def mx_scales_to_tc(rowmajor, K: int):
    """MX scales [R, K/32] in the tensor-core chunk order.  The order depends
    only on the scale matrix's shape (128 rows x 4 scales per 512-byte chunk),
    so it is the NVFP4 order of a matrix with K/32 scales per row."""
    return scales_to_tc(rowmajor, K // 2)


def mx_scales_from_tc(tc, R: int, K: int):
    return scales_from_tc(tc, R, K // 2)
