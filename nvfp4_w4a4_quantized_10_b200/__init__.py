"""Python binding of the NVFP4 W4A4 linear-layer library (libnvfp4.so).

Argument marshalling only: every function below passes raw device pointers,
sizes and the current CUDA stream of the given tensors to the C-ABI function
of the same name (declared in ``include/nvfp4.h``) and raises ``Nvfp4Error``
on a non-OK status.  All quantization and GEMM work runs in the library's
CUDA kernels; there is no CPU fallback.  PyTorch supplies device memory and
streams.

The library is built in-tree by ``python nvfp4_w4a4_quantized_10_b200/build.py``;
importing this package without it raises ImportError.  With the environment
variable NVFP4_DEBUG_BOUNDS=1 the package loads the bounds-checked debug build
(libnvfp4_debug.so) instead: same entry points and results, and a kernel
address outside its buffer is reported (NVFP4_ERR_DEVICE from
nvfp4_last_device_error) instead of being accessed.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
DEBUG_BOUNDS = os.environ.get("NVFP4_DEBUG_BOUNDS", "0") not in ("", "0")
LIB_PATH = os.path.join(HERE, "libnvfp4_debug.so" if DEBUG_BOUNDS else "libnvfp4.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "nvfp4.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{os.path.basename(LIB_PATH)} is not built ({LIB_PATH}); run "
                      "`python nvfp4_w4a4_quantized_10_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

# status / enums (mirror include/nvfp4.h)
OK, ERR_INVALID_ARG, ERR_ALIGNMENT, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE = range(7)
IN_BF16, IN_F32 = 0, 1
OUT_BF16, OUT_F32 = 0, 1
SF_ROWMAJOR, SF_TCGEN05 = 0, 1
MAX_SEGMENTS = 16

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_f32 = ctypes.c_float

_lib.nvfp4_scale_bytes.restype = ctypes.c_size_t
_lib.nvfp4_scale_bytes.argtypes = [_i64, _i64, ctypes.c_int]
_lib.nvfp4_amax.argtypes = [_vp, ctypes.c_int, _i64, _i64, _vp, _vp]
_lib.nvfp4_amax_accumulate.argtypes = [_vp, ctypes.c_int, _i64, _i64, _vp, _vp]
_lib.nvfp4_harmonize_scales.argtypes = [_vp, _i64, _i64, ctypes.c_int, ctypes.POINTER(_i64), ctypes.POINTER(_f32),
                                        ctypes.c_int, _f32, _vp, _vp]
_lib.nvfp4_mx_quantize.argtypes = [_vp, ctypes.c_int, _i64, _i64, _vp, _vp, ctypes.c_int, _vp]
_lib.nvfp4_mx_gemm.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, ctypes.c_int, _vp]
_lib.nvfp4_linear_host.argtypes = [_vp, ctypes.c_int, _i64, _i64, _f32, _vp, _vp, _f32, _i64, _vp, ctypes.c_int, _vp,
                                   _vp, _vp, _vp, _vp]
_lib.nvfp4_quantize.argtypes = [_vp, ctypes.c_int, _i64, _i64, _f32, _vp, _vp, ctypes.c_int, _vp, _vp]
_lib.nvfp4_swizzle_scales.argtypes = [_vp, _i64, _i64, _vp, _vp]
_lib.nvfp4_gemm.argtypes = [_vp, _vp, _f32, _vp, _vp, _f32, _i64, _i64, _i64, _vp, ctypes.c_int, _vp]
_lib.nvfp4_declare_static.argtypes = [_vp, ctypes.c_size_t]
_lib.nvfp4_workspace_bytes.restype = ctypes.c_size_t
_lib.nvfp4_workspace_bytes.argtypes = [_i64, _i64, _i64]
_lib.nvfp4_set_workspace.argtypes = [_vp, _vp, ctypes.c_size_t]
_lib.nvfp4_release_workspaces.argtypes = []
_lib.nvfp4_forget_static.argtypes = []
_lib.nvfp4_forget_static.restype = None
_lib.nvfp4_linear.argtypes = [_vp, ctypes.c_int, _i64, _i64, _f32, _vp, _vp, _f32, _i64, _vp, ctypes.c_int, _vp, _vp,
                              _vp]
_lib.nvfp4_gemm_noalloc.argtypes = [_vp, _vp, _f32, _vp, _vp, _f32, _i64, _i64, _i64, _vp, ctypes.c_int, _vp]
_lib.nvfp4_fused_proj.argtypes = [_vp, _vp, _f32, _vp, _vp, ctypes.POINTER(_i64), ctypes.POINTER(_f32),
                                  ctypes.c_int, _i64, _i64, _vp, ctypes.c_int, _vp]
_lib.nvfp4_convert_e4m3.argtypes = [_vp, _vp, _i64, _vp]
_lib.nvfp4_convert_e2m1.argtypes = [_vp, _vp, _i64, _vp]
_lib.nvfp4_last_device_error.argtypes = []
_lib.nvfp4_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
_lib.nvfp4_set_wait_timeout_ns.restype = None
_lib.nvfp4_set_decode_cooperative.argtypes = [ctypes.c_int]
_lib.nvfp4_bounds_checked.argtypes = []
_lib.nvfp4_bounds_checked.restype = ctypes.c_int
_lib.nvfp4_test_bounds_check.argtypes = [_vp, _i64, _i64, _vp, _vp, _vp]
_lib.nvfp4_set_decode_cooperative.restype = None
_lib.nvfp4_test_wait_timeout.argtypes = [ctypes.c_uint64, _vp]
_lib.nvfp4_test_gemm_stalled_reduction.argtypes = [_vp, _vp, _f32, _vp, _vp, _f32, _i64, _i64, _i64, _vp,
                                                   ctypes.c_int, ctypes.c_int, _vp]
_lib.nvfp4_measure_mma_peak.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_double),
                                        ctypes.POINTER(ctypes.c_double), _vp]
_lib.nvfp4_status_string.restype = ctypes.c_char_p
_lib.nvfp4_status_string.argtypes = [ctypes.c_int]
_lib.nvfp4_version.restype = ctypes.c_int


class Nvfp4Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)} (status {status})")


def lib():
    return _lib


def declared_symbols() -> list[str]:
    """Names of the functions include/nvfp4.h declares."""
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"NVFP4_API\s+[\w\s\*]+?\b(nvfp4_\w+)\s*\(", text)


def status_string(status: int) -> str:
    return _lib.nvfp4_status_string(int(status)).decode()


def version() -> int:
    return int(_lib.nvfp4_version())


def _check(fn, status):
    if status != OK:
        raise Nvfp4Error(fn, status)


def _stream(t: torch.Tensor):
    return _vp(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("device tensor expected")
    if not t.is_contiguous():
        raise ValueError("contiguous tensor expected")
    return _vp(t.data_ptr())


def _hptr(t: torch.Tensor):
    if t.is_cuda:
        raise ValueError("host tensor expected")
    if not t.is_contiguous():
        raise ValueError("contiguous tensor expected")
    return _vp(t.data_ptr())


def _in_dtype(x: torch.Tensor) -> int:
    if x.dtype == torch.bfloat16:
        return IN_BF16
    if x.dtype == torch.float32:
        return IN_F32
    raise ValueError(f"unsupported input dtype {x.dtype}")


def _out_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return OUT_BF16
    if t.dtype == torch.float32:
        return OUT_F32
    raise ValueError(f"unsupported output dtype {t.dtype}")


# ---------------------------------------------------------------- C-ABI calls

def nvfp4_scale_bytes(rows: int, K: int, layout: int = SF_TCGEN05) -> int:
    return int(_lib.nvfp4_scale_bytes(rows, K, layout))


def nvfp4_amax(x: torch.Tensor, amax_out: torch.Tensor) -> None:
    M, K = x.shape
    _check("nvfp4_amax", _lib.nvfp4_amax(_ptr(x), _in_dtype(x), M, K, _ptr(amax_out), _stream(x)))


def nvfp4_amax_accumulate(x: torch.Tensor, running_amax: torch.Tensor) -> None:
    M, K = x.shape
    _check("nvfp4_amax_accumulate",
           _lib.nvfp4_amax_accumulate(_ptr(x), _in_dtype(x), M, K, _ptr(running_amax), _stream(x)))


def nvfp4_quantize(x: torch.Tensor, global_scale: float, codes: torch.Tensor, block_scales: torch.Tensor,
                   layout: int = SF_TCGEN05, amax_out: torch.Tensor | None = None) -> None:
    M, K = x.shape
    _check("nvfp4_quantize", _lib.nvfp4_quantize(_ptr(x), _in_dtype(x), M, K, float(global_scale), _ptr(codes),
                                                 _ptr(block_scales), layout, _ptr(amax_out), _stream(x)))


def nvfp4_swizzle_scales(rowmajor: torch.Tensor, rows: int, K: int, tc: torch.Tensor) -> None:
    _check("nvfp4_swizzle_scales",
           _lib.nvfp4_swizzle_scales(_ptr(rowmajor), rows, K, _ptr(tc), _stream(tc)))


def nvfp4_gemm(a_codes, a_scales, a_global_scale, w_codes, w_scales, w_global_scale, M, N, K,
               out: torch.Tensor) -> None:
    _check("nvfp4_gemm", _lib.nvfp4_gemm(_ptr(a_codes), _ptr(a_scales), float(a_global_scale), _ptr(w_codes),
                                         _ptr(w_scales), float(w_global_scale), M, N, K, _ptr(out),
                                         _out_dtype(out), _stream(out)))


def nvfp4_declare_static(t: torch.Tensor) -> None:
    _check("nvfp4_declare_static", _lib.nvfp4_declare_static(_ptr(t), t.numel() * t.element_size()))


def nvfp4_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_lib.nvfp4_workspace_bytes(M, N, K))


def nvfp4_set_workspace(workspace, stream=None) -> None:
    """Register a zero-filled uint8 device tensor as the K-split workspace of
    `stream` (default: the tensor's current stream); None unregisters."""
    if workspace is None:
        st = torch.cuda.current_stream() if stream is None else stream
        _check("nvfp4_set_workspace", _lib.nvfp4_set_workspace(_vp(st.cuda_stream), None, 0))
        return
    st = torch.cuda.current_stream(workspace.device) if stream is None else stream
    _check("nvfp4_set_workspace",
           _lib.nvfp4_set_workspace(_vp(st.cuda_stream), _ptr(workspace), workspace.numel() * workspace.element_size()))


def nvfp4_release_workspaces() -> None:
    _check("nvfp4_release_workspaces", _lib.nvfp4_release_workspaces())


def nvfp4_forget_static() -> None:
    _lib.nvfp4_forget_static()


def nvfp4_linear(x: torch.Tensor, a_global_scale, w_codes, w_scales, w_global_scale, N, out: torch.Tensor,
                 a_codes=None, a_scales=None) -> None:
    M, K = x.shape
    _check("nvfp4_linear",
           _lib.nvfp4_linear(_ptr(x), _in_dtype(x), M, K, float(a_global_scale), _ptr(w_codes), _ptr(w_scales),
                             float(w_global_scale), N, _ptr(out), _out_dtype(out),
                             _ptr(a_codes) if a_codes is not None else None,
                             _ptr(a_scales) if a_scales is not None else None, _stream(out)))


def nvfp4_linear_host(x_host: torch.Tensor, a_global_scale, w_codes, w_scales, w_global_scale, N,
                      out_host: torch.Tensor, x_dev: torch.Tensor, out_dev: torch.Tensor, a_codes=None,
                      a_scales=None) -> None:
    """x_host / out_host: CPU tensors (page-locked for asynchronous copies);
    x_dev / out_dev: device staging tensors of the same shapes and dtypes."""
    M, K = x_host.shape
    _check("nvfp4_linear_host",
           _lib.nvfp4_linear_host(_hptr(x_host), _in_dtype(x_host), M, K, float(a_global_scale), _ptr(w_codes),
                                  _ptr(w_scales), float(w_global_scale), N, _hptr(out_host), _out_dtype(out_host),
                                  _ptr(x_dev), _ptr(a_codes) if a_codes is not None else None,
                                  _ptr(a_scales) if a_scales is not None else None, _ptr(out_dev),
                                  _stream(out_dev)))


def nvfp4_gemm_noalloc(a_codes, a_scales, a_global_scale, w_codes, w_scales, w_global_scale, M, N, K,
                       out: torch.Tensor) -> None:
    _check("nvfp4_gemm_noalloc",
           _lib.nvfp4_gemm_noalloc(_ptr(a_codes), _ptr(a_scales), float(a_global_scale), _ptr(w_codes),
                                   _ptr(w_scales), float(w_global_scale), M, N, K, _ptr(out), _out_dtype(out),
                                   _stream(out)))


def nvfp4_fused_proj(a_codes, a_scales, a_global_scale, w_codes, w_scales, seg_offsets, seg_global_scales,
                     M, K, out: torch.Tensor) -> None:
    n = len(seg_global_scales)
    offs = (_i64 * (n + 1))(*[int(v) for v in seg_offsets])
    gs = (_f32 * n)(*[float(v) for v in seg_global_scales])
    _check("nvfp4_fused_proj",
           _lib.nvfp4_fused_proj(_ptr(a_codes), _ptr(a_scales), float(a_global_scale), _ptr(w_codes),
                                 _ptr(w_scales), offs, gs, n, M, K, _ptr(out), _out_dtype(out), _stream(out)))


def nvfp4_harmonize_scales(scales: torch.Tensor, N: int, K: int, seg_offsets, seg_global_scales,
                           common_global_scale: float, out: torch.Tensor, layout: int = SF_TCGEN05) -> None:
    n = len(seg_global_scales)
    offs = (_i64 * (n + 1))(*[int(v) for v in seg_offsets])
    gs = (_f32 * n)(*[float(v) for v in seg_global_scales])
    _check("nvfp4_harmonize_scales",
           _lib.nvfp4_harmonize_scales(_ptr(scales), N, K, layout, offs, gs, n, float(common_global_scale),
                                       _ptr(out), _stream(out)))


def nvfp4_mx_quantize(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, layout: int = SF_TCGEN05) -> None:
    M, K = x.shape
    _check("nvfp4_mx_quantize", _lib.nvfp4_mx_quantize(_ptr(x), _in_dtype(x), M, K, _ptr(codes), _ptr(scales),
                                                       layout, _stream(x)))


def alloc_mx_quantized(rows: int, K: int, device, layout: int = SF_TCGEN05):
    """Empty MXFP4 code and scale buffers for a [rows, K] operand."""
    codes = torch.empty(rows, K // 2, dtype=torch.uint8, device=device)
    scales = torch.empty(nvfp4_scale_bytes(rows, K // 2, layout), dtype=torch.uint8, device=device)
    return codes, scales


def nvfp4_mx_gemm(a_codes, a_scales, w_codes, w_scales, M, N, K, out: torch.Tensor) -> None:
    _check("nvfp4_mx_gemm", _lib.nvfp4_mx_gemm(_ptr(a_codes), _ptr(a_scales), _ptr(w_codes), _ptr(w_scales), M, N,
                                               K, _ptr(out), _out_dtype(out), _stream(out)))


def nvfp4_convert_e4m3(x: torch.Tensor, out: torch.Tensor) -> None:
    _check("nvfp4_convert_e4m3", _lib.nvfp4_convert_e4m3(_ptr(x), _ptr(out), x.numel(), _stream(x)))


def nvfp4_convert_e2m1(x: torch.Tensor, out: torch.Tensor) -> None:
    _check("nvfp4_convert_e2m1", _lib.nvfp4_convert_e2m1(_ptr(x), _ptr(out), x.numel(), _stream(x)))


def nvfp4_last_device_error() -> int:
    return int(_lib.nvfp4_last_device_error())


def nvfp4_set_wait_timeout_ns(ns: int) -> None:
    _lib.nvfp4_set_wait_timeout_ns(int(ns))


def nvfp4_bounds_checked() -> bool:
    return bool(_lib.nvfp4_bounds_checked())


def nvfp4_test_bounds_check(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor) -> None:
    M, K = x.shape
    _check("nvfp4_test_bounds_check",
           _lib.nvfp4_test_bounds_check(_ptr(x), M, K, _ptr(codes), _ptr(scales), _stream(x)))


def nvfp4_set_decode_cooperative(enable: bool) -> None:
    _lib.nvfp4_set_decode_cooperative(1 if enable else 0)


def nvfp4_test_wait_timeout(timeout_ns: int, device=None) -> None:
    dev = torch.device("cuda") if device is None else torch.device(device)
    _check("nvfp4_test_wait_timeout",
           _lib.nvfp4_test_wait_timeout(int(timeout_ns), _vp(torch.cuda.current_stream(dev).cuda_stream)))


def nvfp4_test_gemm_stalled_reduction(a_codes, a_scales, a_global_scale, w_codes, w_scales, w_global_scale, M, N,
                                      K, out: torch.Tensor, noalloc: bool = False) -> None:
    _check("nvfp4_test_gemm_stalled_reduction",
           _lib.nvfp4_test_gemm_stalled_reduction(_ptr(a_codes), _ptr(a_scales), float(a_global_scale),
                                                  _ptr(w_codes), _ptr(w_scales), float(w_global_scale), M, N, K,
                                                  _ptr(out), _out_dtype(out), int(bool(noalloc)), _stream(out)))


def nvfp4_measure_mma_peak(iters: int = 5000, device=None):
    """(TFLOP/s, FLOP per clock per SM) of back-to-back dense FP4 MMAs."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    tf, fc = ctypes.c_double(0.0), ctypes.c_double(0.0)
    _check("nvfp4_measure_mma_peak",
           _lib.nvfp4_measure_mma_peak(int(iters), ctypes.byref(tf), ctypes.byref(fc),
                                       _vp(torch.cuda.current_stream(dev).cuda_stream)))
    return tf.value, fc.value


# ---------------------------------------------------------------- buffers

def alloc_quantized(rows: int, K: int, device, layout: int = SF_TCGEN05):
    """Empty (codes, scales) buffers for a [rows, K] NVFP4 operand."""
    codes = torch.empty(rows, K // 2, dtype=torch.uint8, device=device)
    scales = torch.empty(nvfp4_scale_bytes(rows, K, layout), dtype=torch.uint8, device=device)
    return codes, scales
