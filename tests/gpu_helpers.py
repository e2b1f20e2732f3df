"""Shared plumbing for the GPU parity tests: build operands with the oracle
on the CPU, move bytes to the device, run the library through its C-ABI
binding, and compare.  Expected values always come from ``oracle``; the CUDA
path only ever receives inputs."""
import numpy as np
import torch

import nvfp4_w4a4_quantized_10_b200 as nv
import oracle

DEV = "cuda"

# GEMM tolerances for the FP32 output mode against the FP64 oracle: normwise
# max relative error and relative Frobenius error (the BF16 output adds its
# own 2^-9 rounding, so it is checked as bf16(f32 output) instead).
TOL_MAX_REL = 1e-3
TOL_FROB = 1e-5


def oracle_quantize(x_f32: np.ndarray, g=None):
    """Oracle quantization: (codes, row-major scales, g)."""
    if g is None:
        g = oracle.global_scale(oracle.amax(x_f32))
    c, s = oracle.quantize(x_f32, g)
    return c, s, np.float32(g)


def to_dev_operand(codes: np.ndarray, scales_rm: np.ndarray, K: int):
    """Upload oracle codes and its scales re-laid out (by the oracle's layout
    function) in the tensor-core order."""
    tc = oracle.scales_to_tc(scales_rm, K)
    return (torch.from_numpy(np.ascontiguousarray(codes)).to(DEV),
            torch.from_numpy(tc).to(DEV))


def gpu_quantize(x: torch.Tensor, g, layout=nv.SF_TCGEN05, amax=False):
    M, K = x.shape
    codes, scales = nv.alloc_quantized(M, K, x.device, layout)
    am = torch.empty(1, dtype=torch.float32, device=x.device) if amax else None
    nv.nvfp4_quantize(x, float(g), codes, scales, layout, am)
    return codes, scales, am


def gpu_gemm(a_codes, a_sc, ga, w_codes, w_sc, gw, M, N, K, out_dtype=torch.float32):
    out = torch.empty(M, N, dtype=out_dtype, device=DEV)
    nv.nvfp4_gemm(a_codes, a_sc, float(ga), w_codes, w_sc, float(gw), M, N, K, out)
    return out


def rel_errors(out: np.ndarray, ref: np.ndarray):
    out = out.astype(np.float64)
    diff = out - ref
    denom_max = np.max(np.abs(ref))
    max_rel = np.max(np.abs(diff)) / denom_max if denom_max > 0 else np.max(np.abs(diff))
    nref = np.linalg.norm(ref)
    frob = np.linalg.norm(diff) / nref if nref > 0 else np.linalg.norm(diff)
    return float(max_rel), float(frob)


def assert_gemm_close(out: np.ndarray, ref: np.ndarray, what=""):
    max_rel, frob = rel_errors(out, ref)
    assert max_rel <= TOL_MAX_REL and frob <= TOL_FROB, f"{what}: max_rel={max_rel:.3g} frob={frob:.3g}"
    return max_rel, frob


def bf16_rne(t: torch.Tensor) -> torch.Tensor:
    return t.to(torch.bfloat16)


def check_device_error_word():
    st = nv.nvfp4_last_device_error()
    assert st == nv.OK, nv.status_string(st)
