"""MXFP4, the contrast format, on the GPU against the oracle.

32-element blocks with a power-of-two E8M0 scale (OCP Microscaling v1.0
conversion) against NVFP4's 16-element E4M3 blocks [anthology record
LIT-800, "Standing in the anthology"].  Checks: the quantizer's codes and
scales bitwise (both layouts, ragged K, special values), the kind::mxf4
GEMM against the oracle's FP64 GEMM on the normal and split-K paths and
ragged K, BF16 output as the rounding of the FP32 output, and the pages'
claim measured on the GPU: on outlier activations NVFP4's GEMM error is
below MXFP4's."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_10_b200 as nv
import oracle
import synth
from tests.gpu_helpers import DEV, assert_gemm_close, check_device_error_word, gpu_quantize, oracle_quantize

pytestmark = pytest.mark.gpu


def _gpu_mx(x: torch.Tensor, layout=nv.SF_TCGEN05):
    M, K = x.shape
    codes, scales = nv.alloc_mx_quantized(M, K, x.device, layout)
    scales.fill_(0xA5)
    nv.nvfp4_mx_quantize(x, codes, scales, layout)
    return codes, scales


def _special(M, K, seed):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(M, K // 32, 32, generator=g) * torch.exp2(torch.randint(-40, 40, (M, K // 32, 1),
                                                                             generator=g).float())).reshape(M, K)
    x[0, :32] = 0.0
    x[0, 32:64] = -0.0
    if K >= 128:
        x[0, 64:96] = 1e-40                       # subnormal block maximum
        x[0, 96] = 6.0
        x[0, 97] = -7.0                           # clips at 6
    return x


@pytest.mark.parametrize("layout", [nv.SF_ROWMAJOR, nv.SF_TCGEN05])
@pytest.mark.parametrize("M,K,kind", [
    (16, 256, "tiny"), (8, 5120, "decode"), (130, 160, "special"), (3, 96, "special"), (4096, 5120, "prefill"),
])
def test_mx_quantize_bitwise(layout, M, K, kind):
    if kind == "tiny":
        x = synth.activation(synth.TINY, M=M, K=K)
    elif kind == "decode":
        x = synth.activation(synth.DECODE, M=M, K=K)
    elif kind == "prefill":
        x = synth.activation(synth.PREFILL, M=M, K=K)
    else:
        x = _special(M, K, seed=M + K)
    codes, scales = _gpu_mx(x.to(DEV), layout)
    torch.cuda.synchronize()
    check_device_error_word()
    c, s = oracle.mx_quantize(x.float().numpy())
    assert np.array_equal(codes.cpu().numpy(), c)
    want = s if layout == nv.SF_ROWMAJOR else oracle.mx_scales_to_tc(s, K)
    assert np.array_equal(scales.cpu().numpy().reshape(-1), want.reshape(-1))


def _mx_case(M, N, K, seed):
    a = synth.student_t_outliers(M, K, seed=seed, dtype=torch.float32).numpy()
    w = synth.normal((N, K), seed=seed + 1, std=0.02).numpy()
    ac, asc = oracle.mx_quantize(a)
    wc, wsc = oracle.mx_quantize(w)
    dev = lambda c, s: (torch.from_numpy(c).to(DEV), torch.from_numpy(oracle.mx_scales_to_tc(s, K)).to(DEV))  # noqa: E731
    return (ac, asc, wc, wsc), dev(ac, asc), dev(wc, wsc)


@pytest.mark.parametrize("M,N,K", [
    (1, 384, 5120), (8, 1024, 2048), (16, 256, 160), (33, 512, 192), (100, 640, 1024),   # split-K (M <= 128)
    (129, 512, 1024), (256, 512, 160), (512, 768, 5120),                                 # normal tiles
])
def test_mx_gemm_matches_oracle(M, N, K):
    (ac, asc, wc, wsc), (a_d, as_d), (w_d, ws_d) = _mx_case(M, N, K, seed=M * 7 + K)
    out = torch.empty(M, N, dtype=torch.float32, device=DEV)
    nv.nvfp4_mx_gemm(a_d, as_d, w_d, ws_d, M, N, K, out)
    out16 = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    nv.nvfp4_mx_gemm(a_d, as_d, w_d, ws_d, M, N, K, out16)
    torch.cuda.synchronize()
    check_device_error_word()
    assert_gemm_close(out.cpu().numpy(), oracle.mx_gemm(ac, asc, wc, wsc), f"mx {M}x{N}x{K}")
    assert torch.equal(out16, out.to(torch.bfloat16))


def test_mx_gemm_from_the_gpu_quantizer_decode_size():
    wl = synth.DECODE
    x = synth.activation(wl).to(DEV)
    w = synth.weight(wl).to(DEV)
    a_c, a_s = _gpu_mx(x)
    w_c, w_s = _gpu_mx(w)
    out = torch.empty(wl.M, wl.N, dtype=torch.float32, device=DEV)
    nv.nvfp4_mx_gemm(a_c, a_s, w_c, w_s, wl.M, wl.N, wl.K, out)
    torch.cuda.synchronize()
    check_device_error_word()
    ac, asc = oracle.mx_quantize(x.float().cpu().numpy())
    cols = synth.sample_rows(wl.N, 1024)
    wc, wsc = oracle.mx_quantize(w.float().cpu().numpy()[cols])
    assert_gemm_close(out.cpu().numpy()[:, cols], oracle.mx_gemm(ac, asc, wc, wsc), "mx decode")


def test_nvfp4_error_below_mxfp4_on_outlier_activations():
    wl = synth.PREFILL
    M, N, K = 512, 1024, wl.K
    x = synth.activation(wl, M=M).to(DEV)
    w = synth.weight(wl, N=N).to(DEV)
    ref = x.double() @ w.double().T
    ga = oracle.global_scale(oracle.amax(x.float().cpu().numpy()))
    gw = oracle.global_scale(oracle.amax(w.float().cpu().numpy()))
    a_c, a_s, _ = gpu_quantize(x, ga)
    w_c, w_s, _ = gpu_quantize(w, gw)
    o_nv = torch.empty(M, N, dtype=torch.float32, device=DEV)
    nv.nvfp4_gemm(a_c, a_s, float(ga), w_c, w_s, float(gw), M, N, K, o_nv)
    ma, mas = _gpu_mx(x)
    mw, mws = _gpu_mx(w)
    o_mx = torch.empty_like(o_nv)
    nv.nvfp4_mx_gemm(ma, mas, mw, mws, M, N, K, o_mx)
    torch.cuda.synchronize()
    check_device_error_word()
    e_nv = float((o_nv.double() - ref).norm() / ref.norm())
    e_mx = float((o_mx.double() - ref).norm() / ref.norm())
    assert e_nv < 0.85 * e_mx, (e_nv, e_mx)


def test_mx_prefill_full_size_sampled_rows():
    # the full MXFP4 prefill launch the benchmark times (32768 x 17408 x 5120)
    # in FP32 output mode, compared with the oracle at the stated tolerance on
    # 24 evenly spread rows; the BF16 launch is bitwise its BF16 rounding
    w = synth.PREFILL
    x = synth.activation(w, device=DEV)
    wt = synth.weight(w, device=DEV)
    a_c, a_s = _gpu_mx(x)
    w_c, w_s = _gpu_mx(wt)
    out32 = torch.empty(w.M, w.N, dtype=torch.float32, device=DEV)
    nv.nvfp4_mx_gemm(a_c, a_s, w_c, w_s, w.M, w.N, w.K, out32)
    out16 = torch.empty(w.M, w.N, dtype=torch.bfloat16, device=DEV)
    nv.nvfp4_mx_gemm(a_c, a_s, w_c, w_s, w.M, w.N, w.K, out16)
    torch.cuda.synchronize()
    check_device_error_word()
    assert torch.equal(out16, out32.to(torch.bfloat16))
    del out16
    rows = synth.sample_rows(w.M, 24)
    ac, asc = oracle.mx_quantize(x[rows].float().cpu().numpy())
    wc, wsc = oracle.mx_quantize(wt.float().cpu().numpy())
    ref = oracle.mx_gemm(ac, asc, wc, wsc)
    assert_gemm_close(out32[rows].cpu().numpy(), ref, "mx prefill rows")
