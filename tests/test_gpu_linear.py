"""nvfp4_linear: quantize the activation and multiply, through the C-ABI.

For decode shapes, without activation buffers, one kernel quantizes X into
shared memory itself; it must give bitwise the same output as
nvfp4_quantize followed by nvfp4_gemm (same per-block arithmetic, same K
split, same summation order), and so the same oracle agreement.  With
activation buffers the call is exactly those two calls."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_10_b200 as nv
import oracle
import synth
from tests.gpu_helpers import DEV, assert_gemm_close, check_device_error_word, oracle_quantize

pytestmark = pytest.mark.gpu


def _weights(N, K, seed):
    w = synth.normal((N, K), seed=seed, std=0.02)
    wc, wsc, gw = oracle_quantize(w.numpy())
    tc = oracle.scales_to_tc(wsc, K)
    return (torch.from_numpy(np.ascontiguousarray(wc)).to(DEV), torch.from_numpy(tc).to(DEV), float(gw),
            (wc, wsc, gw))


def _two_kernels(x, ga, wcd, wsd, gw, N, out_dtype, noalloc=False):
    M, K = x.shape
    ac, asc = nv.alloc_quantized(M, K, DEV)
    nv.nvfp4_quantize(x, ga, ac, asc)
    out = torch.empty(M, N, dtype=out_dtype, device=DEV)
    gemm = nv.nvfp4_gemm_noalloc if noalloc else nv.nvfp4_gemm
    gemm(ac, asc, ga, wcd, wsd, gw, M, N, K, out)
    return out


# (M, N, K): one kernel for all of these (every CTA's share fits in 16 steps)
FUSED = [(1, 640, 256), (8, 12288, 5120), (5, 1000, 320), (16, 2048, 1088), (17, 4096, 5120), (32, 512, 17408),
         (8, 256, 17408), (3, 48, 32)]


@pytest.mark.parametrize("M,N,K", FUSED)
@pytest.mark.parametrize("xdt", [torch.bfloat16, torch.float32])
def test_linear_one_kernel_equals_quantize_then_gemm(M, N, K, xdt):
    x = synth.student_t_outliers(M, K, seed=M * 3 + K, dtype=torch.float32).to(xdt).to(DEV)
    wcd, wsd, gw, _ = _weights(N, K, seed=N + 1)
    ga = 2688.0 / float(x.float().abs().max())
    for out_dtype in (torch.bfloat16, torch.float32):
        ref = _two_kernels(x, ga, wcd, wsd, gw, N, out_dtype)
        out = torch.full((M, N), float("nan"), dtype=out_dtype, device=DEV)
        nv.nvfp4_linear(x, ga, wcd, wsd, gw, N, out)          # no activation buffers: one kernel
        torch.cuda.synchronize()
        assert torch.equal(out, ref), (M, N, K, xdt, out_dtype)
        # and the allocation-free GEMM runs the same K split: bitwise too
        assert torch.equal(out, _two_kernels(x, ga, wcd, wsd, gw, N, out_dtype, noalloc=True))
    check_device_error_word()


@pytest.mark.parametrize("M,N,K", [(8, 12288, 5120), (5, 1000, 320), (24, 768, 1088)])
def test_linear_matches_oracle(M, N, K):
    xf = synth.student_t_outliers(M, K, seed=7 + M, dtype=torch.float32)
    wcd, wsd, gw, (wc, wsc, _) = _weights(N, K, seed=11)
    ac, asc, ga = oracle_quantize(xf.numpy())
    ref = oracle.gemm(ac, asc, ga, wc, wsc, gw)
    out = torch.empty(M, N, dtype=torch.float32, device=DEV)
    nv.nvfp4_linear(xf.to(DEV), float(ga), wcd, wsd, gw, N, out)
    torch.cuda.synchronize()
    assert_gemm_close(out.cpu().numpy(), ref, f"linear {M}x{N}x{K}")
    check_device_error_word()


@pytest.mark.parametrize("M,N,K,one_kernel_ok", [(64, 1024, 512, False), (8, 12288, 17408, False),
                                                (8, 4096, 5120, True)])
def test_linear_with_buffers_is_quantize_then_gemm(M, N, K, one_kernel_ok):
    # with activation buffers the call is quantize + GEMM (the buffers then
    # hold the quantized activation); without them, shapes the one-kernel
    # form does not cover (M > 32, too many K-steps per CTA) are refused
    x = synth.student_t_outliers(M, K, seed=5, dtype=torch.float32).to(torch.bfloat16).to(DEV)
    wcd, wsd, gw, _ = _weights(N, K, seed=3)
    ga = 2688.0 / float(x.float().abs().max())
    out = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    if not one_kernel_ok:
        with pytest.raises(nv.Nvfp4Error):
            nv.nvfp4_linear(x, ga, wcd, wsd, gw, N, out)
    ac, asc = nv.alloc_quantized(M, K, DEV)
    nv.nvfp4_linear(x, ga, wcd, wsd, gw, N, out, ac, asc)
    ac2, asc2 = nv.alloc_quantized(M, K, DEV)
    nv.nvfp4_quantize(x, ga, ac2, asc2)
    ref = _two_kernels(x, ga, wcd, wsd, gw, N, torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert torch.equal(ac, ac2) and torch.equal(asc, asc2)
    check_device_error_word()


def test_linear_chain_reads_the_previous_layers_output():
    # layer 2's X is layer 1's output, written by the kernel just before on
    # the same stream (which lets its successor start early): the one-kernel
    # path must not read X before that kernel completes
    M, K1, N1, N2 = 8, 5120, 4096, 2048
    w1c, w1s, g1, _ = _weights(N1, K1, seed=21)
    w2c, w2s, g2, _ = _weights(N2, N1, seed=22)
    x = synth.student_t_outliers(M, K1, seed=4, dtype=torch.float32).to(torch.bfloat16).to(DEV)
    ga1 = 2688.0 / float(x.float().abs().max())
    h_ref = _two_kernels(x, ga1, w1c, w1s, g1, N1, torch.bfloat16, noalloc=True)
    ga2 = 2688.0 / float(h_ref.float().abs().max())
    y_ref = _two_kernels(h_ref, ga2, w2c, w2s, g2, N2, torch.float32, noalloc=True)
    torch.cuda.synchronize()
    for _ in range(3):
        h = torch.empty(M, N1, dtype=torch.bfloat16, device=DEV)
        y = torch.empty(M, N2, dtype=torch.float32, device=DEV)
        nv.nvfp4_linear(x, ga1, w1c, w1s, g1, N1, h)
        nv.nvfp4_linear(h, ga2, w2c, w2s, g2, N2, y)
        torch.cuda.synchronize()
        assert torch.equal(h, h_ref) and torch.equal(y, y_ref)
    check_device_error_word()


@pytest.mark.parametrize("M,N,K,buffers,pinned", [(8, 12288, 5120, True, True), (8, 12288, 5120, False, True),
                                                  (64, 1024, 2048, True, False), (5, 1000, 320, False, False)])
def test_linear_host_equals_the_device_call(M, N, K, buffers, pinned):
    x = synth.student_t_outliers(M, K, seed=M + N, dtype=torch.bfloat16)
    wcd, wsd, gw, _ = _weights(N, K, seed=K + 1)
    ga = float(oracle.global_scale(oracle.amax(x.float().numpy())))
    x_host = x.pin_memory() if pinned else x.clone()
    out_host = torch.full((M, N), float("nan"), dtype=torch.bfloat16)
    if pinned:
        out_host = out_host.pin_memory()
    x_dev = torch.empty(M, K, dtype=torch.bfloat16, device=DEV)
    out_dev = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    ac, asc = nv.alloc_quantized(M, K, DEV) if buffers else (None, None)
    nv.nvfp4_linear_host(x_host, ga, wcd, wsd, gw, N, out_host, x_dev, out_dev, ac, asc)
    torch.cuda.synchronize()
    check_device_error_word()
    # the same layer called on device buffers: with activation buffers it is
    # quantize + GEMM, without them the one-kernel form
    want = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    xd = x.to(DEV)
    if buffers:
        ac2, asc2 = nv.alloc_quantized(M, K, DEV)
        nv.nvfp4_linear(xd, ga, wcd, wsd, gw, N, want, ac2, asc2)
    else:
        nv.nvfp4_linear(xd, ga, wcd, wsd, gw, N, want)
    torch.cuda.synchronize()
    assert torch.equal(out_host, want.cpu())
