"""GPU GEMM parity through the C-ABI against the FP64 oracle.

FP32 output mode: normwise max relative error <= 1e-3 and relative Frobenius
error <= 1e-5.  BF16 output mode: bitwise equal to the round-to-nearest-even
BF16 of the FP32 output of the same deterministic kernel (so it is within one
BF16 rounding of a result that meets the FP32 tolerance)."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_10_b200 as nv
import oracle
import synth
from tests.gpu_helpers import (DEV, assert_gemm_close, check_device_error_word, gpu_gemm, gpu_quantize,
                               oracle_quantize, to_dev_operand)

pytestmark = pytest.mark.gpu

# (M, N, K): tiny config, swap (M <= 128) and normal tiles, ragged M/N/K
# tails (K % 64 == 32, K % 256 != 0, N % 8 != 0), several tiles each way
SHAPES = [(16, 256, 256), (1, 48, 32), (3, 200, 96), (8, 512, 1088), (17, 300, 160), (64, 384, 512),
          (100, 256, 256), (128, 640, 512), (129, 520, 320), (200, 264, 1088), (257, 513, 544),
          (300, 1000, 2048), (512, 768, 5120), (40, 136, 17408)]


def _operands(M, N, K, seed):
    a = synth.student_t_outliers(M, K, seed=seed, dtype=torch.float32).numpy()
    w = synth.normal((N, K), seed=seed + 1, std=0.02).numpy()
    ac, asc, ga = oracle_quantize(a)
    wc, wsc, gw = oracle_quantize(w)
    return (ac, asc, ga), (wc, wsc, gw)


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_matches_oracle(M, N, K):
    (ac, asc, ga), (wc, wsc, gw) = _operands(M, N, K, seed=M + N + K)
    ref = oracle.gemm(ac, asc, ga, wc, wsc, gw)
    a_d, as_d = to_dev_operand(ac, asc, K)
    w_d, ws_d = to_dev_operand(wc, wsc, K)
    out32 = gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, M, N, K, torch.float32)
    out16 = gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, M, N, K, torch.bfloat16)
    torch.cuda.synchronize()
    assert_gemm_close(out32.cpu().numpy(), ref, f"{M}x{N}x{K}")
    assert torch.equal(out16, out32.to(torch.bfloat16))
    check_device_error_word()


def test_tiny_end_to_end_quantize_then_gemm():
    # the tiny workload: fp32 X[16,256], W[256,256]; GPU quantize -> GPU GEMM
    w = synth.TINY
    x = synth.activation(w)
    wt = synth.weight(w)
    ga = oracle.global_scale(oracle.amax(x.numpy()))
    gw = oracle.global_scale(oracle.amax(wt.numpy()))
    ac, asc, _ = oracle_quantize(x.numpy(), ga)
    wc, wsc, _ = oracle_quantize(wt.numpy(), gw)
    ref = oracle.gemm(ac, asc, ga, wc, wsc, gw)
    a_codes, a_sc, _ = gpu_quantize(x.to(DEV), ga)
    w_codes, w_sc, _ = gpu_quantize(wt.to(DEV), gw)
    out = gpu_gemm(a_codes, a_sc, ga, w_codes, w_sc, gw, w.M, w.N, w.K)
    assert_gemm_close(out.cpu().numpy(), ref, "tiny")


def test_one_hot_weight_closed_form():
    M, N, K = 37, 64, 512
    a = synth.student_t_outliers(M, K, seed=4, dtype=torch.float32).numpy()
    ac, asc, ga = oracle_quantize(a)
    cols = np.random.default_rng(0).integers(0, K, size=N)
    nib = np.zeros((N, K), np.uint8)
    nib[np.arange(N), cols] = 0x2                  # 1.0
    wc = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    wsc = np.full((N, K // 16), 0x38, np.uint8)     # scale 1.0
    expect = oracle.dequantize(ac, asc, ga)[:, cols]
    a_d, as_d = to_dev_operand(ac, asc, K)
    w_d, ws_d = to_dev_operand(wc, wsc, K)
    out = gpu_gemm(a_d, as_d, ga, w_d, ws_d, 1.0, M, N, K).cpu().numpy()
    assert np.allclose(out, expect, rtol=2.5e-7, atol=0)


def test_all_six_closed_form_nibble_and_scale_placement():
    # every code 6, per-block scales 2^j: any misplaced nibble or scale changes
    # the result by an exact power-of-two factor
    M, N, K = 130, 260, 320
    rng = np.random.default_rng(1)
    sa = (0x38 + 8 * rng.integers(-3, 4, size=(M, K // 16))).astype(np.uint8)
    sw = (0x38 + 8 * rng.integers(-3, 4, size=(N, K // 16))).astype(np.uint8)
    ac = np.full((M, K // 2), 0x77, np.uint8)
    row_sign = np.where(rng.random(N) < 0.5, 0x77, 0xFF).astype(np.uint8)   # all +6 or all -6
    wc = np.repeat(row_sign[:, None], K // 2, axis=1)
    ref = oracle.gemm(ac, sa, 1.0, wc, sw, 1.0)
    a_d, as_d = to_dev_operand(ac, sa, K)
    w_d, ws_d = to_dev_operand(wc, sw, K)
    out = gpu_gemm(a_d, as_d, 1.0, w_d, ws_d, 1.0, M, N, K).cpu().numpy()
    assert np.array_equal(out, ref.astype(np.float32))


def test_decode_full_size_all_rows():
    w = synth.DECODE
    x = synth.activation(w).float().numpy()
    wt = synth.weight(w).float().numpy()
    (ac, asc, ga) = oracle_quantize(x)
    (wc, wsc, gw) = oracle_quantize(wt)
    ref = oracle.gemm(ac, asc, ga, wc, wsc, gw)
    a_d, as_d = to_dev_operand(ac, asc, w.K)
    w_d, ws_d = to_dev_operand(wc, wsc, w.K)
    out = gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, w.M, w.N, w.K)
    assert_gemm_close(out.cpu().numpy(), ref, "decode")
    out16 = gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, w.M, w.N, w.K, torch.bfloat16)
    assert torch.equal(out16, out.to(torch.bfloat16))


def test_prefill_full_size_sampled_rows():
    # the full prefill launch the benchmark times (32768 x 17408 x 5120, all
    # 17,408 tiles on the persistent grid), run in FP32 output mode and
    # compared with the oracle at the stated tolerance on 24 evenly spread
    # rows; the BF16 launch is bitwise the BF16 rounding of the FP32 one
    w = synth.PREFILL
    x = synth.activation(w, device=DEV)
    wt = synth.weight(w, device=DEV)
    ga = oracle.global_scale(oracle.amax(x.float().cpu().numpy()))
    wt_cpu = wt.float().cpu().numpy()
    gw = oracle.global_scale(oracle.amax(wt_cpu))
    a_codes, a_sc, _ = gpu_quantize(x, ga)
    w_codes, w_sc, _ = gpu_quantize(wt, gw)
    out32 = gpu_gemm(a_codes, a_sc, ga, w_codes, w_sc, gw, w.M, w.N, w.K, torch.float32)
    out16 = gpu_gemm(a_codes, a_sc, ga, w_codes, w_sc, gw, w.M, w.N, w.K, torch.bfloat16)
    torch.cuda.synchronize()
    check_device_error_word()
    assert torch.equal(out16, out32.to(torch.bfloat16))
    del out16
    rows = synth.sample_rows(w.M, 24)
    ac, asc, _ = oracle_quantize(x[rows].float().cpu().numpy(), ga)
    wc, wsc, _ = oracle_quantize(wt_cpu, gw)
    ref = oracle.gemm(ac, asc, ga, wc, wsc, gw)
    assert_gemm_close(out32[rows].cpu().numpy(), ref, "prefill rows")


def test_gemm_deterministic():
    M, N, K = 1024, 2048, 5120
    x = synth.student_t_outliers(M, K, seed=2, dtype=torch.bfloat16, device=DEV)
    wt = synth.normal((N, K), seed=3, std=0.02, dtype=torch.bfloat16, device=DEV)
    a = gpu_quantize(x, 10.0)
    b = gpu_quantize(wt, 20000.0)
    o1 = gpu_gemm(a[0], a[1], 10.0, b[0], b[1], 20000.0, M, N, K, torch.bfloat16)
    o2 = gpu_gemm(a[0], a[1], 10.0, b[0], b[1], 20000.0, M, N, K, torch.bfloat16)
    assert torch.equal(o1, o2)


def test_output_guard_bands_untouched():
    # the epilogue writes exactly [M, N]: sentinels around the output survive
    M, N, K = 130, 264, 320
    (ac, asc, ga), (wc, wsc, gw) = _operands(M, N, K, seed=11)
    a_d, as_d = to_dev_operand(ac, asc, K)
    w_d, ws_d = to_dev_operand(wc, wsc, K)
    pad = 4096
    buf = torch.full((pad + M * N + pad,), -7.0, dtype=torch.float32, device=DEV)
    out = buf[pad:pad + M * N].view(M, N)
    nv.nvfp4_gemm(a_d, as_d, float(ga), w_d, ws_d, float(gw), M, N, K, out)
    torch.cuda.synchronize()
    assert torch.all(buf[:pad] == -7.0) and torch.all(buf[pad + M * N:] == -7.0)


@pytest.mark.parametrize("M,N,K", [(200, 128, 512), (300, 48, 256), (260, 320, 512), (131, 72, 320)])
def test_gemm_partial_last_tile_bf16(M, N, K):
    # normal tiles whose last 64-column output sub-tiles fall past N: the
    # bf16 result must still be bf16(f32 result) everywhere
    (ac, asc, ga), (wc, wsc, gw) = _operands(M, N, K, seed=M * N + K)
    ref = oracle.gemm(ac, asc, ga, wc, wsc, gw)
    a_d, as_d = to_dev_operand(ac, asc, K)
    w_d, ws_d = to_dev_operand(wc, wsc, K)
    for _ in range(3):
        out32 = gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, M, N, K, torch.float32)
        out16 = gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, M, N, K, torch.bfloat16)
        assert torch.equal(out16, out32.to(torch.bfloat16))
    assert_gemm_close(out32.cpu().numpy(), ref, f"{M}x{N}x{K}")


def test_split_k_decode_deterministic_and_stream_local():
    # decode shapes split K over the CTAs; partials are summed in a fixed
    # order, so repeated runs match bitwise, also on two streams at once
    M, N, K = 8, 4096, 5120
    (ac, asc, ga), (wc, wsc, gw) = _operands(M, N, K, seed=21)
    a_d, as_d = to_dev_operand(ac, asc, K)
    w_d, ws_d = to_dev_operand(wc, wsc, K)
    ref = gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, M, N, K, torch.bfloat16)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    for s in (s1, s2):
        with torch.cuda.stream(s):   # first call on each stream (sets up its workspace)
            outs.append(gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, M, N, K, torch.bfloat16))
    torch.cuda.synchronize()
    for _ in range(5):
        o = []
        for s in (s1, s2):
            with torch.cuda.stream(s):
                o.append(gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, M, N, K, torch.bfloat16))
        torch.cuda.synchronize()
        for t in o:
            assert torch.equal(t, ref)
    assert all(torch.equal(t, ref) for t in outs)
    check_device_error_word()


@pytest.mark.parametrize("M,N,K", [(32, 4096, 17408), (8, 12288, 5120), (512, 2048, 5120)])
def test_gemm_right_after_the_kernel_that_writes_its_operands(M, N, K):
    # the weight and the activation are quantized on the GPU by the kernels
    # just before the GEMM on the same stream, with no synchronization: the
    # GEMM may start early (programmatic dependent launch) but must not read
    # either operand before those kernels have finished
    a = synth.student_t_outliers(M, K, seed=M + 1, dtype=torch.float32)
    w = synth.normal((N, K), seed=N + 2, std=0.02)
    ac, asc, ga = oracle_quantize(a.numpy())
    wc, wsc, gw = oracle_quantize(w.numpy())
    ref = oracle.gemm(ac, asc, ga, wc, wsc, gw)
    a_d = a.to(DEV)
    w_d = w.to(DEV)
    torch.cuda.synchronize()
    for _ in range(2):
        wcd, wsd, _ = gpu_quantize(w_d, gw)
        acd, asd, _ = gpu_quantize(a_d, ga)
        out = torch.empty(M, N, dtype=torch.float32, device=DEV)
        nv.nvfp4_gemm(acd, asd, float(ga), wcd, wsd, float(gw), M, N, K, out)
        torch.cuda.synchronize()
        assert_gemm_close(out.cpu().numpy(), ref, f"{M}x{N}x{K}")
        del wcd, wsd, acd, asd
    check_device_error_word()


@pytest.mark.parametrize("M,N,K", [(8, 12288, 5120), (512, 2048, 5120), (3, 200, 96)])
def test_static_weights_give_the_same_result(M, N, K):
    # weights declared read-only are loaded before the preceding kernel ends;
    # the arithmetic is unchanged, so results are bitwise those of the
    # default path, also when the GEMMs follow each other and the quantizer
    # back to back
    (ac, asc, ga), (wc, wsc, gw) = _operands(M, N, K, seed=77)
    a_d, as_d = to_dev_operand(ac, asc, K)
    w_d, ws_d = to_dev_operand(wc, wsc, K)
    x = synth.student_t_outliers(M, K, seed=78, dtype=torch.float32).to(DEV)
    ref = gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, M, N, K, torch.float32)
    nv.nvfp4_declare_static(w_d)
    nv.nvfp4_declare_static(ws_d)
    try:
        outs = []
        for _ in range(3):
            qa, qs, _ = gpu_quantize(x, ga)              # a kernel just before, as in a decode step
            outs.append(gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, M, N, K, torch.float32))
        torch.cuda.synchronize()
    finally:
        nv.nvfp4_forget_static()
    assert all(torch.equal(o, ref) for o in outs)
    check_device_error_word()
