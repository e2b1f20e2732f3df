"""GPU quantizer parity: codes and block scales bit-exact against the oracle
(through the C-ABI), in both scale layouts, bf16 and f32 inputs, ragged and
degenerate shapes, and at the benchmark's full sizes on sampled rows."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_10_b200 as nv
import oracle
import synth
from tests.gpu_helpers import DEV, check_device_error_word, gpu_quantize, oracle_quantize

pytestmark = pytest.mark.gpu

SHAPES = [(1, 32), (3, 96), (17, 160), (130, 320), (256, 5120), (300, 1088), (129, 17408)]


def _inputs(M, K, kind, seed):
    if kind == "student_t":
        return synth.student_t_outliers(M, K, seed=seed, dtype=torch.float32)
    if kind == "outliers":
        return synth.normal_with_outlier_channels(M, K, seed=seed, dtype=torch.float32)
    return synth.normal((M, K), seed=seed)


def _compare(x_cpu_f32: torch.Tensor, x_dev: torch.Tensor, g, layout):
    M, K = x_cpu_f32.shape
    c_ref, s_ref, _ = oracle_quantize(x_cpu_f32.numpy(), g)
    codes, scales, am = gpu_quantize(x_dev, g, layout, amax=True)
    torch.cuda.synchronize()
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    if layout == nv.SF_TCGEN05:
        assert np.array_equal(scales.cpu().numpy(), oracle.scales_to_tc(s_ref, K))
    else:
        assert np.array_equal(scales.cpu().numpy().reshape(M, K // 16), s_ref)
    assert am.item() == oracle.amax(x_cpu_f32.numpy())


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("layout", [nv.SF_TCGEN05, nv.SF_ROWMAJOR])
def test_quantize_bit_exact(M, K, dtype, layout):
    x = _inputs(M, K, "student_t", seed=M * 7 + K).to(dtype)
    xf = x.float()
    g = oracle.global_scale(oracle.amax(xf.numpy()))
    _compare(xf, x.to(DEV), g, layout)
    check_device_error_word()


@pytest.mark.parametrize("kind", ["normal", "outliers"])
def test_quantize_other_distributions(kind):
    x = _inputs(64, 2048, kind, seed=5).to(torch.bfloat16)
    xf = x.float()
    g = oracle.global_scale(oracle.amax(xf.numpy()))
    _compare(xf, x.to(DEV), g, nv.SF_TCGEN05)


def test_quantize_special_values():
    # zeros, negative zeros, underflowing blocks, saturating blocks (static g
    # calibrated on a smaller tensor), exact E2M1 midpoints
    K = 256
    x = np.zeros((6, K), np.float32)
    x[1, :] = -0.0
    x[2, :16] = 1e-7
    x[2, 16:32] = -1e-7
    x[3, :] = np.tile(np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], np.float32), K // 8)
    x[4, :] = np.linspace(-1000, 1000, K, dtype=np.float32)
    x[5, ::3] = -3.0
    xt = torch.from_numpy(x)
    for g in (np.float32(1.0), np.float32(6.0), np.float32(2688.0 / 1000.0), np.float32(0.37)):
        _compare(xt, xt.to(DEV), g, nv.SF_TCGEN05)
        _compare(xt, xt.to(DEV), g, nv.SF_ROWMAJOR)


def test_quantize_tc_padding_is_zero():
    # rows 3..127 and the K % 64 == 32 tail of each 128-row chunk are padding
    M, K = 3, 96
    x = torch.randn(M, K, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    codes, scales = nv.alloc_quantized(M, K, DEV)
    scales.fill_(0xAB)
    g = oracle.global_scale(oracle.amax(x.float().numpy()))
    nv.nvfp4_quantize(x.to(DEV), float(g), codes, scales)
    tc = scales.cpu().numpy()
    _, s_ref, _ = oracle_quantize(x.float().numpy(), g)
    assert np.array_equal(tc, oracle.scales_to_tc(s_ref, K))


@pytest.mark.parametrize("M,K", [(1, 5120), (64, 17408), (4096, 5120), (32768, 5120), (32768, 17408)])
def test_quantize_sweep_full_size_sampled_rows(M, K):
    # the quantize-sweep workload: full tensor on the GPU, sampled rows on the oracle
    x = synth.quant_sweep_activation(M, K, device=DEV)
    rows = synth.sample_rows(M, 64)
    xs = x[rows].float().cpu()
    amax_dev = torch.empty(1, dtype=torch.float32, device=DEV)
    nv.nvfp4_amax(x, amax_dev)
    full_amax = oracle.amax(x.cpu().float().numpy())
    assert amax_dev.item() == full_amax
    g = np.float32(2688.0) / np.float32(full_amax)
    codes, scales, am = gpu_quantize(x, g, nv.SF_TCGEN05, amax=True)
    assert am.item() == full_amax
    c_ref, s_ref, _ = oracle_quantize(xs.numpy(), g)
    assert np.array_equal(codes[rows].cpu().numpy(), c_ref)
    tc = scales.cpu().numpy()
    got = oracle.scales_from_tc(tc, M, K)[rows]
    assert np.array_equal(got, s_ref)
    check_device_error_word()


@pytest.mark.parametrize("M,K", [(1, 32), (5, 64), (300, 1088), (4096, 5120)])
def test_amax_matches_oracle(M, K):
    x = synth.student_t_outliers(M, K, seed=3, dtype=torch.float32)
    out = torch.empty(1, dtype=torch.float32, device=DEV)
    for dt in (torch.bfloat16, torch.float32):
        xd = x.to(dt)
        nv.nvfp4_amax(xd.to(DEV), out)
        assert out.item() == oracle.amax(xd.float().numpy())


@pytest.mark.parametrize("R,K", [(1, 32), (17, 96), (300, 1088), (12288, 5120)])
def test_swizzle_scales_matches_layout(R, K):
    rng = np.random.default_rng(R + K)
    rm = rng.integers(0, 0x7F, size=(R, K // 16), dtype=np.uint8)
    tc = torch.empty(nv.nvfp4_scale_bytes(R, K), dtype=torch.uint8, device=DEV)
    tc.fill_(0xCD)
    nv.nvfp4_swizzle_scales(torch.from_numpy(rm).to(DEV), R, K, tc)
    assert np.array_equal(tc.cpu().numpy(), oracle.scales_to_tc(rm, K))


def test_quantize_deterministic():
    x = synth.student_t_outliers(512, 5120, seed=9, dtype=torch.bfloat16, device=DEV)
    g = 2688.0 / torch.abs(x.float()).max().item()
    a = gpu_quantize(x, g)
    b = gpu_quantize(x, g)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
