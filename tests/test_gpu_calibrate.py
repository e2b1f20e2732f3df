"""Static calibration on the GPU, against the oracle.

The activation scale is fixed from calibration batches (running amax over the
batches) and then quantizes a held-out batch whose outliers are larger, so
some of its block scales saturate at 448 and their largest codes clip at 6
[anthology record LIT-800, "Key takeaways": calibration-only recipe;
cctest.ai article, "Introduction"].  Checks: the running amax is bitwise the
oracle's, in any batch order; the held-out batch's codes and scales under
the static scale are bitwise the oracle's; the GEMM on them matches."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_10_b200 as nv
import oracle
import synth
from tests.gpu_helpers import (DEV, assert_gemm_close, check_device_error_word, gpu_quantize, oracle_quantize,
                               to_dev_operand)

pytestmark = pytest.mark.gpu


def _running_amax(batches):
    r = torch.zeros(1, dtype=torch.float32, device=DEV)
    for b in batches:
        nv.nvfp4_amax_accumulate(b, r)
    torch.cuda.synchronize()
    check_device_error_word()
    return np.float32(r.item())


@pytest.mark.parametrize("M,K", [(1024, 5120), (synth.CALIB_M, synth.CALIB_K)])
def test_running_amax_over_batches_bitwise(M, K):
    cal = [synth.calibration_batch(i, M, K, device=DEV) for i in range(synth.CALIB_BATCHES)]
    want = oracle.calibrate_amax([b.float().cpu().numpy() for b in cal])
    assert _running_amax(cal) == want
    assert _running_amax(cal[::-1]) == want
    held = synth.held_out_batch(M, K, device=DEV)
    assert _running_amax(cal + [held]) == oracle.calibrate_amax(
        [b.float().cpu().numpy() for b in cal] + [held.float().cpu().numpy()])


def test_running_amax_f32_and_starting_value():
    x = synth.normal((16, 256), seed=3, device=DEV)
    r = torch.full((1,), 100.0, dtype=torch.float32, device=DEV)
    nv.nvfp4_amax_accumulate(x, r)                      # a larger running value is kept
    torch.cuda.synchronize()
    assert r.item() == 100.0
    r.zero_()
    nv.nvfp4_amax_accumulate(x, r)
    torch.cuda.synchronize()
    assert np.float32(r.item()) == oracle.amax(x.cpu().numpy())


@pytest.mark.parametrize("layout", [nv.SF_ROWMAJOR, nv.SF_TCGEN05])
def test_held_out_batch_under_the_static_scale_bitwise(layout):
    M, K = synth.CALIB_M, synth.CALIB_K
    cal = [synth.calibration_batch(i, M, K, device=DEV) for i in range(synth.CALIB_BATCHES)]
    g = oracle.global_scale(_running_amax(cal))
    held = synth.held_out_batch(M, K, device=DEV)
    h = held.float().cpu().numpy()
    assert oracle.saturation(h, g)[0] > 0                # some block scales clip
    codes, scales, _ = gpu_quantize(held, g, layout)
    torch.cuda.synchronize()
    check_device_error_word()
    c, s = oracle.quantize(h, g)
    assert np.array_equal(codes.cpu().numpy(), c)
    want = s if layout == nv.SF_ROWMAJOR else oracle.scales_to_tc(s, K)
    assert np.array_equal(scales.cpu().numpy().reshape(-1), want.reshape(-1))


def test_gemm_on_the_clipped_activation():
    M, K, N = 1024, 5120, 384
    cal = [synth.calibration_batch(i, M, K) for i in range(synth.CALIB_BATCHES)]
    g = oracle.global_scale(oracle.calibrate_amax([b.float().numpy() for b in cal]))
    held = synth.held_out_batch(M, K)
    ac, asc = oracle.quantize(held.float().numpy(), g)
    w = synth.normal((N, K), seed=44, std=0.02).numpy()
    wc, wsc, gw = oracle_quantize(w)
    a_codes, a_sc, _ = gpu_quantize(held.to(DEV), g)
    w_d, ws_d = to_dev_operand(wc, wsc, K)
    out = torch.empty(M, N, dtype=torch.float32, device=DEV)
    nv.nvfp4_gemm(a_codes, a_sc, float(g), w_d, ws_d, float(gw), M, N, K, out)
    torch.cuda.synchronize()
    check_device_error_word()
    assert_gemm_close(out.cpu().numpy(), oracle.gemm(ac, asc, g, wc, wsc, gw), "static scale")
