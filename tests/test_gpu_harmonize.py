"""Offline global-scale harmonisation on the GPU, against the oracle.

A fused projection weight whose segments were calibrated with their own
global scales is rewritten to one common scale, so that a GEMM applying one
scale serves every segment ("pre-harmonized" checkpoint) [cctest.ai article,
"Main findings"; anthology record LIT-800, "Standing in the anthology"].
Checks: bitwise equality of the rewritten scale bytes in both layouts,
ragged segments and buffer tails, in-place use, and the single-scale GEMM on
harmonized scales against the oracle, with its error against the exact
per-segment result far below that of the unrepaired single-scale GEMM."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_10_b200 as nv
import oracle
import synth
from tests.gpu_helpers import (DEV, assert_gemm_close, check_device_error_word, oracle_quantize, rel_errors,
                               to_dev_operand)

pytestmark = pytest.mark.gpu

FINITE = np.array([b for b in range(256) if b not in (0x7F, 0xFF)], np.uint8)


def _segment_weight(segs, sigmas, K, seed):
    codes, scales, gs = [], [], []
    for i, (n, sd) in enumerate(zip(segs, sigmas)):
        w = synth.normal((n, K), seed=seed + 31 * i, std=sd).numpy()
        c, s, g = oracle_quantize(w)
        codes.append(c), scales.append(s), gs.append(g)
    offs = np.cumsum([0] + list(segs)).astype(np.int64)
    return np.concatenate(codes), np.concatenate(scales), offs, np.array(gs, np.float32)


def _gpu_harmonize(scales_rm, K, offs, gs, g, layout, in_place=False):
    N = scales_rm.shape[0]
    src = scales_rm if layout == nv.SF_ROWMAJOR else oracle.scales_to_tc(scales_rm, K)
    d = torch.from_numpy(np.ascontiguousarray(src)).to(DEV)
    out = d if in_place else torch.full_like(d, 0x5A)
    nv.nvfp4_harmonize_scales(d, N, K, offs, gs, g, out, layout)
    torch.cuda.synchronize()
    check_device_error_word()
    return out.cpu().numpy()


def _expect(scales_rm, K, offs, gs, g, layout):
    h = oracle.harmonize_scales(scales_rm, offs, gs, g)
    return h if layout == nv.SF_ROWMAJOR else oracle.scales_to_tc(h, K)


@pytest.mark.parametrize("layout", [nv.SF_ROWMAJOR, nv.SF_TCGEN05])
def test_fused_gdn_weight_scales_bitwise(layout):
    wl = synth.FUSED_GDN
    K = wl.K
    _, sc, offs, gs = _segment_weight(wl.segments, wl.seg_sigma, K, seed=40)
    g = gs.min()
    got = _gpu_harmonize(sc, K, offs, gs, g, layout)
    assert np.array_equal(got, _expect(sc, K, offs, gs, g, layout))


@pytest.mark.parametrize("layout", [nv.SF_ROWMAJOR, nv.SF_TCGEN05])
@pytest.mark.parametrize("N,K,offs", [
    (19, 96, [0, 5, 8, 9, 16]),          # rows 16..18 outside every segment; 114 bytes: partial vector
    (300, 80, [0, 1, 130, 300]),         # 1500 row-major bytes; TCGEN05 row and column padding
    (3, 16, [0, 3]),
    (257, 4064, [0, 128, 129, 257]),     # every finite byte value in every row
])
def test_ragged_segments_and_tails_bitwise(layout, N, K, offs):
    rng = np.random.default_rng(N + K)
    if K == 4064:
        sc = np.tile(FINITE, (N, 1))
    else:
        sc = rng.choice(FINITE, size=(N, K // 16)).astype(np.uint8)
    gs = rng.uniform(1.0, 5000.0, size=len(offs) - 1).astype(np.float32)
    for g in (gs.min(), np.float32(gs.max() * 3)):         # the second one saturates
        got = _gpu_harmonize(sc, K, offs, gs, g, layout)
        assert np.array_equal(got, _expect(sc, K, offs, gs, g, layout)), g


def test_in_place():
    K = 512
    _, sc, offs, gs = _segment_weight((256, 128, 48, 48), (0.02, 0.005, 0.00125, 0.0003125), K, seed=41)
    got = _gpu_harmonize(sc, K, offs, gs, gs.min(), nv.SF_TCGEN05, in_place=True)
    assert np.array_equal(got, _expect(sc, K, offs, gs, gs.min(), nv.SF_TCGEN05))


def test_single_scale_gemm_on_harmonized_weights():
    wl = synth.FUSED_GDN
    M, K = 256, 1024
    x = synth.activation(wl, M=M, K=K).float().numpy()
    ac, asc, ga = oracle_quantize(x)
    wc, wsc, offs, gs = _segment_weight(wl.segments, wl.seg_sigma, K, seed=42)
    N = int(offs[-1])
    g = gs.min()
    a_d, as_d = to_dev_operand(ac, asc, K)
    w_d, ws_d = to_dev_operand(wc, wsc, K)
    h_d = torch.empty_like(ws_d)
    nv.nvfp4_harmonize_scales(ws_d, N, K, offs, gs, g, h_d)
    out = torch.empty(M, N, dtype=torch.float32, device=DEV)
    nv.nvfp4_gemm(a_d, as_d, float(ga), w_d, h_d, float(g), M, N, K, out)
    broken = torch.empty_like(out)
    nv.nvfp4_gemm(a_d, as_d, float(ga), w_d, ws_d, float(gs[0]), M, N, K, broken)
    torch.cuda.synchronize()
    check_device_error_word()
    h = oracle.harmonize_scales(wsc, offs, gs, g)
    assert_gemm_close(out.cpu().numpy(), oracle.gemm(ac, asc, ga, wc, h, g), "harmonized")
    exact = oracle.fused_proj(ac, asc, ga, wc, wsc, offs, gs)
    for i in range(len(gs)):
        seg = slice(int(offs[i]), int(offs[i + 1]))
        _, e_h = rel_errors(out.cpu().numpy()[:, seg], exact[:, seg])
        _, e_b = rel_errors(broken.cpu().numpy()[:, seg], exact[:, seg])
        assert e_h < 0.05, (i, e_h)          # half an E4M3 step per scale at most
        if i > 0:
            assert e_b > 1.0, (i, e_b)       # g_i / g_0 is 4 or more there


def test_cases_where_the_fp32_order_decides():
    """Ratios that put s * g / g_i next to an E4M3 rounding midpoint, where
    rounding g / g_i to FP32 first and rounding once at the end disagree
    (found on the CPU); the kernel must take the oracle's FP32 order."""
    vals = torch.arange(1, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    rng = np.random.default_rng(61)
    found = 0
    for _ in range(20000):
        v = float(vals[rng.integers(len(vals))])
        k = int(rng.integers(0, len(vals) - 1))
        if vals[k + 1] > v:
            continue
        mid = (float(vals[k]) + float(vals[k + 1])) / 2
        g_i = np.float32(rng.uniform(1, 4000))
        g = np.float32(np.float32(mid / v) * g_i)
        byte = int(torch.tensor(np.float32(v)).to(torch.float8_e4m3fn).view(torch.uint8))
        sc = np.full((1, 2), byte, np.uint8)                # N = 1, K = 32
        want = oracle.harmonize_scales(sc, [0, 1], [g_i], g)
        exact = np.float32(v * float(g) / float(g_i))       # double product, one rounding
        if want[0, 0] == int(torch.tensor(exact).to(torch.float8_e4m3fn).view(torch.uint8)):
            continue
        for layout in (nv.SF_ROWMAJOR, nv.SF_TCGEN05):
            got = _gpu_harmonize(sc, 32, [0, 1], [g_i], g, layout)
            assert np.array_equal(got, _expect(sc, 32, [0, 1], [g_i], g, layout)), (v, g_i, g, layout)
        found += 1
        if found == 12:
            break
    assert found == 12
