"""Pins for the oracle's FP64 GEMM and fused projection (CPU only).

  * an exact integer evaluation of the same block-scaled sum (every E2M1 value
    is a multiple of 1/2 and every E4M3 value a multiple of 2^-9, so the sum is
    an integer times 2^-20) must agree with the FP64 result to 1e-12;
  * numpy's FP64 matmul of the dequantized operands (catches transposed or
    mis-indexed operands);
  * closed forms: hand-derived golden values, a one-hot weight that copies
    one dequantized activation column, exact halving when g_A doubles;
  * the fused projection: each output segment equals the plain GEMM of that
    segment with its own weight scale [anthology record LIT-800, "Standing in
    the anthology"; cctest.ai article, "Main findings"], and a single shared
    scale gives the mis-scaled gate outputs the pages describe.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.test_oracle_codecs import golden_lines


def quant(x):
    x = np.asarray(x, np.float32)
    g = oracle.global_scale(oracle.amax(x))
    c, s = oracle.quantize(x, g)
    return c, s, g


def test_gemm_golden_closed_forms():
    lines = golden_lines("gemm")
    assert len(lines) == 3
    for line in lines:
        _, K, ac, asc, ga, wc, wsc, gw, out = line.split()
        K = int(K)
        a_codes = np.full((1, K // 2), int(ac, 16) * 17, np.uint8)   # both nibbles
        a_sc = np.full((1, K // 16), int(asc, 16), np.uint8)
        w_codes = np.full((1, K // 2), int(wc, 16) * 17, np.uint8)
        w_sc = np.full((1, K // 16), int(wsc, 16), np.uint8)
        r = oracle.gemm(a_codes, a_sc, float(ga), w_codes, w_sc, float(gw))
        assert r[0, 0] == float(out), line


@pytest.mark.parametrize("M,N,K", [(3, 5, 32), (16, 40, 256), (7, 33, 1088)])
def test_gemm_fp64_matches_exact_integer_sum(M, N, K):
    a = synth.student_t_outliers(M, K, seed=M, dtype=torch.float32).numpy()
    w = synth.normal((N, K), seed=N, std=0.02).numpy()
    ac, as_, ga = quant(a)
    wc, ws, gw = quant(w)
    r = oracle.gemm(ac, as_, ga, wc, ws, gw)
    S = oracle.gemm_exact(ac, as_, wc, ws)
    exact = S.astype(np.float64) * 2.0 ** -20 / (np.float64(ga) * np.float64(gw))
    assert np.max(np.abs(r - exact)) <= 1e-12 * np.max(np.abs(exact))


def test_exact_path_large_k_fits_int64():
    # all-max codes and scales at K = 17408: the exact sum must not overflow
    K = 17408
    c = np.full((1, K // 2), 0x77, np.uint8)
    s = np.full((1, K // 16), 0x7E, np.uint8)
    S = oracle.gemm_exact(c, s, c, s)
    assert S[0, 0] == 144 * K * (448 * 512) ** 2


def test_gemm_matches_numpy_on_dequantized():
    a = synth.student_t_outliers(9, 320, seed=4, dtype=torch.float32).numpy()
    w = synth.normal((21, 320), seed=8, std=0.02).numpy()
    ac, as_, ga = quant(a)
    wc, ws, gw = quant(w)
    ref = oracle.dequantize(ac, as_, ga) @ oracle.dequantize(wc, ws, gw).T
    r = oracle.gemm(ac, as_, ga, wc, ws, gw)
    assert np.allclose(r, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_one_hot_weight_copies_an_activation_column():
    M, N, K = 5, 12, 128
    a = synth.student_t_outliers(M, K, seed=6, dtype=torch.float32).numpy()
    ac, as_, ga = quant(a)
    rng = np.random.default_rng(2)
    cols = rng.integers(0, K, size=N)
    w_nib = np.zeros((N, K), np.uint8)
    w_nib[np.arange(N), cols] = 0x2          # value 1.0
    wc = (w_nib[:, 0::2] | (w_nib[:, 1::2] << 4)).astype(np.uint8)
    ws = np.full((N, K // 16), 0x38, np.uint8)  # scale 1.0
    r = oracle.gemm(ac, as_, ga, wc, ws, 1.0)
    deq = oracle.dequantize(ac, as_, ga)
    assert np.array_equal(r, deq[:, cols])


def test_doubling_activation_scale_halves_output():
    a = synth.normal((4, 256), seed=1).numpy()
    w = synth.normal((6, 256), seed=2, std=0.02).numpy()
    ac, as_, ga = quant(a)
    wc, ws, gw = quant(w)
    r1 = oracle.gemm(ac, as_, ga, wc, ws, gw)
    r2 = oracle.gemm(ac, as_, np.float32(2 * ga), wc, ws, gw)
    assert np.array_equal(r2 * 2, r1)


def test_all_six_blocks_closed_form():
    K = 96
    rng = np.random.default_rng(3)
    sa = rng.integers(0x08, 0x7F, size=(1, K // 16)).astype(np.uint8)
    sw = rng.integers(0x08, 0x7F, size=(1, K // 16)).astype(np.uint8)
    c = np.full((1, K // 2), 0x77, np.uint8)
    r = oracle.gemm(c, sa, 1.5, c, sw, 0.75)
    e = np.array([oracle.e4m3_decode(int(v)) for v in sa[0]])
    f = np.array([oracle.e4m3_decode(int(v)) for v in sw[0]])
    expected = np.sum(36.0 * 16 * e * f) / (1.5 * 0.75)
    assert abs(r[0, 0] - expected) <= 1e-14 * abs(expected)


# ---- fused projection ------------------------------------------------------

def _fused_case(M=6, K=256, segs=(40, 24, 8, 8), sig=(0.02, 0.005, 0.00125, 0.0003125)):
    a = synth.student_t_outliers(M, K, seed=12, dtype=torch.float32).numpy()
    ac, as_, ga = quant(a)
    parts, gs = [], []
    for i, (n, sd) in enumerate(zip(segs, sig)):
        w = synth.normal((n, K), seed=100 + i, std=sd).numpy()
        wc, ws, gw = quant(w)
        parts.append((wc, ws))
        gs.append(gw)
    offs = np.cumsum([0] + list(segs))
    wc = np.concatenate([p[0] for p in parts])
    ws = np.concatenate([p[1] for p in parts])
    return ac, as_, ga, wc, ws, offs, np.array(gs, np.float32), parts


def test_fused_segments_equal_unfused():
    ac, as_, ga, wc, ws, offs, gs, parts = _fused_case()
    fused = oracle.fused_proj(ac, as_, ga, wc, ws, offs, gs)
    for i, (pc, ps) in enumerate(parts):
        alone = oracle.gemm(ac, as_, ga, pc, ps, gs[i])
        assert np.array_equal(fused[:, offs[i]:offs[i + 1]], alone)


def test_fused_shared_scale_mis_scales_the_small_segments():
    # the failure the pages report: the gate segments computed with the
    # first module's scale come out off by the ratio of the scales
    ac, as_, ga, wc, ws, offs, gs, parts = _fused_case()
    good = oracle.fused_proj(ac, as_, ga, wc, ws, offs, gs)
    bad = oracle.fused_proj(ac, as_, ga, wc, ws, offs, np.full_like(gs, gs[0]))
    assert np.array_equal(bad[:, :offs[1]], good[:, :offs[1]])
    for i in (2, 3):
        sl = slice(offs[i], offs[i + 1])
        ratio = np.linalg.norm(bad[:, sl]) / np.linalg.norm(good[:, sl])
        assert abs(ratio - np.float64(gs[i]) / np.float64(gs[0])) < 1e-9 * ratio
        assert abs(ratio - 1) > 1.0
