"""Pins for the oracle's MXFP4 contrast format (CPU only).

The pages contrast NVFP4's 16-element E4M3-scaled blocks with the MX
format's 32-element blocks sharing a power-of-two scale, and credit the
finer blocks with keeping outliers local [anthology record LIT-800,
"Standing in the anthology"].  The oracle follows the published OCP
Microscaling v1.0 conversion: E = floor(log2 amax) - 2, scale byte E + 127,
codes E2M1(x / 2^E), nearest even, saturating.

What fixes it, other than the oracle itself:
  * hand-derived blocks (scale byte and codes worked out by hand);
  * torch's float8_e8m0fnu decoding of every finite scale byte;
  * Python's frexp for floor(log2 amax), and amax / 2^E in [4, 8);
  * brute force over the E2M1 values in exact rational arithmetic;
  * the exact rational GEMM sum on small operands, numpy's FP64 matmul on
    larger ones;
  * the chunk order's byte positions worked out by hand;
  * the pages' qualitative claim, as an inequality on outlier inputs.
"""
import math
from fractions import Fraction

import numpy as np
import torch

import oracle
import synth

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _codes(c):
    lo, hi = c & 0xF, c >> 4
    return np.stack([lo, hi], -1).reshape(c.shape[0], -1)


def test_hand_derived_blocks():
    cases = [
        # (first values of a 32-block, rest zero), scale byte, first codes
        ([6.0, 3.0, -1.5, 0.25], 127, [0x7, 0x5, 0xB, 0x0]),      # E = 0; 0.25 ties to 0
        ([7.0, -7.0, 5.0, 0.75], 127, [0x7, 0xF, 0x6, 0x2]),      # 7 clips to 6; 5 ties to 4; 0.75 ties to 1
        ([0.3, 0.2, -0.05, 0.1], 123, [0x6, 0x5, 0xA, 0x3]),      # E = -4: 4.8, 3.2, -0.8, 1.6
        ([1000.0, 64.0, -100.0], 134, [0x7, 0x1, 0xA]),           # E = 7: 7.8125 clips, 0.5, -0.78 -> -1
        ([1e-40, -1e-40], 0, [0x0, 0x8]),                          # E clamps at -127; signed zeros
        ([0.0, -0.0], 0, [0x0, 0x8]),                              # all-zero block
    ]
    for vals, scale, codes in cases:
        x = np.zeros((1, 32), np.float32)
        x[0, :len(vals)] = vals
        c, s = oracle.mx_quantize(x)
        assert s[0, 0] == scale, vals
        assert list(_codes(c)[0, :len(codes)]) == codes, vals
        assert oracle.e8m0_decode(scale) == 2.0 ** (scale - 127)


def _brute_code(y: Fraction) -> int:
    a = abs(y)
    best = min(range(8), key=lambda i: (abs(Fraction(E2M1[i]) - a), i & 1))  # ties: even code
    if a >= 6:
        best = 7
    return best | (8 if y < 0 else 0)


def test_scale_rule_and_brute_force_codes():
    rng = np.random.default_rng(50)
    for trial in range(300):
        spread = rng.uniform(-30, 30)
        x = (rng.standard_normal(32) * 2.0 ** spread).astype(np.float32)
        if trial % 7 == 0:
            x[rng.integers(32)] *= 200                      # an outlier in the block
        c, s = oracle.mx_quantize(x[None, :])
        amax = float(np.abs(x).max())
        _, e2 = math.frexp(amax)
        E = max(-127, min(127, e2 - 1 - 2))
        assert s[0, 0] == E + 127
        assert 4 <= amax / 2.0 ** E < 8
        codes = _codes(c)[0]
        for i in range(32):
            y = Fraction(float(x[i])) / Fraction(2) ** E
            want = _brute_code(y)
            if y == 0:
                want = 0x8 if math.copysign(1.0, float(x[i])) < 0 else 0x0
            assert codes[i] == want, (trial, i, float(x[i]), E)


def test_dequantize_and_gemm_exactly():
    rng = np.random.default_rng(51)
    M, N, K = 2, 3, 64
    a = (rng.standard_normal((M, K)) * 3).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    ac, asc = oracle.mx_quantize(a)
    wc, wsc = oracle.mx_quantize(w)
    da, dw = oracle.mx_dequantize(ac, asc), oracle.mx_dequantize(wc, wsc)
    sign = lambda c: -1 if c & 8 else 1  # noqa: E731
    for (codes, sc, d) in ((ac, asc, da), (wc, wsc, dw)):
        cc = _codes(codes)
        for r in range(cc.shape[0]):
            for k in range(K):
                v = sign(cc[r, k]) * E2M1[cc[r, k] & 7] * 2.0 ** (int(sc[r, k // 32]) - 127)
                assert d[r, k] == v
    out = oracle.mx_gemm(ac, asc, wc, wsc)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(da[m, k])) * Fraction(float(dw[n, k])) for k in range(K))
            assert out[m, n] == float(exact)      # dyadic values: the FP64 sum is exact here
    x = synth.student_t_outliers(64, 1024, seed=52, dtype=torch.float32).numpy()
    y = synth.normal((96, 1024), seed=53, std=0.02).numpy()
    xc, xs = oracle.mx_quantize(x)
    yc, ys = oracle.mx_quantize(y)
    ref = oracle.mx_dequantize(xc, xs) @ oracle.mx_dequantize(yc, ys).T
    np.testing.assert_allclose(oracle.mx_gemm(xc, xs, yc, ys), ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_chunk_order_byte_positions():
    R, K = 130, 384                                   # 12 scales per row: 3 chunks per row block
    s = np.arange(R * (K // 32), dtype=np.int64).reshape(R, K // 32).astype(np.uint8)
    tc = oracle.mx_scales_to_tc(s, K)
    assert tc.size == 2 * 3 * 512
    for r, j in ((0, 0), (1, 0), (0, 5), (33, 2), (127, 11), (128, 0), (129, 7)):
        off = ((r // 128) * 3 + j // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + j % 4
        assert tc[off] == s[r, j], (r, j)
    assert np.array_equal(oracle.mx_scales_from_tc(tc, R, K), s)


def test_sixteen_element_blocks_keep_outliers_local():
    """On heavy-tailed activations with outlier channels, NVFP4's error is
    below MXFP4's (the pages' qualitative claim)."""
    for x in (synth.student_t_outliers(256, 2048, seed=54, dtype=torch.float32).numpy(),
              synth.normal_with_outlier_channels(256, 2048, seed=55, dtype=torch.float32).numpy()):
        g = oracle.global_scale(oracle.amax(x))
        c, s = oracle.quantize(x, g)
        e_nv = np.linalg.norm(oracle.dequantize(c, s, g) - x) / np.linalg.norm(x)
        mc, ms = oracle.mx_quantize(x)
        e_mx = np.linalg.norm(oracle.mx_dequantize(mc, ms) - x) / np.linalg.norm(x)
        assert e_nv < 0.85 * e_mx, (e_nv, e_mx)


def test_e8m0_decode_matches_torch():
    """torch's float8_e8m0fnu (the OCP E8M0 scale type) decodes every finite
    byte to the same power of two."""
    t = torch.arange(0, 255, dtype=torch.uint8).view(torch.float8_e8m0fnu).float().double().numpy()
    for b in range(255):
        assert oracle.e8m0_decode(b) == t[b], b
