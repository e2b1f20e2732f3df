"""Pins for the oracle's offline global-scale harmonisation (CPU only).

A fused projection weight whose row segments were calibrated with their own
global scales is rewritten so that one common scale serves the whole GEMM:
codes kept, every block scale multiplied by q_i = g / g_i and re-encoded
[cctest.ai article, "Main findings": the released checkpoint is
pre-harmonized; anthology record LIT-800, "Standing in the anthology": per-
module scales served by a fused kernel give mis-scaled gates].

What fixes it, other than the oracle itself:
  * q = 1 is the identity on every finite scale byte;
  * q = 2^-k moves the exponent field down by k while the result stays
    normal (a closed form on the bit layout);
  * torch's float8_e4m3fn cast (round to nearest even) of the FP32 product,
    for random ratios, over all 254 finite bytes;
  * segment bookkeeping: the whole-matrix call equals per-segment calls, and
    rows outside every segment are untouched;
  * the dequantized value moves by at most half an E4M3 step;
  * the mismatch the pages describe, in closed form: one GEMM with one weight
    scale g_0 gives segment i scaled by g_i / g_0.
"""
import numpy as np
import torch

import oracle
import synth

FINITE = np.array([b for b in range(256) if b not in (0x7F, 0xFF)], np.uint8)


def _grid(rows):
    """rows x 254 scale bytes (K = 254 * 16), every finite byte in each row."""
    return np.tile(FINITE, (rows, 1))


def _decode(b):
    return np.array([oracle.e4m3_decode(int(v)) for v in np.ravel(b)]).reshape(np.shape(b))


def test_unit_ratio_is_the_identity():
    s = _grid(3)
    g = np.float32(2688.0 / 3.7)
    out = oracle.harmonize_scales(s, [0, 2, 3], [g, g], g)
    assert np.array_equal(out, s)


def test_power_of_two_ratio_lowers_the_exponent_field():
    s = _grid(1)
    out = oracle.harmonize_scales(s, [0, 1], [np.float32(3.0)], np.float32(0.375))  # q = 2^-3
    exp_field = (s[0] >> 3) & 0xF
    normal_after = exp_field >= 4
    assert normal_after.sum() > 150
    assert np.array_equal(out[0][normal_after], s[0][normal_after] - (3 << 3))
    # below that the exact value v / 8 is rounded onto the subnormal grid
    low = ~normal_after
    assert np.all(np.abs(_decode(out[0][low]) - _decode(s[0][low]) / 8) <= 2.0 ** -10)


def test_random_ratios_match_torch_e4m3_cast():
    rng = np.random.default_rng(20)
    s = _grid(1)
    v = torch.tensor(s[0]).view(torch.float8_e4m3fn).float()  # independent decode
    for _ in range(40):
        g_i = np.float32(rng.uniform(0.5, 3000.0))
        g = np.float32(g_i * rng.uniform(1e-3, 1.0))
        q = torch.tensor(np.float32(g / g_i))
        expect = (v * q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        out = oracle.harmonize_scales(s, [0, 1], [g_i], g)
        assert np.array_equal(out[0], expect), (g_i, g)


def test_each_segment_uses_its_own_scale_and_outside_rows_are_kept():
    rng = np.random.default_rng(21)
    s = rng.integers(0, 0x7F, size=(19, 8), dtype=np.uint8)
    offs = [0, 5, 8, 9, 16]                     # rows 16..18 belong to no segment
    gs = [np.float32(v) for v in (11.0, 37.5, 300.0, 2.25)]
    g = np.float32(1.75)
    out = oracle.harmonize_scales(s, offs, gs, g)
    for i in range(4):
        part = oracle.harmonize_scales(s[offs[i]:offs[i + 1]], [0, offs[i + 1] - offs[i]], [gs[i]], g)
        assert np.array_equal(out[offs[i]:offs[i + 1]], part)
    assert np.array_equal(out[16:], s[16:])
    # the segment scales differ, so a shifted offset would show
    assert not np.array_equal(out[4], oracle.harmonize_scales(s[4:5], [0, 1], [gs[1]], g)[0])


def test_dequantized_values_move_by_at_most_half_a_step():
    w = synth.weight(synth.FUSED_GDN, N=None, K=256).float().numpy()
    offs = synth.segment_offsets(synth.FUSED_GDN)
    gs, scales = [], []
    for i in range(4):
        part = w[offs[i]:offs[i + 1]]
        g_i = oracle.global_scale(oracle.amax(part))
        gs.append(g_i)
        scales.append(oracle.quantize(part, g_i)[1])
    scales = np.concatenate(scales)
    g = min(gs)
    h = oracle.harmonize_scales(scales, offs, gs, g)
    before = np.concatenate([_decode(scales[offs[i]:offs[i + 1]]) / float(gs[i]) for i in range(4)])
    after = _decode(h) / float(g)
    normal = _decode(h) >= 2.0 ** -6
    err = np.abs(after - before)
    assert np.all(err[normal] <= before[normal] * (2.0 ** -4 + 1e-6))
    assert np.all(err[~normal] <= 2.0 ** -10 / float(g) * (1 + 1e-6))
    # segments with g_i != g are re-rounded (g / g_i is not a power of two)
    assert (err[offs[1]:] > 0).any()
    assert np.all(err[:offs[1]] == 0)


def test_one_weight_scale_for_all_segments_scales_segment_i_by_g_i_over_g_0():
    wl = synth.FUSED_GDN
    M, K = 8, 128
    x = synth.activation(wl, M=M, K=K).float().numpy()
    w = synth.weight(wl, K=K).float().numpy()
    offs = synth.segment_offsets(wl)
    ga = oracle.global_scale(oracle.amax(x))
    ac, asc = oracle.quantize(x, ga)
    gs, wc, wsc = [], [], []
    for i in range(4):
        part = w[offs[i]:offs[i + 1]]
        g_i = oracle.global_scale(oracle.amax(part))
        c, s = oracle.quantize(part, g_i)
        gs.append(g_i), wc.append(c), wsc.append(s)
    wc, wsc = np.concatenate(wc), np.concatenate(wsc)
    exact = oracle.fused_proj(ac, asc, ga, wc, wsc, offs, gs)
    broken = oracle.gemm(ac, asc, ga, wc, wsc, gs[0])
    for i in range(4):
        seg = slice(offs[i], offs[i + 1])
        want = exact[:, seg] * (float(gs[i]) / float(gs[0]))
        # FP64 sums in another order: compare against the segment's scale
        np.testing.assert_allclose(broken[:, seg], want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    assert float(gs[3]) / float(gs[0]) > 20  # the last segments come out far too large


def test_the_fp32_order_decides_near_e4m3_midpoints():
    """Cases where s * g / g_i lands next to an E4M3 rounding midpoint, so
    that rounding g / g_i to FP32 first (the reading taken) and rounding the
    exact product once give different bytes; the oracle must give the first,
    as torch's cast of the FP32 product does."""
    from fractions import Fraction

    vals = torch.arange(1, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    cast = lambda y: int(torch.tensor(np.float32(y)).to(torch.float8_e4m3fn).view(torch.uint8))  # noqa: E731
    rng = np.random.default_rng(60)
    found = 0
    for _ in range(20000):
        v = float(vals[rng.integers(len(vals))])
        k = int(rng.integers(0, len(vals) - 1))
        if vals[k + 1] > v:
            continue
        mid = (float(vals[k]) + float(vals[k + 1])) / 2
        g_i = np.float32(rng.uniform(1, 4000))
        g = np.float32(np.float32(mid / v) * g_i)
        fp32_order = cast(np.float32(np.float32(v) * np.float32(g / g_i)))
        exact_order = cast(float(Fraction(v) * Fraction(float(g)) / Fraction(float(g_i))))
        if fp32_order == exact_order:
            continue
        byte = np.uint8(cast(v))
        out = oracle.harmonize_scales(np.full((1, 2), byte, np.uint8), [0, 1], [g_i], g)
        assert out[0, 0] == fp32_order and out[0, 1] == fp32_order, (v, g_i, g)
        found += 1
        if found == 12:
            break
    assert found == 12
