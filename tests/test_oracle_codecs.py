"""Pins for the oracle's scalar codecs (CPU only).

The oracle is checked against things other than itself: hand-derived worked
examples (tests/golden), brute-force nearest-value searches written here as
argmin over every code, and the library casts ``ml_dtypes.float4_e2m1fn`` and
``torch.float8_e4m3fn`` in the ranges where they implement the same
round-to-nearest-even rule.
"""
import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_worked_examples.txt")


def golden_lines(kind):
    out = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.split()[0] == kind:
                out.append(line)
    return out


def same_float(a, b):
    if math.isnan(b):
        return math.isnan(a)
    return a == b and math.copysign(1.0, a) == math.copysign(1.0, b)


# ---- P1: E2M1 codec ------------------------------------------------------

def test_e2m1_decode_golden():
    lines = golden_lines("e2m1_dec")
    assert len(lines) == 16
    for line in lines:
        _, code, val = line.split()
        assert same_float(oracle.e2m1_decode(int(code, 16)), float(val)), line


def test_e2m1_grid_roundtrip():
    grid = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    for code in range(16):
        v = oracle.e2m1_decode(code)
        assert oracle.e2m1_encode(v) == code
    for mag in grid:
        for s in (1.0, -1.0):
            v = s * mag
            c = oracle.e2m1_encode(v)
            assert oracle.e2m1_decode(c) == v


def test_e2m1_encode_golden():
    for line in golden_lines("e2m1_enc"):
        _, v, code = line.split()
        assert oracle.e2m1_encode(float(v)) == int(code, 16), line


# ---- P2: E2M1 rounding by brute force -------------------------------------

def brute_e2m1(v):
    """argmin over all 16 codes of |v - value|; ties: even mantissa bit; the
    sign of the result follows v (signed zero included); |v| >= 6 -> 6."""
    vals = np.array([oracle.e2m1_decode(c) for c in range(16)])
    out = np.empty(v.shape, np.uint8)
    for i, x in enumerate(v.astype(np.float64)):
        neg = math.copysign(1.0, x) < 0
        cands = [c for c in range(16) if ((c & 8) != 0) == neg]
        if abs(x) >= 6:
            out[i] = 0xF if neg else 0x7
            continue
        d = [abs(x - vals[c]) for c in cands]
        best = min(d)
        ties = [c for c, dd in zip(cands, d) if dd == best]
        ties = [c for c in ties if c & 1 == 0] or ties
        out[i] = ties[0]
    return out


def e2m1_probe_values():
    lattice = np.arange(-8 * 1024, 8 * 1024 + 1, dtype=np.float64) / 1024.0
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], np.float32)
    around = []
    for m in mids:
        for s in (1, -1):
            x = np.float32(s * m)
            around += [np.nextafter(x, np.float32(-np.inf)), x, np.nextafter(x, np.float32(np.inf))]
    return np.concatenate([lattice.astype(np.float32), np.array(around, np.float32),
                           np.array([-0.0, 0.0, 1e-30, -1e-30, 7.0, -7.0, 1e30], np.float32)])


def test_e2m1_brute_force():
    v = e2m1_probe_values()
    assert np.array_equal(oracle.e2m1_encode_array(v), brute_e2m1(v))


def test_e2m1_against_ml_dtypes():
    # ml_dtypes' float4_e2m1fn rounds to nearest-even and saturates at 6; it
    # drops the sign of zero, so compare decoded values with abs for zeros.
    rng = np.random.default_rng(0)
    v = np.concatenate([e2m1_probe_values(),
                        (rng.standard_normal(200000) * 3).astype(np.float32)])
    ours = np.array([oracle.e2m1_decode(c) for c in range(16)])[oracle.e2m1_encode_array(v)]
    lib = v.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(ours, lib)


# ---- P3: E4M3 codec --------------------------------------------------------

def test_e4m3_decode_golden():
    for line in golden_lines("e4m3_dec"):
        _, code, val = line.split()
        assert same_float(oracle.e4m3_decode(int(code, 16)), float(val)), line


def test_e4m3_all_finite_roundtrip():
    n = 0
    for code in range(256):
        v = oracle.e4m3_decode(code)
        if math.isnan(v):
            assert code in (0x7F, 0xFF)
            continue
        n += 1
        assert oracle.e4m3_encode(v) == code
    assert n == 254


def test_e4m3_decode_matches_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    ours = np.array([oracle.e4m3_decode(c) for c in range(256)])
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    ok = ~np.isnan(ours)
    assert np.array_equal(ours[ok], lib[ok])


def test_e4m3_encode_golden():
    for line in golden_lines("e4m3_enc"):
        _, v, code = line.split()
        assert oracle.e4m3_encode(float(v)) == int(code, 16), line


def e4m3_probe_values():
    vals = np.array([oracle.e4m3_decode(c) for c in range(0x7F)])
    mids = (vals[:-1] + vals[1:]) / 2
    pts = []
    for m in np.concatenate([vals, mids]).astype(np.float32):
        pts += [np.nextafter(m, np.float32(-np.inf)), m, np.nextafter(m, np.float32(np.inf))]
    return np.array([p for p in pts if p >= 0], np.float32)


def test_e4m3_brute_force():
    vals = np.array([oracle.e4m3_decode(c) for c in range(0x7F)])
    v = np.concatenate([e4m3_probe_values(),
                        np.array([0.0, 1e-30, 460.0, 1e10], np.float32)])
    ours = oracle.e4m3_encode_array(v)
    for x, c in zip(v.astype(np.float64), ours):
        if x >= 448:
            assert c == 0x7E
            continue
        d = np.abs(x - vals)
        best = d.min()
        ties = [k for k in np.nonzero(d == best)[0]]
        even = [k for k in ties if k % 2 == 0] or ties
        assert c == even[0], (x, c, ties)


def test_e4m3_dense_against_torch():
    # every 61st positive float32 bit pattern up to 464, plus every midpoint
    # +-1 ulp; torch's cast rounds to nearest-even and agrees with saturation
    # up to 464 (above that it gives NaN, which the scale path never uses).
    top = np.float32(464.0).view(np.uint32)
    bits = np.arange(0, int(top) + 1, 61, dtype=np.uint32)
    v = np.concatenate([bits.view(np.float32), e4m3_probe_values()])
    v = v[v <= 464.0]
    ours = oracle.e4m3_encode_array(v)
    lib = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, lib)


def test_e4m3_negative_mirrors_positive():
    v = e4m3_probe_values()
    assert np.array_equal(oracle.e4m3_encode_array(-v), oracle.e4m3_encode_array(v) | 0x80)
