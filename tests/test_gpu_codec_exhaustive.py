"""Exhaustive check of the quantizer's element encoders on the GPU against
the oracle, over every non-NaN float32 bit pattern.

The GPU converts all 2^32 patterns (in chunks).  On the host each chunk is cut
into runs of equal output; the oracle is evaluated on both ends of every run
(and of the chunk).  Within one sign both encoders are monotone in |x|
(nearest-value rounding; pinned by the oracle tests), so equal ends and a
constant GPU run mean equality on every value of the run."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_10_b200 as nv
import oracle
from tests.gpu_helpers import DEV

pytestmark = pytest.mark.gpu

CHUNK = 1 << 28
POS_NAN_LO, POS_NAN_HI = 0x7F800001, 0x7FFFFFFF
NEG_NAN_LO, NEG_NAN_HI = 0xFF800001, 0xFFFFFFFF


def _ranges():
    # non-NaN patterns: [0, 0x7F800000] and [0x80000000, 0xFF800000]
    return [(0, POS_NAN_LO), (0x80000000, NEG_NAN_LO)]


def _check_runs(bits_lo: int, codes: np.ndarray, enc):
    n = codes.size
    change = np.nonzero(codes[1:] != codes[:-1])[0]
    idx = np.unique(np.concatenate([[0, n - 1], change, change + 1]))
    v = (np.uint64(bits_lo) + idx.astype(np.uint64)).astype(np.uint32).view(np.float32)
    ref = enc(v)
    bad = np.nonzero(ref != codes[idx])[0]
    assert bad.size == 0, [(hex(int(np.float32(v[i]).view(np.uint32))), int(codes[idx[i]]), int(ref[i]))
                           for i in bad[:5]]
    return change.size


@pytest.mark.parametrize("fmt", ["e4m3", "e2m1"])
def test_encoder_exhaustive(fmt):
    total_runs = 0
    for lo, hi in _ranges():
        start = lo
        while start < hi:
            n = min(CHUNK, hi - start)
            n -= n & 1
            if n == 0:          # the last pattern of a range (an infinity) has its own test below
                break
            bits = torch.arange(n, dtype=torch.int64, device=DEV) + start
            bits = torch.where(bits >= 2 ** 31, bits - 2 ** 32, bits)     # uint32 pattern as int32
            x = bits.to(torch.int32).view(torch.float32)
            if fmt == "e4m3":
                out = torch.empty(n, dtype=torch.uint8, device=DEV)
                nv.nvfp4_convert_e4m3(x, out)
                codes = out.cpu().numpy()
                total_runs += _check_runs(start, codes, oracle.e4m3_encode_array)
            else:
                out = torch.empty(n // 2, dtype=torch.uint8, device=DEV)
                nv.nvfp4_convert_e2m1(x, out)
                packed = out.cpu().numpy()
                codes = np.empty(n, np.uint8)
                codes[0::2] = packed & 0xF        # element 2j: low nibble
                codes[1::2] = packed >> 4
                total_runs += _check_runs(start, codes, oracle.e2m1_encode_array)
            del bits, x, out
            start += n
    assert total_runs > 0


@pytest.mark.parametrize("fmt", ["e4m3", "e2m1"])
def test_encoder_infinities(fmt):
    x = torch.tensor([float("inf"), float("-inf")], dtype=torch.float32, device=DEV)
    v = x.cpu().numpy()
    if fmt == "e4m3":
        out = torch.empty(2, dtype=torch.uint8, device=DEV)
        nv.nvfp4_convert_e4m3(x, out)
        assert list(out.cpu().numpy()) == list(oracle.e4m3_encode_array(v))
    else:
        out = torch.empty(1, dtype=torch.uint8, device=DEV)
        nv.nvfp4_convert_e2m1(x, out)
        ref = oracle.e2m1_encode_array(v)
        assert int(out.item()) == int(ref[0]) | (int(ref[1]) << 4)
