"""Pins for the oracle's static-calibration helpers (CPU only).

The recipe on the pages is calibration-only: the activation scale is fixed
from a set of calibration sequences and then serves every later input
[anthology record LIT-800, "Key takeaways"; cctest.ai article,
"Introduction"].  A later input with a larger outlier than any calibration
batch then has blocks whose scale target exceeds the largest E4M3 value.

What fixes the helpers, other than the oracle itself:
  * numpy's max over the concatenated batches, with the largest value placed
    in the first, a middle and the last batch;
  * hand-built blocks whose clipping is known in closed form;
  * invariants of a saturated block: scale byte 0x7E and a largest code of
    magnitude 6.
"""
import numpy as np

import oracle
import synth


def test_calibrated_amax_is_the_max_over_all_batches():
    rng = np.random.default_rng(30)
    for where in (0, 2, 4):
        batches = [rng.standard_normal((3, 32)).astype(np.float32) for _ in range(5)]
        batches[where][1, 7] = -50.0 - where
        assert oracle.calibrate_amax(batches) == np.float32(np.abs(np.concatenate(batches)).max())
        assert oracle.calibrate_amax(batches) == np.float32(50.0 + where)
    assert oracle.calibrate_amax([np.zeros((2, 16), np.float32)]) == 0.0


def test_saturation_counts_on_hand_built_blocks():
    g = np.float32(1.0)
    x = np.zeros((1, 80), np.float32)
    # block 0: amax 5376 -> t = 896 > 448, s = 448, r = 1/448: 5376 and -3000
    # map beyond 6 (12 and 6.7), 2000 maps to 4.46
    x[0, 0:3] = [5376.0, -3000.0, 2000.0]
    # block 1: amax 6 * 2^3 -> t = 8 exactly, the largest element maps to 6.0
    x[0, 16:18] = [48.0, -20.0]
    # block 2: all zero (neither clipped nor underflowed)
    # block 3: amax 1e-6 -> t below half the smallest subnormal, s = 0
    x[0, 48] = 1e-6
    # block 4: all 5 -> t = 5/6 rounds down to 0.8125, so 5 / 0.8125 > 6
    x[0, 64:80] = 5.0
    assert oracle.saturation(x, g) == (1, 2 + 16, 1)
    codes, scales = oracle.quantize(x, g)
    assert list(scales[0]) == [0x7E, 0x50, 0x00, 0x00, 0x35]
    assert codes[0, 0] & 0xF == 0x7 and codes[0, 0] >> 4 == 0xF   # +6, -6


def test_static_scale_clips_the_held_out_batch_only():
    M, K = 1024, 5120   # wide enough for 368x-RMS outlier channels
    cal = [synth.calibration_batch(i, M, K).float().numpy() for i in range(synth.CALIB_BATCHES)]
    held = synth.held_out_batch(M, K).float().numpy()
    g = oracle.global_scale(oracle.calibrate_amax(cal))
    for b in cal:
        assert oracle.saturation(b, g)[0] == 0
    sat_blocks, sat_codes, _ = oracle.saturation(held, g)
    assert sat_blocks > 0 and sat_codes >= sat_blocks
    codes, scales = oracle.quantize(held, g)
    nb = K // 16
    q = np.float32(np.abs(held).reshape(M, nb, 16).max(-1) / np.float32(6.0))
    clipped = q * g > 448
    assert np.array_equal(np.argwhere(scales == 0x7E), np.argwhere(clipped | (scales == 0x7E)))
    lo, hi = codes & 0xF, codes >> 4
    mag = np.maximum(lo & 7, hi & 7).reshape(M, nb, 8).max(-1)
    assert np.all(mag[clipped] == 7)
