"""Persistent multi-tile GEMM paths at the stated FP32 tolerance, on all rows.

The prefill-shaped kernel runs persistent CTA pairs (one pair per two SMs)
over 256 x 256 output tiles.  A pair that computes more than one tile
exercises paths that a one-tile-per-pair launch never reaches: the second
accumulator buffer (which overlaps the first in TMEM), the drain order of
the shared 64-column slots, the early hand-back of the accumulator to the
pair's MMA warp, the ring of TMEM scale regions across tile boundaries, and
(M > 8192) a last raster group with fewer than 32 pair rows (8192
activation rows).  Each case below runs through the C-ABI and is compared
element by element with the FP64 oracle: normwise max relative error <= 1e-3
and relative Frobenius error <= 1e-5 in FP32 output mode, and the BF16
output is bitwise the BF16 rounding of the FP32 output [picx.dev summary,
"Background": native 4-bit tensor-core GEMMs; anthology record LIT-800,
"Standing in the anthology": per-segment scales of a fused projection]."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_10_b200 as nv
import oracle
import synth
from tests.gpu_helpers import (DEV, assert_gemm_close, check_device_error_word, gpu_gemm, oracle_quantize,
                               to_dev_operand)

pytestmark = pytest.mark.gpu

# (M, N, K):
#   4096 x 4096 x 256  - 16 x 16 = 256 pair tiles on 74 pairs: 3-4 tiles per pair
#   8392 x 512 x 256   - 33 pair rows: the raster's second group holds 1
#   2048 x 4103 x 160  - 8 x 17 = 136 pair tiles (about 2 per pair), ragged N
#                        (odd, so no TMA store for f32 rows) and a K tail of
#                        half a 64-block
MULTI_TILE = [(4096, 4096, 256), (8192 + 200, 512, 256), (2048, 4103, 160)]


def _operands(M, N, K, seed):
    a = synth.student_t_outliers(M, K, seed=seed, dtype=torch.float32).numpy()
    w = synth.normal((N, K), seed=seed + 1, std=0.02).numpy()
    return oracle_quantize(a), oracle_quantize(w)


@pytest.mark.parametrize("M,N,K", MULTI_TILE)
def test_gemm_multi_tile_all_rows(M, N, K):
    (ac, asc, ga), (wc, wsc, gw) = _operands(M, N, K, seed=M + 3 * N + K)
    ref = oracle.gemm(ac, asc, ga, wc, wsc, gw)
    a_d, as_d = to_dev_operand(ac, asc, K)
    w_d, ws_d = to_dev_operand(wc, wsc, K)
    out32 = gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, M, N, K, torch.float32)
    out16 = gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, M, N, K, torch.bfloat16)
    torch.cuda.synchronize()
    check_device_error_word()
    assert_gemm_close(out32.cpu().numpy(), ref, f"{M}x{N}x{K}")
    assert torch.equal(out16, out32.to(torch.bfloat16))


# segment boundaries that fall inside 64-column output slots (offsets not
# multiples of 64), on the multi-tile shapes above
FUSED_MULTI = [(4096, 256, (2000, 1000, 1048, 48)), (8192 + 200, 256, (200, 100, 164, 48))]


@pytest.mark.parametrize("M,K,segs", FUSED_MULTI)
def test_fused_multi_tile_all_rows(M, K, segs):
    a = synth.student_t_outliers(M, K, seed=M + K, dtype=torch.float32).numpy()
    ac, asc, ga = oracle_quantize(a)
    sig = (0.02, 0.02 / 4, 0.02 / 16, 0.02 / 64)
    parts, gs = [], []
    for i, n in enumerate(segs):
        w = synth.normal((n, K), seed=M + 100 + i, std=sig[i]).numpy()
        wc, wsc, gw = oracle_quantize(w)
        parts.append((wc, wsc))
        gs.append(gw)
    offs = np.cumsum([0] + list(segs)).astype(np.int64)
    gs = np.array(gs, np.float32)
    wc = np.concatenate([p[0] for p in parts])
    wsc = np.concatenate([p[1] for p in parts])
    assert any(o % 64 for o in offs[1:-1])
    ref = oracle.fused_proj(ac, asc, ga, wc, wsc, offs, gs)
    a_d, as_d = to_dev_operand(ac, asc, K)
    w_d, ws_d = to_dev_operand(wc, wsc, K)
    N = int(offs[-1])
    out32 = torch.empty(M, N, dtype=torch.float32, device=DEV)
    out16 = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    nv.nvfp4_fused_proj(a_d, as_d, float(ga), w_d, ws_d, offs, gs, M, K, out32)
    nv.nvfp4_fused_proj(a_d, as_d, float(ga), w_d, ws_d, offs, gs, M, K, out16)
    torch.cuda.synchronize()
    check_device_error_word()
    f = out32.cpu().numpy()
    for i in range(len(segs)):
        sl = slice(offs[i], offs[i + 1])
        assert_gemm_close(f[:, sl], ref[:, sl], f"{M}x{K} segment {i}")
    assert torch.equal(out16, out32.to(torch.bfloat16))
    # each segment bitwise equal to the plain GEMM on that segment alone
    for i, ((c, s), g) in enumerate(zip(parts, gs)):
        cd, sd = to_dev_operand(c, s, K)
        alone = gpu_gemm(a_d, as_d, ga, cd, sd, g, M, c.shape[0], K, torch.float32)
        torch.cuda.synchronize()
        assert torch.equal(out32[:, offs[i]:offs[i + 1]], alone), f"segment {i}"


@pytest.mark.parametrize("M,N,K", MULTI_TILE)
def test_mx_gemm_multi_tile_all_rows(M, N, K):
    a = synth.student_t_outliers(M, K, seed=M + N, dtype=torch.float32).numpy()
    w = synth.normal((N, K), seed=M + N + 1, std=0.02).numpy()
    ac, asc = oracle.mx_quantize(a)
    wc, wsc = oracle.mx_quantize(w)
    ref = oracle.mx_gemm(ac, asc, wc, wsc)
    a_d = torch.from_numpy(ac).to(DEV)
    as_d = torch.from_numpy(oracle.mx_scales_to_tc(asc, K)).to(DEV)
    w_d = torch.from_numpy(wc).to(DEV)
    ws_d = torch.from_numpy(oracle.mx_scales_to_tc(wsc, K)).to(DEV)
    out32 = torch.empty(M, N, dtype=torch.float32, device=DEV)
    out16 = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    nv.nvfp4_mx_gemm(a_d, as_d, w_d, ws_d, M, N, K, out32)
    nv.nvfp4_mx_gemm(a_d, as_d, w_d, ws_d, M, N, K, out16)
    torch.cuda.synchronize()
    check_device_error_word()
    assert_gemm_close(out32.cpu().numpy(), ref, f"mx {M}x{N}x{K}")
    assert torch.equal(out16, out32.to(torch.bfloat16))
