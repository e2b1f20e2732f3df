"""Decode-shaped GEMMs (at most 16 activation rows) through the C-ABI.

These run the swapped-operand path: the weight is the 128-row MMA operand,
the K loop of each weight tile is split over the CTAs of the grid
(stream-K) and the partial tiles are summed in a fixed order.  Compared
element by element with the FP64 oracle at the stated FP32 tolerance
(normwise max relative error <= 1e-3, relative Frobenius error <= 1e-5);
the BF16 output is bitwise the BF16 rounding of the FP32 output, and
repeated calls are bitwise equal [picx.dev summary, "Background": native
4-bit tensor-core GEMMs; anthology record LIT-800, "Standing in the
anthology": per-segment scales of a fused projection]."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_10_b200 as nv
import oracle
import synth
from tests.gpu_helpers import (DEV, TOL_FROB, TOL_MAX_REL, assert_gemm_close, check_device_error_word, gpu_gemm,
                               oracle_quantize, rel_errors, to_dev_operand)

pytestmark = pytest.mark.gpu

# (M, N, K): one K step and one tile; the decode workload and its 16-row
# variant; ragged N (odd column counts); a long K split over many CTAs; a K
# tail of one 64-block; one row.
SHAPES = [(1, 48, 32), (8, 12288, 5120), (16, 12288, 5120), (9, 4100, 2048), (5, 1000, 17408),
          (13, 257, 320), (2, 2048, 160), (16, 4097, 1024), (1, 12288, 5120)]


def _operands(M, N, K, seed):
    a = synth.student_t_outliers(M, K, seed=seed, dtype=torch.float32).numpy()
    w = synth.normal((N, K), seed=seed + 1, std=0.02).numpy()
    return oracle_quantize(a), oracle_quantize(w)


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_decode_matches_oracle(M, N, K):
    (ac, asc, ga), (wc, wsc, gw) = _operands(M, N, K, seed=3 * M + N + K)
    ref = oracle.gemm(ac, asc, ga, wc, wsc, gw)
    a_d, as_d = to_dev_operand(ac, asc, K)
    w_d, ws_d = to_dev_operand(wc, wsc, K)
    out32 = gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, M, N, K, torch.float32)
    again = gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, M, N, K, torch.float32)
    out16 = gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, M, N, K, torch.bfloat16)
    torch.cuda.synchronize()
    check_device_error_word()
    assert_gemm_close(out32.cpu().numpy(), ref, f"{M}x{N}x{K}")
    assert torch.equal(out32, again)
    assert torch.equal(out16, out32.to(torch.bfloat16))


def test_decode_guard_bands():
    # the K-split adders write exactly the [M, N] output
    M, N, K = 7, 1000, 2048
    (ac, asc, ga), (wc, wsc, gw) = _operands(M, N, K, seed=5)
    a_d, as_d = to_dev_operand(ac, asc, K)
    w_d, ws_d = to_dev_operand(wc, wsc, K)
    pad = 4096
    for dtype in (torch.float32, torch.bfloat16):
        buf = torch.full((pad + M * N + pad,), -7.0, dtype=dtype, device=DEV)
        out = buf[pad:pad + M * N].view(M, N)
        nv.nvfp4_gemm(a_d, as_d, float(ga), w_d, ws_d, float(gw), M, N, K, out)
        torch.cuda.synchronize()
        assert torch.all(buf[:pad] == -7.0) and torch.all(buf[pad + M * N:] == -7.0)
    check_device_error_word()


@pytest.mark.parametrize("M,K,segs", [(8, 1024, (256, 100, 48, 48)), (16, 5120, (8192, 4096, 48, 48)),
                                      (3, 320, (40, 8, 200))])
def test_decode_fused_projection(M, K, segs):
    a = synth.student_t_outliers(M, K, seed=M + K, dtype=torch.float32).numpy()
    ac, asc, ga = oracle_quantize(a)
    sig = (0.02, 0.02 / 4, 0.02 / 16, 0.02 / 64)
    parts, gs = [], []
    for i, n in enumerate(segs):
        w = synth.normal((n, K), seed=M + 50 + i, std=sig[i]).numpy()
        c, s_, g = oracle_quantize(w)
        parts.append((c, s_))
        gs.append(g)
    offs = np.cumsum([0] + list(segs)).astype(np.int64)
    gs = np.array(gs, np.float32)
    wc = np.concatenate([p[0] for p in parts])
    wsc = np.concatenate([p[1] for p in parts])
    ref = oracle.fused_proj(ac, asc, ga, wc, wsc, offs, gs)
    a_d, as_d = to_dev_operand(ac, asc, K)
    w_d, ws_d = to_dev_operand(wc, wsc, K)
    out = torch.empty(M, int(offs[-1]), dtype=torch.float32, device=DEV)
    nv.nvfp4_fused_proj(a_d, as_d, float(ga), w_d, ws_d, offs, gs, M, K, out)
    torch.cuda.synchronize()
    check_device_error_word()
    f = out.cpu().numpy()
    for i in range(len(segs)):
        sl = slice(offs[i], offs[i + 1])
        assert_gemm_close(f[:, sl], ref[:, sl], f"segment {i}")
        # the unfused GEMM of the segment: equal up to the FP32 summation
        # order of the K split, which depends on the number of weight tiles
        cd, sd = to_dev_operand(*parts[i], K)
        alone = gpu_gemm(a_d, as_d, ga, cd, sd, gs[i], M, parts[i][0].shape[0], K, torch.float32)
        torch.cuda.synchronize()
        max_rel, frob = rel_errors(f[:, sl], alone.double().cpu().numpy())
        assert max_rel <= TOL_MAX_REL and frob <= TOL_FROB, (i, max_rel, frob)


@pytest.mark.parametrize("M,N,K", [(8, 12288, 5120), (3, 500, 1024), (16, 300, 17408)])
def test_decode_mxfp4(M, N, K):
    a = synth.student_t_outliers(M, K, seed=M * 5 + K, dtype=torch.float32).numpy()
    w = synth.normal((N, K), seed=N, std=0.02).numpy()
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


@pytest.mark.parametrize("M,N,K", [(8, 12288, 5120), (16, 4097, 1024), (24, 3000, 5120), (64, 1000, 2048),
                                   (128, 3000, 768)])
def test_decode_cooperative_launch(M, N, K):
    # The opt-in co-residency guarantee launches the split-K grid
    # cooperatively, sized to what the occupancy API admits per SM.  Where
    # that is the default grid (M > 16) the result is bitwise the default's;
    # for M <= 16 the default grid has two CTAs per SM, more than are
    # resident at once, so the cooperative grid can split K differently:
    # the same sum up to FP32 rounding order.
    (ac, asc, ga), (wc, wsc, gw) = _operands(M, N, K, seed=7 * M + K)
    a_d, as_d = to_dev_operand(ac, asc, K)
    w_d, ws_d = to_dev_operand(wc, wsc, K)
    default = gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, M, N, K, torch.float32)
    torch.cuda.synchronize()
    nv.nvfp4_set_decode_cooperative(True)
    try:
        coop = gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, M, N, K, torch.float32)
        again = gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, M, N, K, torch.float32)
        if M <= 32:
            noalloc = torch.empty(M, N, dtype=torch.float32, device=DEV)
            nv.nvfp4_gemm_noalloc(a_d, as_d, float(ga), w_d, ws_d, float(gw), M, N, K, noalloc)
        torch.cuda.synchronize()
    finally:
        nv.nvfp4_set_decode_cooperative(False)
    check_device_error_word()
    assert torch.equal(coop, again)
    if M <= 32:
        assert torch.equal(noalloc, coop)          # the same cooperative grid
    assert_gemm_close(coop.cpu().numpy(), oracle.gemm(ac, asc, ga, wc, wsc, gw), f"cooperative {M}x{N}x{K}")
    if M > 16:
        assert torch.equal(coop, default)
    else:
        max_rel, frob = rel_errors(coop.double().cpu().numpy(), default.double().cpu().numpy())
        assert max_rel <= TOL_MAX_REL and frob <= TOL_FROB, (max_rel, frob)


@pytest.mark.parametrize("M,N,K", [(8, 12288, 5120), (16, 2048, 4096), (4, 700, 17408)])
def test_back_to_back_decode_calls_on_one_stream(M, N, K):
    # Consecutive split-K GEMMs on one stream share its workspace and overlap
    # under programmatic dependent launch: each must see only its own
    # partials.  Different weights per call make a partial taken from the
    # wrong launch visible in the result.
    (ac, asc, ga), _ = _operands(M, N, K, seed=M + 2 * K)
    a_d, as_d = to_dev_operand(ac, asc, K)
    ws = []
    for i in range(4):
        wc, wsc, gw = oracle_quantize(synth.normal((N, K), seed=100 + i, std=0.02 * (i + 1)).numpy())
        ws.append((*to_dev_operand(wc, wsc, K), gw))
    refs = []
    for w_d, ws_d, gw in ws:
        refs.append(gpu_gemm(a_d, as_d, ga, w_d, ws_d, gw, M, N, K, torch.float32))
        torch.cuda.synchronize()
    outs = [torch.empty(M, N, dtype=torch.float32, device=DEV) for _ in range(24)]
    for i, o in enumerate(outs):
        w_d, ws_d, gw = ws[i % 4]
        nv.nvfp4_gemm(a_d, as_d, float(ga), w_d, ws_d, float(gw), M, N, K, o)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    gouts = [torch.empty(M, N, dtype=torch.float32, device=DEV) for _ in range(24)]
    with torch.cuda.stream(s):                     # this stream's workspace, before the capture
        nv.nvfp4_gemm(a_d, as_d, float(ga), ws[0][0], ws[0][1], float(ws[0][2]), M, N, K, gouts[0])
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        for i, o in enumerate(gouts):
            w_d, ws_d, gw = ws[i % 4]
            nv.nvfp4_gemm(a_d, as_d, float(ga), w_d, ws_d, float(gw), M, N, K, o)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    del g
    check_device_error_word()
    for i in range(24):
        assert torch.equal(outs[i], refs[i % 4]), i
        assert torch.equal(gouts[i], refs[i % 4]), i
