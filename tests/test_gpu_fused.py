"""Fused projection on the GPU: several separately calibrated weight segments
in one GEMM, each output segment rescaled by its own global scale
[anthology record LIT-800, "Standing in the anthology"; cctest.ai article,
"Main findings"].  Checks: oracle parity, bitwise fused == unfused per
segment, and the shared-scale failure mode as a negative control."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_10_b200 as nv
import oracle
import synth
from tests.gpu_helpers import (DEV, assert_gemm_close, check_device_error_word, gpu_quantize, oracle_quantize,
                               rel_errors, to_dev_operand)

pytestmark = pytest.mark.gpu


def _case(M, K, segs, sig, seed=0):
    a = synth.student_t_outliers(M, K, seed=seed, dtype=torch.float32).numpy()
    ac, asc, ga = oracle_quantize(a)
    parts, gs = [], []
    for i, (n, sd) in enumerate(zip(segs, sig)):
        w = synth.normal((n, K), seed=seed + 100 + i, std=sd).numpy()
        wc, wsc, gw = oracle_quantize(w)
        parts.append((wc, wsc))
        gs.append(gw)
    offs = np.cumsum([0] + list(segs)).astype(np.int64)
    wc = np.concatenate([p[0] for p in parts])
    wsc = np.concatenate([p[1] for p in parts])
    return ac, asc, ga, wc, wsc, offs, np.array(gs, np.float32), parts


def _fused_gpu(a_d, as_d, ga, w_d, ws_d, offs, gs, M, K, dtype=torch.float32):
    out = torch.empty(M, int(offs[-1]), dtype=dtype, device=DEV)
    nv.nvfp4_fused_proj(a_d, as_d, float(ga), w_d, ws_d, offs, gs, M, K, out)
    return out


def _unfused_gpu(a_d, as_d, ga, parts, gs, M, K, dtype=torch.float32):
    outs = []
    for (wc, wsc), g in zip(parts, gs):
        w_d, ws_d = to_dev_operand(wc, wsc, K)
        o = torch.empty(M, wc.shape[0], dtype=dtype, device=DEV)
        nv.nvfp4_gemm(a_d, as_d, float(ga), w_d, ws_d, float(g), M, wc.shape[0], K, o)
        outs.append(o)
    return outs


GDN_SIG = (0.02, 0.02 / 4, 0.02 / 16, 0.02 / 64)


@pytest.mark.parametrize("M,K,segs", [(200, 512, (256, 128, 48, 48)), (64, 1024, (96, 40, 8, 24)),
                                      (300, 320, (8, 8, 8)), (130, 5120, (512, 256, 48, 48))])
def test_fused_matches_oracle_and_unfused(M, K, segs):
    sig = (GDN_SIG * 4)[:len(segs)]
    ac, asc, ga, wc, wsc, offs, gs, parts = _case(M, K, segs, sig, seed=M + K)
    ref = oracle.fused_proj(ac, asc, ga, wc, wsc, offs, gs)
    a_d, as_d = to_dev_operand(ac, asc, K)
    w_d, ws_d = to_dev_operand(wc, wsc, K)
    for dtype in (torch.float32, torch.bfloat16):
        fused = _fused_gpu(a_d, as_d, ga, w_d, ws_d, offs, gs, M, K, dtype)
        alone = _unfused_gpu(a_d, as_d, ga, parts, gs, M, K, dtype)
        for i, o in enumerate(alone):
            assert torch.equal(fused[:, offs[i]:offs[i + 1]], o), f"segment {i}"
        if dtype == torch.float32:
            f = fused.cpu().numpy()
            for i in range(len(segs)):
                sl = slice(offs[i], offs[i + 1])
                assert_gemm_close(f[:, sl], ref[:, sl], f"segment {i}")
    check_device_error_word()


def test_shared_scale_negative_control():
    # one shared weight scale (the first module's) for every segment: the gate
    # segments come out scaled by g_i / g_0 and fail the tolerance by far
    M, K = 128, 1024
    ac, asc, ga, wc, wsc, offs, gs, parts = _case(M, K, (256, 128, 48, 48), GDN_SIG, seed=3)
    ref = oracle.fused_proj(ac, asc, ga, wc, wsc, offs, gs)
    a_d, as_d = to_dev_operand(ac, asc, K)
    w_d, ws_d = to_dev_operand(wc, wsc, K)
    bad = _fused_gpu(a_d, as_d, ga, w_d, ws_d, offs, np.full_like(gs, gs[0]), M, K).cpu().numpy()
    for i in (2, 3):
        sl = slice(offs[i], offs[i + 1])
        max_rel, frob = rel_errors(bad[:, sl], ref[:, sl])
        assert frob > 1.0, (i, frob)


def test_fused_gdn_full_size():
    # the fused GDN workload: X[4096, 5120], segments 8192/4096/48/48 with
    # their own scales; oracle on sampled rows, fused == unfused on all rows
    w = synth.FUSED_GDN
    x = synth.activation(w, device=DEV)
    wt = synth.weight(w, device=DEV)
    offs = np.array(synth.segment_offsets(w), np.int64)
    ga = oracle.global_scale(oracle.amax(x.float().cpu().numpy()))
    wt_cpu = wt.float().cpu().numpy()
    gs = np.array([oracle.global_scale(oracle.amax(wt_cpu[offs[i]:offs[i + 1]])) for i in range(4)], np.float32)
    assert gs.max() / gs.min() > 16        # the segment scales span more than 16x
    a_codes, a_sc, _ = gpu_quantize(x, ga)
    w_codes = torch.empty(w.N, w.K // 2, dtype=torch.uint8, device=DEV)
    w_parts = []
    for i in range(4):
        c, s, _ = gpu_quantize(wt[offs[i]:offs[i + 1]].contiguous(), gs[i], nv.SF_ROWMAJOR)
        w_codes[offs[i]:offs[i + 1]] = c
        w_parts.append(s.view(-1, w.K // 16))
    w_rm = torch.cat(w_parts)
    w_sc = torch.empty(nv.nvfp4_scale_bytes(w.N, w.K), dtype=torch.uint8, device=DEV)
    nv.nvfp4_swizzle_scales(w_rm.contiguous(), w.N, w.K, w_sc)
    fused = torch.empty(w.M, w.N, dtype=torch.bfloat16, device=DEV)
    nv.nvfp4_fused_proj(a_codes, a_sc, float(ga), w_codes, w_sc, offs, gs, w.M, w.K, fused)
    fused32 = torch.empty(w.M, w.N, dtype=torch.float32, device=DEV)
    nv.nvfp4_fused_proj(a_codes, a_sc, float(ga), w_codes, w_sc, offs, gs, w.M, w.K, fused32)
    torch.cuda.synchronize()
    assert torch.equal(fused, fused32.to(torch.bfloat16))
    for i in range(4):
        n = int(offs[i + 1] - offs[i])
        sc = torch.empty(nv.nvfp4_scale_bytes(n, w.K), dtype=torch.uint8, device=DEV)
        nv.nvfp4_swizzle_scales(w_parts[i].contiguous(), n, w.K, sc)
        alone = torch.empty(w.M, n, dtype=torch.bfloat16, device=DEV)
        nv.nvfp4_gemm(a_codes, a_sc, float(ga), w_codes[offs[i]:offs[i + 1]].contiguous(), sc, float(gs[i]),
                      w.M, n, w.K, alone)
        assert torch.equal(fused[:, offs[i]:offs[i + 1]], alone), f"segment {i}"
    rows = synth.sample_rows(w.M, 16)
    ac, asc, _ = oracle_quantize(x[rows].float().cpu().numpy(), ga)
    wc_list, wsc_list = [], []
    for i in range(4):
        c, s, _ = oracle_quantize(wt_cpu[offs[i]:offs[i + 1]], gs[i])
        wc_list.append(c)
        wsc_list.append(s)
    ref = oracle.fused_proj(ac, asc, ga, np.concatenate(wc_list), np.concatenate(wsc_list), offs, gs)
    # the full launch (1,568 tiles on the persistent grid) in FP32 output
    # mode, at the stated tolerance on the sampled rows, segment by segment
    got = fused32[rows].cpu().numpy()
    for i in range(4):
        sl = slice(offs[i], offs[i + 1])
        assert_gemm_close(got[:, sl], ref[:, sl], f"GDN segment {i}")
    check_device_error_word()
