"""Ownership of the decode GEMM's K-split workspace through the C-ABI.

A decode-shaped GEMM (M <= 128) splits each weight tile's K loop over the
CTAs and exchanges partial tiles through a per-stream workspace.  The caller
may register its own (zero-filled) workspace for a stream; the library then
allocates nothing for that stream, the call can be the first one on a stream
that is being captured into a CUDA graph, and every launch leaves the
workspace zero again.  Library-allocated workspaces are freed by
nvfp4_release_workspaces.  Results do not depend on which workspace is used:
they are bitwise equal to the default path and within the FP32 tolerance of
the oracle [picx.dev summary, "Background": native 4-bit tensor-core GEMMs]."""
import ctypes

import pytest
import torch

import nvfp4_w4a4_quantized_10_b200 as nv
import oracle
import synth
from tests.gpu_helpers import DEV, assert_gemm_close, check_device_error_word, oracle_quantize, to_dev_operand

pytestmark = pytest.mark.gpu


def _problem(M, N, K, seed):
    a = synth.student_t_outliers(M, K, seed=seed, dtype=torch.float32).numpy()
    w = synth.normal((N, K), seed=seed + 1, std=0.02).numpy()
    (ac, asc, ga), (wc, wsc, gw) = oracle_quantize(a), oracle_quantize(w)
    a_d, as_d = to_dev_operand(ac, asc, K)
    w_d, ws_d = to_dev_operand(wc, wsc, K)
    return (ac, asc, ga, wc, wsc, gw), (a_d, as_d, float(ga), w_d, ws_d, float(gw))


def test_workspace_bytes_rule():
    sm = torch.cuda.get_device_properties(0).multi_processor_count
    # two slots of bn x 128 words per CTA; the bn = 16 grid has two CTAs per SM
    for M, bn in ((1, 16), (16, 16), (17, 32), (32, 32), (33, 64), (64, 64), (65, 128), (128, 128)):
        ctas = 2 * sm if bn == 16 else sm
        assert nv.nvfp4_workspace_bytes(M, 4096, 1024) == 2 * ctas * bn * 128 * 8, M
    assert nv.nvfp4_workspace_bytes(129, 4096, 1024) == 0
    assert nv.nvfp4_workspace_bytes(0, 4096, 1024) == 0
    assert nv.nvfp4_workspace_bytes(8, 4096, 48) == 0


@pytest.mark.parametrize("M,N,K", [(8, 12288, 5120), (16, 4097, 1024), (64, 1000, 2048), (128, 3000, 768)])
def test_registered_workspace_matches_default(M, N, K):
    host, dev = _problem(M, N, K, seed=M + N)
    ref = oracle.gemm(*host)
    default = torch.empty(M, N, dtype=torch.float32, device=DEV)
    nv.nvfp4_gemm(*dev, M, N, K, default)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    ws = torch.zeros(nv.nvfp4_workspace_bytes(M, N, K), dtype=torch.uint8, device=DEV)
    nv.nvfp4_set_workspace(ws, stream=s)
    try:
        out = torch.empty(M, N, dtype=torch.float32, device=DEV)
        out2 = torch.empty_like(out)
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        with torch.cuda.stream(s):
            nv.nvfp4_gemm(*dev, M, N, K, out)
            nv.nvfp4_gemm(*dev, M, N, K, out2)
        s.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        check_device_error_word()
        assert free1 >= free0 - (1 << 20), (free0, free1)   # the library allocated nothing for this stream
        assert torch.equal(out, default) and torch.equal(out2, default)
        assert int(torch.count_nonzero(ws)) == 0      # every word left empty
        assert_gemm_close(out.cpu().numpy(), ref, f"{M}x{N}x{K}")
    finally:
        nv.nvfp4_set_workspace(None, stream=s)


def test_registered_workspace_too_small():
    M, N, K = 64, 512, 1024
    _, dev = _problem(M, N, K, seed=2)
    s = torch.cuda.Stream()
    ws = torch.zeros(nv.nvfp4_workspace_bytes(16, N, K), dtype=torch.uint8, device=DEV)
    nv.nvfp4_set_workspace(ws, stream=s)
    try:
        out = torch.empty(M, N, dtype=torch.float32, device=DEV)
        st = nv._lib.nvfp4_gemm(nv._ptr(dev[0]), nv._ptr(dev[1]), dev[2], nv._ptr(dev[3]), nv._ptr(dev[4]), dev[5],
                                M, N, K, nv._ptr(out), nv.OUT_F32, ctypes.c_void_p(s.cuda_stream))
        assert st == nv.ERR_INVALID_ARG
        # the 16-row tile fits
        with torch.cuda.stream(s):
            small = torch.empty(16, N, dtype=torch.float32, device=DEV)
            nv.nvfp4_gemm(dev[0][:16], dev[1], dev[2], *dev[3:], 16, N, K, small)
        s.synchronize()
        check_device_error_word()
    finally:
        nv.nvfp4_set_workspace(None, stream=s)


def test_set_workspace_rejects_bad_arguments():
    s = torch.cuda.Stream()
    sv = ctypes.c_void_p(s.cuda_stream)
    ws = torch.zeros(nv.nvfp4_workspace_bytes(16, 1, 32) + 64, dtype=torch.uint8, device=DEV)
    assert nv._lib.nvfp4_set_workspace(sv, None, 16) == nv.ERR_INVALID_ARG
    assert nv._lib.nvfp4_set_workspace(sv, ctypes.c_void_p(ws.data_ptr() + 8), 1 << 20) == nv.ERR_ALIGNMENT
    assert nv._lib.nvfp4_set_workspace(sv, nv._ptr(ws), 1024) == nv.ERR_INVALID_ARG
    assert nv._lib.nvfp4_set_workspace(sv, None, 0) == nv.OK


def test_first_call_inside_capture_with_registered_workspace():
    M, N, K = 8, 4096, 2048
    host, dev = _problem(M, N, K, seed=11)
    ref = oracle.gemm(*host)
    warm = torch.empty(M, N, dtype=torch.float32, device=DEV)
    nv.nvfp4_gemm(*dev, M, N, K, warm)          # kernel attributes set outside the capture (default stream)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    ws = torch.zeros(nv.nvfp4_workspace_bytes(M, N, K), dtype=torch.uint8, device=DEV)
    nv.nvfp4_set_workspace(ws, stream=s)
    try:
        out = torch.zeros(M, N, dtype=torch.float32, device=DEV)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            nv.nvfp4_gemm(*dev, M, N, K, out)     # the first call ever made on this stream
        for _ in range(3):
            out.zero_()
            g.replay()
        torch.cuda.synchronize()
        check_device_error_word()
        assert_gemm_close(out.cpu().numpy(), ref, "captured")
        assert int(torch.count_nonzero(ws)) == 0
        del g
    finally:
        nv.nvfp4_set_workspace(None, stream=s)


def test_first_call_inside_capture_without_workspace_is_unsupported():
    M, N, K = 8, 1024, 1024
    _, dev = _problem(M, N, K, seed=12)
    s = torch.cuda.Stream()
    out = torch.zeros(M, N, dtype=torch.float32, device=DEV)
    g = torch.cuda.CUDAGraph()
    status = []
    with torch.cuda.graph(g, stream=s):
        status.append(nv._lib.nvfp4_gemm(nv._ptr(dev[0]), nv._ptr(dev[1]), dev[2], nv._ptr(dev[3]), nv._ptr(dev[4]),
                                         dev[5], M, N, K, nv._ptr(out), nv.OUT_F32, ctypes.c_void_p(s.cuda_stream)))
    del g
    torch.cuda.synchronize()
    assert status == [nv.ERR_UNSUPPORTED]


def test_release_workspaces_then_reallocate():
    M, N, K = 16, 2048, 1024
    host, dev = _problem(M, N, K, seed=13)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        first = torch.empty(M, N, dtype=torch.float32, device=DEV)
        nv.nvfp4_gemm(*dev, M, N, K, first)      # the library allocates this stream's workspace
    s.synchronize()
    nv.nvfp4_release_workspaces()                   # frees it (and every other library-allocated one)
    with torch.cuda.stream(s):
        second = torch.empty_like(first)
        nv.nvfp4_gemm(*dev, M, N, K, second)     # allocates again
    s.synchronize()
    check_device_error_word()
    assert torch.equal(first, second)
    assert_gemm_close(second.cpu().numpy(), oracle.gemm(*host), "after release")
