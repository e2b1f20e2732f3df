"""Failure detection without a GPU fault: a kernel's bounded wait runs out on
a barrier that nothing arrives on, the kernel records NVFP4_ERR_TIMEOUT and
returns, the host reads the status, and the context keeps working."""
import pytest
import torch

import nvfp4_w4a4_quantized_10_b200 as nv
from tests.gpu_helpers import DEV, gpu_quantize

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    assert nv.nvfp4_last_device_error() == nv.OK
    nv.nvfp4_test_wait_timeout(1_000_000, DEV)          # 1 ms
    assert nv.nvfp4_last_device_error() == nv.ERR_TIMEOUT
    assert nv.nvfp4_last_device_error() == nv.OK         # the word is cleared on read
    x = torch.randn(64, 256, device=DEV).to(torch.bfloat16)
    codes, scales, _ = gpu_quantize(x, 100.0)
    torch.cuda.synchronize()
    assert codes.shape == (64, 128)


def test_wait_timeout_setting_round_trips():
    nv.nvfp4_set_wait_timeout_ns(500_000_000)
    nv.nvfp4_set_wait_timeout_ns(0)                       # back to the default
    x = torch.randn(16, 256, device=DEV).to(torch.bfloat16)
    gpu_quantize(x, 50.0)
    torch.cuda.synchronize()
    assert nv.nvfp4_last_device_error() == nv.OK


def test_error_read_back_clears_gemm_scratch_and_gemm_still_agrees():
    # reading back a device error also empties the decode GEMM's K-split
    # scratch (library workspaces and the allocation-free array); GEMMs on
    # both paths (the same kernel, K split and summation order) must give the
    # same result before and after
    M, N, K = 8, 4096, 5120
    x = torch.randn(M, K, device=DEV).to(torch.bfloat16)
    w = (0.02 * torch.randn(N, K, device=DEV)).to(torch.bfloat16)
    ac, asc, _ = gpu_quantize(x, 300.0)
    wc, wsc, _ = gpu_quantize(w, 20000.0)
    outs = []
    for _ in range(2):
        o1 = torch.empty(M, N, dtype=torch.float32, device=DEV)
        o2 = torch.empty(M, N, dtype=torch.float32, device=DEV)
        nv.nvfp4_gemm(ac, asc, 300.0, wc, wsc, 20000.0, M, N, K, o1)
        nv.nvfp4_gemm_noalloc(ac, asc, 300.0, wc, wsc, 20000.0, M, N, K, o2)
        assert nv.nvfp4_last_device_error() == nv.OK
        outs += [o1, o2]
        nv.nvfp4_test_wait_timeout(1_000_000, DEV)
        assert nv.nvfp4_last_device_error() == nv.ERR_TIMEOUT
    assert all(torch.equal(o, outs[0]) for o in outs[1:])


def _decode_operands(M, N, K, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16).to(DEV)
    w = (0.02 * torch.randn(N, K, generator=g)).to(torch.bfloat16).to(DEV)
    ac, asc, _ = gpu_quantize(x, 300.0)
    wc, wsc, _ = gpu_quantize(w, 20000.0)
    return ac, asc, wc, wsc


def test_timed_out_split_k_reduction_leaves_no_stale_partials():
    # a decode GEMM whose split-tile adders never see their helpers'
    # partials: the bounded wait runs out, the launch reports a timeout and
    # the helpers' partial words stay full.  Reading the error back empties
    # the scratch, so the next GEMMs on it give the reference result.  The
    # stalled launch uses other operands, so a stale word that survived would
    # be the wrong value.
    M, N, K = 8, 4096, 5120
    ac, asc, wc, wsc = _decode_operands(M, N, K, seed=31)
    bc, bsc, vc, vsc = _decode_operands(M, N, K, seed=32)
    ref = torch.empty(M, N, dtype=torch.float32, device=DEV)
    nv.nvfp4_gemm(ac, asc, 300.0, wc, wsc, 20000.0, M, N, K, ref)
    torch.cuda.synchronize()
    assert nv.nvfp4_last_device_error() == nv.OK
    junk = torch.empty(M, N, dtype=torch.float32, device=DEV)
    nv.nvfp4_set_wait_timeout_ns(1_000_000)                 # 1 ms
    try:
        nv.nvfp4_test_gemm_stalled_reduction(bc, bsc, 300.0, vc, vsc, 20000.0, M, N, K, junk)
        st = nv.nvfp4_last_device_error()
    finally:
        nv.nvfp4_set_wait_timeout_ns(0)
    assert st == nv.ERR_TIMEOUT
    for _ in range(2):
        o = torch.full((M, N), float("nan"), dtype=torch.float32, device=DEV)
        nv.nvfp4_gemm(ac, asc, 300.0, wc, wsc, 20000.0, M, N, K, o)
        torch.cuda.synchronize()
        assert torch.equal(o, ref)
    assert nv.nvfp4_last_device_error() == nv.OK
