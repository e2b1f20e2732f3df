"""nvfp4_gemm_noalloc: the decode GEMM whose K-split scratch is a fixed
static device array instead of a workspace allocated on first use, for
callers that cannot allocate device memory.  It runs the same kernel with
the same work split as nvfp4_gemm, so through the C-ABI it must agree with
nvfp4_gemm within the GEMM tolerance (and in practice bitwise), on two calls
in a row, whether this file runs alone or after the rest of the suite.  The
file name sorts last so that it is collected last."""
import ctypes

import pytest
import torch

import nvfp4_w4a4_quantized_10_b200 as nv

from gpu_helpers import TOL_FROB, TOL_MAX_REL, check_device_error_word, rel_errors


def _operands(M, N, K, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    w = (0.02 * torch.randn(N, K, generator=g)).to(torch.bfloat16).cuda()
    am = torch.empty(1, dtype=torch.float32, device="cuda")
    nv.nvfp4_amax(x, am)
    ga = 2688.0 / am.item()
    nv.nvfp4_amax(w, am)
    gw = 2688.0 / am.item()
    ac, asc = nv.alloc_quantized(M, K, "cuda")
    wc, wsc = nv.alloc_quantized(N, K, "cuda")
    nv.nvfp4_quantize(x, ga, ac, asc)
    nv.nvfp4_quantize(w, gw, wc, wsc)
    return ac, asc, ga, wc, wsc, gw


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K,dtype", [(8, 12288, 5120, torch.bfloat16), (8, 12288, 5120, torch.float32),
                                         (1, 640, 256, torch.float32), (29, 1000, 320, torch.float32),
                                         (32, 4096, 17408, torch.bfloat16)])
def test_noalloc_matches_gemm_two_calls(M, N, K, dtype):
    ac, asc, ga, wc, wsc, gw = _operands(M, N, K, seed=M * 7 + N + K)
    ref32 = torch.empty(M, N, dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm(ac, asc, ga, wc, wsc, gw, M, N, K, ref32)
    o32 = torch.empty(M, N, dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm_noalloc(ac, asc, ga, wc, wsc, gw, M, N, K, o32)
    outs = []
    for _ in range(2):                      # two calls in a row on one stream
        o = torch.full((M, N), float("nan"), dtype=dtype, device="cuda")
        nv.nvfp4_gemm_noalloc(ac, asc, ga, wc, wsc, gw, M, N, K, o)
        outs.append(o)
    torch.cuda.synchronize()
    check_device_error_word()
    # the GEMM tolerance (FP32 output) against nvfp4_gemm
    max_rel, frob = rel_errors(o32.cpu().numpy(), ref32.double().cpu().numpy())
    assert max_rel <= TOL_MAX_REL and frob <= TOL_FROB, (max_rel, frob)
    # both calls: the same fixed summation order, so bitwise the output type's
    # rounding of the FP32 result, and (same kernel, same K split) bitwise
    # nvfp4_gemm's
    ref = torch.empty(M, N, dtype=dtype, device="cuda")
    nv.nvfp4_gemm(ac, asc, ga, wc, wsc, gw, M, N, K, ref)
    torch.cuda.synchronize()
    for o in outs:
        assert torch.equal(o, o32.to(dtype))
        assert torch.equal(o, ref)


@pytest.mark.gpu
def test_noalloc_takes_no_device_memory():
    M, N, K = 8, 12288, 5120
    ac, asc, ga, wc, wsc, gw = _operands(M, N, K, seed=5)
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    nv.nvfp4_gemm_noalloc(ac, asc, ga, wc, wsc, gw, M, N, K, out)   # scratch address resolved
    torch.cuda.synchronize()
    s = torch.cuda.Stream()                 # a stream nvfp4_gemm would give a new workspace
    free0, _ = torch.cuda.mem_get_info()
    with torch.cuda.stream(s):
        for _ in range(2):
            nv.nvfp4_gemm_noalloc(ac, asc, ga, wc, wsc, gw, M, N, K, out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 >= free0 - (1 << 20), (free0, free1)
    check_device_error_word()


@pytest.mark.gpu
def test_noalloc_scratch_is_emptied_after_a_timed_out_launch():
    # A launch whose bounded wait runs out leaves partial words full in the
    # shared static scratch (here: the adders never see their helpers'
    # partials).  Reading the device error back empties the array, so the
    # next calls agree with nvfp4_gemm again.  The stalled launch multiplies
    # other operands, so a stale word that survived would be a wrong value.
    M, N, K = 8, 4096, 5120
    ac, asc, ga, wc, wsc, gw = _operands(M, N, K, seed=41)
    bc, bsc, gb, vc, vsc, gv = _operands(M, N, K, seed=42)
    ref = torch.empty(M, N, dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm(ac, asc, ga, wc, wsc, gw, M, N, K, ref)
    torch.cuda.synchronize()
    check_device_error_word()
    junk = torch.empty(M, N, dtype=torch.float32, device="cuda")
    nv.nvfp4_set_wait_timeout_ns(1_000_000)                 # 1 ms
    try:
        nv.nvfp4_test_gemm_stalled_reduction(bc, bsc, gb, vc, vsc, gv, M, N, K, junk, noalloc=True)
        st = nv.nvfp4_last_device_error()
    finally:
        nv.nvfp4_set_wait_timeout_ns(0)
    assert st == nv.ERR_TIMEOUT
    r = ref.double().cpu().numpy()
    for _ in range(2):
        o = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        nv.nvfp4_gemm_noalloc(ac, asc, ga, wc, wsc, gw, M, N, K, o)
        torch.cuda.synchronize()
        max_rel, frob = rel_errors(o.cpu().numpy(), r)
        assert max_rel <= TOL_MAX_REL and frob <= TOL_FROB, (max_rel, frob)
    check_device_error_word()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # validation runs before anything touches a device: fake, aligned pointers
    p = ctypes.c_void_p(4096)
    lib = nv._lib
    for M, N in ((33, 1024), (128, 1024), (4096, 64), (8, 1 << 31)):
        st = lib.nvfp4_gemm_noalloc(p, p, 1.0, p, p, 1.0, M, N, 256, p, nv.OUT_BF16, None)
        assert st == nv.ERR_UNSUPPORTED, (M, N, st)
    st = lib.nvfp4_gemm_noalloc(p, p, 1.0, p, p, 1.0, 0, 1024, 256, p, nv.OUT_BF16, None)
    assert st == nv.ERR_INVALID_ARG
