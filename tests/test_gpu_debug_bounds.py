"""The bounds-checked debug build (libnvfp4_debug.so, loaded with
NVFP4_DEBUG_BOUNDS=1): the GPU parity suites pass through it unchanged with
the device error word clear, and a planted out-of-range declaration is
reported as NVFP4_ERR_DEVICE, not accessed.  Each case runs in a child
process, because the package loads one library per process."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SUITES = ["tests/test_gpu_quantize.py", "tests/test_gpu_decode.py", "tests/test_gpu_multitile.py",
          "tests/test_gpu_fused.py", "tests/test_gpu_mx.py", "tests/test_gpu_linear.py",
          "tests/test_gpu_calibrate.py", "tests/test_gpu_workspace.py", "tests/test_zz_no_alloc.py"]


def _env():
    env = dict(os.environ)
    env["NVFP4_DEBUG_BOUNDS"] = "1"
    return env


def test_parity_suites_pass_on_the_debug_build():
    # every check passes on every shape those suites use (a failed one would
    # set the error word, which each suite checks after its launches)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-p", "no:cacheprovider"] + SUITES,
                       cwd=ROOT, env=_env(), capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


PLANTED = r"""
import torch
import nvfp4_w4a4_quantized_10_b200 as nv
assert nv.nvfp4_bounds_checked()
M, K = 200, 512
x = torch.randn(M, K, device="cuda").to(torch.bfloat16)
codes, scales = nv.alloc_quantized(M, K, "cuda")
nv.nvfp4_test_bounds_check(x, codes, scales)
torch.cuda.synchronize()
st = nv._lib.nvfp4_last_device_error()
assert st == nv.ERR_DEVICE, st
# the context is intact and the same call with the true sizes is clean
ref_c, ref_s = nv.alloc_quantized(M, K, "cuda")
nv.nvfp4_quantize(x, 1.0, ref_c, ref_s)
torch.cuda.synchronize()
assert nv._lib.nvfp4_last_device_error() == nv.OK
# the checked stores were skipped, the rest written as usual
assert torch.equal(codes, ref_c)
assert torch.equal(scales[:-512], ref_s[:-512])
print("planted bounds failure reported")
"""


def test_planted_out_of_range_declaration_is_reported():
    r = subprocess.run([sys.executable, "-c", PLANTED], cwd=ROOT, env=_env(), capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "planted bounds failure reported" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]


def test_release_build_has_no_checks_to_exercise():
    import torch
    import nvfp4_w4a4_quantized_10_b200 as nv
    if nv.DEBUG_BOUNDS:
        pytest.skip("this process runs the debug build")
    assert not nv.nvfp4_bounds_checked()
    x = torch.zeros(128, 64, dtype=torch.bfloat16, device="cuda")
    c, s = nv.alloc_quantized(128, 64, "cuda")
    with pytest.raises(nv.Nvfp4Error):
        nv.nvfp4_test_bounds_check(x, c, s)
