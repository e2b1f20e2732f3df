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
