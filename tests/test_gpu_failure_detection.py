"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every pipeline in libvi waits on mbarriers with a time limit; when a limit
runs out the kernel records the fact in a device error word and returns, and
vi_take_device_errors() reports VI_ERR_DEVICE_TIMEOUT.  This test makes such a
wait run out on purpose (an mbarrier nothing arrives at, 5 ms limit), checks
the status, and checks the context is still usable afterwards."""
import pytest
import torch

import clip_temporal_modules_b200 as vi

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_is_reported_and_context_survives(cuda_device):
    L = vi.lib()
    vi.take_device_errors()                                  # start clean
    s = torch.cuda.current_stream().cuda_stream
    assert L.vi_selftest_wait_timeout(5000, s) == 0
    assert L.vi_take_device_errors() == -5                   # VI_ERR_DEVICE_TIMEOUT
    assert L.vi_take_device_errors() == 0                    # cleared by the read
    x = torch.randn(4, 32, 64, device="cuda", dtype=torch.bfloat16)
    g = torch.ones(64, device="cuda", dtype=torch.bfloat16)
    b = torch.zeros(64, device="cuda", dtype=torch.bfloat16)
    y = vi.groupnorm_global(x, g, b, N=2, groups=8)          # the context still works
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all()
    vi.take_device_errors()


def test_selftest_rejects_bad_limits(cuda_device):
    L = vi.lib()
    assert L.vi_selftest_wait_timeout(0, None) == -1
    assert L.vi_selftest_wait_timeout(2000000, None) == -1
