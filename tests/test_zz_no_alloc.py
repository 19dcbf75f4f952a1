"""The allocation-free GroupNorm entry point, vi_groupnorm_global_noalloc.

Some users of this library cannot allocate device memory once they are
running (an inference-engine plugin whose execution step may not allocate, a
service whose device memory is fixed at start-up).  For them the library has
a GroupNorm entry point that keeps its scratch in an array inside the library
instead of calling the stream-ordered allocator.  These tests call it through
the C ABI and check that it gives the same result as vi_groupnorm_global,
twice in a row (the array keeps the previous call's contents), and that it
refuses a shape whose scratch would not fit.

This file is collected last on purpose, and it passes both alone in a fresh
process (where its first call sets the array up) and after the other tests.
"""
import ctypes

import pytest
import torch

import clip_temporal_modules_b200 as vi
import synth
from parity import assert_close, from_device, to_device

pytestmark = pytest.mark.gpu

VI_ERR_UNSUPPORTED = -3


def _noalloc(L, x, g, b, y, w, stream):
    return L.vi_groupnorm_global_noalloc(x.data_ptr(), g.data_ptr(), b.data_ptr(), y.data_ptr(),
                                         w.F, w.N, w.P, w.C, w.groups, ctypes.c_float(w.eps),
                                         stream)


@pytest.mark.parametrize("name", ["bf16_F128_P2560_C320", "bf16_F1024_P640_C640"])
def test_noalloc_matches_allocating_entry_point_twice_in_a_row(cuda_device, name):
    w = synth.BY_NAME[name]
    x, g, b = (to_device(synth.make(w, t), w.dtype) for t in ("gn_x", "gn_gamma", "gn_beta"))
    ref = vi.groupnorm_global(x, g, b, N=w.N, groups=w.groups, eps=w.eps)   # allocating path
    torch.cuda.synchronize()
    want = from_device(ref)
    L = vi.lib()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        y = torch.full_like(x, float("nan"))
        assert _noalloc(L, x, g, b, y, w, stream) == 0
        torch.cuda.synchronize()
        vi.take_device_errors()
        assert_close(from_device(y), want, w.dtype, "gn", f"{name} no-alloc call {call + 1}")


def test_noalloc_in_place_matches(cuda_device):
    w = synth.BY_NAME["bf16_F128_P2560_C320"]
    x, g, b = (to_device(synth.make(w, t), w.dtype) for t in ("gn_x", "gn_gamma", "gn_beta"))
    want = from_device(vi.groupnorm_global(x, g, b, N=w.N, groups=w.groups, eps=w.eps))
    assert _noalloc(vi.lib(), x, g, b, x, w, torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert_close(from_device(x), want, w.dtype, "gn", "no-alloc in place")


def test_noalloc_rejects_scratch_beyond_its_array(cuda_device):
    """512 groups of 8 channels take the streaming path with one partial record
    per SM: 24 B x 512 groups x (at least 86) SMs does not fit in the 1 MiB array."""
    w = synth.Workload("too_many_groups", "bf16", F=16, N=1, P=64, C=4096, heads=1, d=4096,
                       groups=512)
    x = torch.zeros(w.P, w.F, w.C, dtype=torch.bfloat16, device="cuda")
    g = torch.ones(w.C, dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(w.C, dtype=torch.bfloat16, device="cuda")
    y = torch.empty_like(x)
    assert _noalloc(vi.lib(), x, g, b, y, w, torch.cuda.current_stream().cuda_stream) == \
        VI_ERR_UNSUPPORTED
