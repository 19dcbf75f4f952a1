"""Degenerate shapes through the Python binding on the GPU: no positions
(P == 0) is a valid call that returns an empty result and launches nothing."""
import pytest
import torch

import clip_temporal_modules_b200 as vi

pytestmark = pytest.mark.gpu


def test_empty_position_axis_everywhere(cuda_device):
    F, C, heads = 64, 128, 2
    e = torch.empty(0, F, C, dtype=torch.bfloat16, device="cuda")
    w = torch.randn(C, C, 3, device="cuda").to(torch.bfloat16)
    w1 = torch.randn(3 * C, C, device="cuda").to(torch.bfloat16)
    wo = torch.randn(C, C, device="cuda").to(torch.bfloat16)
    c = torch.randn(C, device="cuda").to(torch.bfloat16)
    c3 = torch.randn(3 * C, device="cuda").to(torch.bfloat16)
    n0 = vi.launch_count()
    outs = [
        vi.dual_attn(e, e, e, N=4, heads=heads),
        vi.temporal_conv(e, w, c, N=4),
        vi.groupnorm_global(e, c, c, N=4, groups=8),
        vi.groupnorm_conv(e, c, c, w, c, N=4, groups=8),
        vi.temporal_attention(e, w1, c3, wo, c, N=4, heads=heads),
    ]
    torch.cuda.synchronize()
    vi.take_device_errors()
    assert vi.launch_count() == n0
    assert all(o.shape == (0, F, C) for o in outs)
