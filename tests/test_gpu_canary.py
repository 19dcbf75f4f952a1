"""No kernel writes outside its output: each call writes into the middle of a
larger buffer filled with a sentinel, and the sentinel must survive on both
sides.  The shapes have ragged frame tails (the conv's TMA stores clip the
rows past the last frame; the last position's last tile is where an unclipped
store would spill past the tensor) and odd position counts.  The results must
also equal the same call writing into a fresh tensor."""
import pytest
import torch

import clip_temporal_modules_b200 as vi
import synth
from parity import to_device

pytestmark = pytest.mark.gpu

PAD = 4096                      # elements of sentinel on each side
SENTINEL = -12345.0


def _padded_like(t):
    n = t.numel()
    buf = torch.full((n + 2 * PAD,), SENTINEL, dtype=t.dtype, device=t.device)
    return buf, buf[PAD:PAD + n].view_as(t)


def _intact(buf, n):
    return bool(torch.all(buf[:PAD] == SENTINEL)) and bool(torch.all(buf[PAD + n:] == SENTINEL))


CONV = [synth.Workload("canary_conv_F200_P3", "bf16", F=200, N=8, P=3, C=320, heads=5, d=64),
        synth.Workload("canary_conv_F130_P5_k5", "bf16", F=130, N=10, P=5, C=128, heads=2, d=64,
                       k=5),
        synth.Workload("canary_conv_F24_P3_k1", "bf16", F=24, N=3, P=3, C=320, heads=5, d=64,
                       k=1)]


@pytest.mark.parametrize("w", CONV, ids=lambda w: w.name)
def test_conv_writes_only_its_output(cuda_device, w):
    x, wt, b = (to_device(synth.make(w, t), w.dtype) for t in ("conv_x", "conv_w", "conv_b"))
    buf, y = _padded_like(x)
    vi.temporal_conv(x, wt, b, y, N=w.N)
    ref = vi.temporal_conv(x, wt, b, N=w.N)
    torch.cuda.synchronize()
    vi.take_device_errors()
    assert _intact(buf, x.numel())
    assert torch.equal(y, ref)


def test_groupnorm_and_fused_conv_write_only_their_output(cuda_device):
    w = synth.Workload("canary_gn_F200_P3", "bf16", F=200, N=8, P=3, C=320, heads=5, d=64)
    x, g, bt, wt, b = (to_device(synth.make(w, t), w.dtype)
                       for t in ("gn_x", "gn_gamma", "gn_beta", "conv_w", "conv_b"))
    buf, z = _padded_like(x)
    vi.groupnorm_global(x, g, bt, z, N=w.N, groups=w.groups)
    buf2, y = _padded_like(x)
    vi.groupnorm_conv(x, g, bt, wt, b, y, N=w.N, groups=w.groups)
    ref_z = vi.groupnorm_global(x, g, bt, N=w.N, groups=w.groups)
    ref_y = vi.groupnorm_conv(x, g, bt, wt, b, N=w.N, groups=w.groups)
    torch.cuda.synchronize()
    vi.take_device_errors()
    assert _intact(buf, x.numel()) and _intact(buf2, x.numel())
    assert torch.equal(z, ref_z) and torch.equal(y, ref_y)


def test_attention_module_writes_only_its_output(cuda_device):
    w = synth.Workload("canary_tattn_F48_P3", "bf16", F=48, N=3, P=3, C=128, heads=2, d=64)
    x = to_device(synth.make(w, "attn_x"), w.dtype)
    wq = to_device(synth.make(w, "w_qkv"), w.dtype)
    bq = to_device(synth.make(w, "b_qkv"), w.dtype)
    wo = to_device(synth.make(w, "w_out"), w.dtype)
    bo = to_device(synth.make(w, "b_out"), w.dtype)
    buf, out = _padded_like(x)
    vi.temporal_attention(x, wq, bq, wo, bo, out, N=w.N, heads=w.heads)
    ref = vi.temporal_attention(x, wq, bq, wo, bo, N=w.N, heads=w.heads)
    torch.cuda.synchronize()
    vi.take_device_errors()
    assert _intact(buf, x.numel())
    assert torch.equal(out, ref)
