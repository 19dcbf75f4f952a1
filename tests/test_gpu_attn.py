"""GPU parity of dual-domain attention against the fp64 oracle.

Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
write-up), attention-module paragraph.  Small cases are compared element by
element and span several CTA tiles, ragged tails and every branch of the key
list (absent ends, short context, no global frames, one clip); the five
workloads run at full size and are compared on sampled positions."""
import numpy as np
import pytest
import torch

import clip_temporal_modules_b200 as vi
import oracle
import synth
from parity import assert_close, from_device, sample_positions, to_device

pytestmark = pytest.mark.gpu


def run_case(w: synth.Workload, positions=None):
    q, k, v = (synth.make(w, t) for t in ("q", "k", "v"))
    dq, dk, dv = (to_device(a, w.dtype) for a in (q, k, v))
    out = vi.dual_attn(dq, dk, dv, N=w.N, heads=w.heads, n_pre=w.n_pre, n_post=w.n_post,
                       n_global=w.n_global)
    torch.cuda.synchronize()
    vi.take_device_errors()
    got = from_device(out)
    ref = oracle.dual_attn(q, k, v, w.F, w.N, w.heads, w.d, w.n_pre, w.n_post, w.n_global,
                           positions=positions)
    if positions is not None:
        got = got[positions]
    return assert_close(got, ref, w.dtype, "attn", w.name)


def W(name, dtype, F, N, P, heads, **kw):
    return synth.Workload(name, dtype, F=F, N=N, P=P, C=heads * 64, heads=heads, d=64, **kw)


SMALL = [
    synth.WORKLOADS[0],                                        # tiny fp32 (generic path)
    W("bf16_1blk_ragged", "bf16", 48, 3, 5, 2),                # fast path, 3 of 8 clips
    W("bf16_2blk_ragged", "bf16", 160, 10, 3, 3),              # 8 + 2 clips, stride 10
    W("bf16_short_ctx", "bf16", 64, 4, 4, 2, n_pre=3, n_post=5, n_global=7),
    W("bf16_no_global", "bf16", 64, 4, 3, 1, n_global=0),
    W("bf16_one_clip", "bf16", 16, 1, 6, 2, n_global=4),
    W("bf16_no_context", "bf16", 48, 3, 2, 1, n_pre=0, n_post=0, n_global=0),
    W("bf16_halo16", "bf16", 64, 4, 3, 2, n_pre=16, n_post=16, n_global=16),   # 16-row window
    W("bf16_halo12_2blk_ragged", "bf16", 160, 10, 3, 2, n_pre=12, n_post=9, n_global=7),
    W("bf16_halo_mixed", "bf16", 96, 6, 2, 1, n_pre=4, n_post=13, n_global=16),
    W("bf16_halo16_no_global", "bf16", 48, 3, 2, 1, n_pre=16, n_post=10, n_global=0),
    # clips of 8 frames on the fast path: two clips per warp, each its own mask
    W("bf16_L8_1blk_ragged", "bf16", 40, 5, 5, 2),             # warps (0,1) (2,3) (4,-)
    W("bf16_L8_2blk_ragged", "bf16", 200, 25, 3, 3),           # 16 + 9 clips
    W("bf16_L8_two_clips", "bf16", 16, 2, 4, 1, n_global=2),
    W("bf16_L8_one_clip", "bf16", 8, 1, 6, 2, n_global=4),
    W("bf16_L8_short_ctx", "bf16", 64, 8, 4, 2, n_pre=3, n_post=5, n_global=7),
    W("bf16_L8_one_sided", "bf16", 96, 12, 3, 1, n_pre=0, n_post=8, n_global=0),
    W("bf16_L8_pre_only", "bf16", 48, 6, 2, 1, n_pre=8, n_post=1, n_global=16),
    # clips of 32 frames on the fast path: two warps per clip
    W("bf16_L32_1blk_ragged", "bf16", 96, 3, 4, 2),            # 3 of 4 clips in the block
    W("bf16_L32_3blk_ctx", "bf16", 320, 10, 2, 3, n_pre=5, n_post=8, n_global=10),
    W("bf16_L32_one_clip", "bf16", 32, 1, 5, 1, n_global=4),
    W("bf16_L32_no_global", "bf16", 128, 4, 3, 2, n_global=0),
    # shapes outside the fast path: the generic kernel
    W("bf16_L4_generic", "bf16", 32, 8, 4, 2, n_pre=4, n_post=4),
    W("bf16_L32_generic", "bf16", 64, 2, 3, 1, n_pre=16, n_post=12, n_global=20),
    W("bf16_L8_global20_generic", "bf16", 64, 8, 2, 1, n_global=20),
    # key lists too long to stage in shared memory: the unstaged generic kernel
    W("bf16_L128_ctx128_unstaged", "bf16", 256, 2, 2, 1, n_pre=128, n_post=128, n_global=16),
    W("f32_generic", "f32", 48, 3, 3, 2),
    W("f32_L16_short", "f32", 64, 4, 2, 1, n_pre=2, n_post=0, n_global=5),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_small_elementwise(cuda_device, w):
    run_case(w)


@pytest.mark.parametrize("w", synth.WORKLOADS[1:], ids=lambda w: w.name)
def test_full_size_sampled_positions(cuda_device, w):
    run_case(w, positions=sample_positions(w.P))


def test_clips_of_8_frames_at_size(cuda_device):
    """F = 1024 in 128 clips of 8 frames (the fast path, two clips per warp)."""
    w = W("bf16_F1024_N128_P64_C320_L8", "bf16", 1024, 128, 64, 5)
    run_case(w, positions=sample_positions(w.P, count=2))


def test_clips_of_32_frames_at_size(cuda_device):
    """F = 1024 in 32 clips of 32 frames (the fast path, two warps per clip)."""
    w = W("bf16_F1024_N32_P64_C320_L32", "bf16", 1024, 32, 64, 5)
    run_case(w, positions=sample_positions(w.P, count=2))


# Ablation settings of the write-up's study (attention without global context,
# without local context, and with no context exchange at all) at full size.
ABLATIONS = [dict(n_pre=8, n_post=8, n_global=0), dict(n_pre=0, n_post=0, n_global=16),
             dict(n_pre=0, n_post=0, n_global=0)]


@pytest.mark.parametrize("ctx", ABLATIONS, ids=["local_only", "global_only", "no_sync"])
def test_ablation_settings_full_size(cuda_device, ctx):
    w = synth.BY_NAME["bf16_F1024_P2560_C320"].with_(**ctx)
    run_case(w, positions=sample_positions(w.P, count=2))


def test_fp32_tiny_full_workload_all_positions(cuda_device):
    run_case(synth.WORKLOADS[0])


def test_runs_on_given_stream_and_leaves_neighbours_untouched(cuda_device):
    w = W("bf16_stream", "bf16", 64, 4, 3, 2)
    q, k, v = (to_device(synth.make(w, t), w.dtype) for t in ("q", "k", "v"))
    n = q.numel()
    buf = torch.full((n + 64,), 7.0, dtype=torch.bfloat16, device="cuda")
    out = buf[32:32 + n].view_as(q)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        vi.dual_attn(q, k, v, out, N=w.N, heads=w.heads, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    assert torch.all(buf[:32] == 7.0) and torch.all(buf[32 + n:] == 7.0)
    ref = vi.dual_attn(q, k, v, N=w.N, heads=w.heads)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def test_no_global_frames_ignores_stale_shared_memory(cuda_device):
    """With n_global = 0 the global K/V tiles are not loaded; whatever an
    earlier kernel left in that shared memory (here NaN) must not leak."""
    w = W("bf16_poison", "bf16", 1024, 64, 64, 5)
    nan = torch.full((w.P, w.F, w.C), float("nan"), dtype=torch.bfloat16, device="cuda")
    vi.dual_attn(nan, nan, nan, torch.empty_like(nan), N=w.N, heads=w.heads)   # fills smem
    torch.cuda.synchronize()
    ctx = dict(n_pre=0, n_post=0, n_global=0)
    q, k, v = (synth.make(w, t) for t in ("q", "k", "v"))
    dq, dk, dv = (to_device(a, w.dtype) for a in (q, k, v))
    for _ in range(3):
        vi.dual_attn(nan, nan, nan, torch.empty_like(nan), N=w.N, heads=w.heads)
        out = vi.dual_attn(dq, dk, dv, N=w.N, heads=w.heads, **ctx)
        torch.cuda.synchronize()
        got = from_device(out)
        assert np.all(np.isfinite(got))
    pos = [0, 17, 63]
    ref = oracle.dual_attn(q, k, v, w.F, w.N, w.heads, w.d, positions=pos, **ctx)
    assert_close(got[pos], ref, w.dtype, "attn", "no global after NaN")
