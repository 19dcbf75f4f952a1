"""GPU parity of the temporal attention module (projections + dual-domain
attention + output projection) against the fp64 oracle.

Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
write-up), attention-module paragraph: the module's keys and values are
gathered from the clip, its neighbours and the global frames; the linear
projections around the attention are the module's own layers.  The oracle
composes its pinned projection (single-tap conv) and attention functions with
bf16 intermediates, the tensors the module's stages exchange.  Tolerance: the
attention's 2e-2 (the outputs are convex combinations of v projected with
fan-in-scaled weights, sigma ~ 1)."""
import numpy as np
import pytest
import torch

import clip_temporal_modules_b200 as vi
import oracle
import synth
from parity import assert_close, from_device, sample_positions, to_device

pytestmark = pytest.mark.gpu

NAMES = ("attn_x", "w_qkv", "b_qkv", "w_out", "b_out")


def run_case(w, positions=None):
    x, wq, bq, wo, bo = (synth.make(w, t) for t in NAMES)
    dev = [to_device(a, w.dtype) for a in (x, wq, bq, wo, bo)]
    out = vi.temporal_attention(*dev, N=w.N, heads=w.heads, n_pre=w.n_pre, n_post=w.n_post,
                                n_global=w.n_global)
    torch.cuda.synchronize()
    vi.take_device_errors()
    got = from_device(out)
    ref = oracle.temporal_attention(x, wq, bq, wo, bo, w.F, w.N, w.heads, w.d, w.n_pre,
                                    w.n_post, w.n_global, positions=positions)
    if positions is not None:
        got = got[positions]
    # the attention tolerance (2e-2): module outputs have sigma ~ 1
    return assert_close(got, ref, w.dtype, "attn", w.name)


def W(name, F, N, P, heads, **kw):
    return synth.Workload(name, "bf16", F=F, N=N, P=P, C=heads * 64, heads=heads, d=64, **kw)


SMALL = [
    W("attnmod_F160_N10_P3_h2", 160, 10, 3, 2),          # fast attention path, 2 blocks
    W("attnmod_F32_N4_P4_h1_L8", 32, 4, 4, 1),            # generic attention path
    W("attnmod_F64_N4_P2_h5_ctx", 64, 4, 2, 5, n_pre=3, n_post=5, n_global=7),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_small_elementwise(cuda_device, w):
    run_case(w)


def test_full_size_sampled_positions(cuda_device):
    w = synth.BY_NAME["bf16_F1024_P2560_C320"]
    run_case(w, positions=sample_positions(w.P, count=2))


def test_workspace_size_and_caller_workspace(cuda_device):
    w = SMALL[0]
    n = vi.lib().vi_temporal_attention_workspace_bytes(w.F, w.P, w.C)
    assert n == 4 * w.F * w.P * w.C * 2
    x, wq, bq, wo, bo = (to_device(synth.make(w, t), w.dtype) for t in NAMES)
    ws = torch.full((n // 2,), float("nan"), dtype=torch.bfloat16, device="cuda")
    a = vi.temporal_attention(x, wq, bq, wo, bo, workspace=ws, N=w.N, heads=w.heads)
    b = vi.temporal_attention(x, wq, bq, wo, bo, N=w.N, heads=w.heads)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
