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


def run_case(w, positions=None, fused=None):
    """fused: None = the library's choice; True / False = that form forced."""
    x, wq, bq, wo, bo = (synth.make(w, t) for t in NAMES)
    dev = [to_device(a, w.dtype) for a in (x, wq, bq, wo, bo)]
    if fused is None:
        out = vi.temporal_attention(*dev, N=w.N, heads=w.heads, n_pre=w.n_pre, n_post=w.n_post,
                                    n_global=w.n_global)
    else:
        from clip_temporal_modules_b200._binding import temporal_attention_forced_form
        out = temporal_attention_forced_form(*dev, N=w.N, heads=w.heads, fused=fused,
                                             n_pre=w.n_pre, n_post=w.n_post,
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
    W("attnmod_F32_N8_P4_h1_L4", 32, 8, 4, 1, n_pre=4, n_post=4),   # generic attention path
    W("attnmod_F64_N4_P2_h5_ctx", 64, 4, 2, 5, n_pre=3, n_post=5, n_global=7),
]


# Shapes of the fused form (attention + output projection in one kernel):
# every head count it takes (C = 64 .. 320: one to five 32-column groups per
# epilogue warp, 64- and 32-channel store boxes), both window widths, ragged
# last clip blocks, one clip, no global frames, context sizes off the window.
FUSED = [
    W("attnmod_fused_F160_N10_P3_h2", 160, 10, 3, 2),                 # 2 blocks, 2 clips in the last
    W("attnmod_fused_F48_N3_P5_h1_noglobal", 48, 3, 5, 1, n_global=0),
    W("attnmod_fused_F16_N1_P7_h3_oneclip", 16, 1, 7, 3, n_global=4),
    W("attnmod_fused_F128_N8_P3_h4", 128, 8, 3, 4),
    W("attnmod_fused_F288_N18_P2_h5_ctx8", 288, 18, 2, 5, n_pre=8, n_post=7, n_global=9),
    W("attnmod_fused_F256_N16_P2_h5_ctx", 256, 16, 2, 5, n_pre=0, n_post=3, n_global=16),
    W("attnmod_fused_F72_N9_P3_h3_L8", 72, 9, 3, 3, n_pre=5, n_post=8, n_global=9),   # 8-frame clips
    W("attnmod_fused_F160_N5_P3_h4_L32", 160, 5, 3, 4, n_pre=8, n_post=2, n_global=5),  # 32-frame
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_small_elementwise(cuda_device, w):
    run_case(w)


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "attn_then_gemm"])
@pytest.mark.parametrize("w", FUSED, ids=lambda w: w.name)
def test_both_forms_elementwise(cuda_device, w, fused):
    run_case(w, fused=fused)


def oproj_case(w, positions=None):
    """The fused kernel alone on q, k, v: out = bf16(a) W_out^T + b_out with a the
    dual-domain attention, against the oracle's attention rounded to bf16 (the
    operand the kernel hands the tensor core) and its single-tap projection."""
    from clip_temporal_modules_b200._binding import dual_attn_oproj
    q, k, v, wo, bo = (synth.make(w, t) for t in ("q", "k", "v", "w_out", "b_out"))
    dq, dk, dv, dwo, dbo = (to_device(a, w.dtype) for a in (q, k, v, wo, bo))
    out = dual_attn_oproj(dq, dk, dv, dwo, dbo, N=w.N, heads=w.heads, n_pre=w.n_pre,
                          n_post=w.n_post, n_global=w.n_global)
    torch.cuda.synchronize()
    vi.take_device_errors()
    got = from_device(out)
    a = oracle.dual_attn(q, k, v, w.F, w.N, w.heads, w.d, w.n_pre, w.n_post, w.n_global,
                         positions=positions)
    a = np.ascontiguousarray(oracle.round_bf16(a), dtype=np.float32)
    ref = oracle.temporal_conv(a, np.ascontiguousarray(wo).reshape(w.C, w.C, 1),
                               np.ascontiguousarray(bo), w.F, w.N, 1)
    if positions is not None:
        got = got[positions]
    return assert_close(got, ref, w.dtype, "attn", w.name)


@pytest.mark.parametrize("w", FUSED, ids=lambda w: w.name)
def test_fused_kernel_alone_elementwise(cuda_device, w):
    oproj_case(w)


def test_fused_kernel_alone_full_size_sampled_positions(cuda_device):
    w = synth.BY_NAME["bf16_F1024_P2560_C320"]
    oproj_case(w, positions=sample_positions(w.P, count=3))


def test_fused_form_refuses_context_above_8(cuda_device):
    """Context above 8 frames needs the 16-row window, whose stages do not fit
    beside the fused kernel's W_out slice and staging: the forced fused form is
    refused before any launch, and the library's choice runs the attention
    kernel (16-row window) and the output GEMM (checked against the oracle)."""
    from clip_temporal_modules_b200._binding import dual_attn_oproj, temporal_attention_forced_form
    w = W("attnmod_F288_N18_P2_h5_halo16", 288, 18, 2, 5, n_pre=12, n_post=16, n_global=9)
    x, wq, bq, wo, bo = (to_device(synth.make(w, t), w.dtype) for t in NAMES)
    n0 = vi.launch_count()
    with pytest.raises(vi.ViError):
        temporal_attention_forced_form(x, wq, bq, wo, bo, N=w.N, heads=w.heads, fused=True,
                                       n_pre=w.n_pre, n_post=w.n_post, n_global=w.n_global)
    with pytest.raises(vi.ViError):
        dual_attn_oproj(x, x, x, wo, bo, N=w.N, heads=w.heads, n_pre=w.n_pre, n_post=w.n_post,
                        n_global=w.n_global)
    assert vi.launch_count() == n0
    run_case(w)


def test_fused_form_refuses_more_than_five_heads(cuda_device):
    """Six heads (C = 384) exceed the fused kernel's TMEM and shared-memory plan:
    the forced fused form is refused before any launch, and the library's
    choice runs the attention kernel and the output GEMM (checked against the
    oracle)."""
    from clip_temporal_modules_b200._binding import temporal_attention_forced_form
    w = W("attnmod_F32_N2_P2_h6", 32, 2, 2, 6)
    x, wq, bq, wo, bo = (to_device(synth.make(w, t), w.dtype) for t in NAMES)
    n0 = vi.launch_count()
    with pytest.raises(vi.ViError):
        temporal_attention_forced_form(x, wq, bq, wo, bo, N=w.N, heads=w.heads, fused=True)
    assert vi.launch_count() == n0
    run_case(w)


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "attn_then_gemm"])
def test_full_size_sampled_positions(cuda_device, fused):
    w = synth.BY_NAME["bf16_F1024_P2560_C320"]
    run_case(w, positions=sample_positions(w.P, count=2), fused=fused)


def test_full_size_library_choice(cuda_device):
    w = synth.BY_NAME["bf16_F1024_P2560_C320"]
    run_case(w, positions=sample_positions(w.P, count=1))


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
