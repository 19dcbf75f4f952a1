"""Tensors past 2^31 elements (4.3 GB of bf16 each): every offset computation
of the kernels must be 64-bit.

The inputs are a seeded block of P0 positions repeated along the position
axis.  Attention and the conv act on each position separately, so output
position p must equal the oracle's output at position p mod P0, sampled at
the first, middle and last positions (the last ones sit beyond element 2^31).
GroupNorm statistics of a tensor repeated a whole number of times equal those
of the block, so the oracle runs on the block alone.

Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
write-up), attention-, conv- and GroupNorm-module paragraphs."""
import numpy as np
import pytest
import torch

import clip_temporal_modules_b200 as vi
import oracle
import synth
from parity import assert_close, from_device, to_device

pytestmark = pytest.mark.gpu

P0 = 64
REPS = 104                      # P = 6656 positions: 6656 * 1024 * 320 = 2.18e9 elements
BASE = synth.Workload("large_bf16_F1024_C320", "bf16", F=1024, N=64, P=P0, C=320, heads=5,
                      d=64)
P = P0 * REPS
assert P * BASE.F * BASE.C > 2 ** 31


def big(a: np.ndarray, dtype: str) -> torch.Tensor:
    return to_device(a, dtype).repeat(REPS, 1, 1)


def sample_positions():
    return [0, P0 - 1, P // 2 + 5, P - P0 + 3, P - 1]


def check(out_big: torch.Tensor, ref_fn, dtype: str, kind: str, what: str):
    pos = sample_positions()
    got = from_device(out_big[pos])
    ref = ref_fn(sorted({p % P0 for p in pos}))
    idx = {b: i for i, b in enumerate(sorted({p % P0 for p in pos}))}
    ref = np.stack([ref[idx[p % P0]] for p in pos])
    assert_close(got, ref, dtype, kind, what)


def free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def test_attention_beyond_2_31_elements(cuda_device):
    w = BASE
    q, k, v = (synth.make(w, t) for t in ("q", "k", "v"))
    dq, dk, dv = (big(a, w.dtype) for a in (q, k, v))
    out = vi.dual_attn(dq, dk, dv, N=w.N, heads=w.heads)
    vi.take_device_errors()
    check(out, lambda ps: oracle.dual_attn(q, k, v, w.F, w.N, w.heads, w.d, positions=ps),
          w.dtype, "attn", "attention, 2.18e9 elements")
    del dq, dk, dv, out
    free()


def test_conv_beyond_2_31_elements(cuda_device):
    w = BASE
    x, wt, b = (synth.make(w, t) for t in ("conv_x", "conv_w", "conv_b"))
    dx = big(x, w.dtype)
    y = vi.temporal_conv(dx, to_device(wt, w.dtype), to_device(b, w.dtype), N=w.N)
    vi.take_device_errors()
    check(y, lambda ps: oracle.temporal_conv(x, wt, b, w.F, w.N, w.k, positions=ps),
          w.dtype, "conv", "conv, 2.18e9 elements")
    del dx, y
    free()


def test_groupnorm_beyond_2_31_elements(cuda_device):
    w = BASE
    x, g, bt = (synth.make(w, t) for t in ("gn_x", "gn_gamma", "gn_beta"))
    dx = big(x, w.dtype)
    y = vi.groupnorm_global(dx, to_device(g, w.dtype), to_device(bt, w.dtype), N=w.N,
                            groups=w.groups, eps=w.eps)
    vi.take_device_errors()
    ref_all, _, _ = oracle.groupnorm_global(x, g, bt, w.F, w.N, w.groups, w.eps)
    check(y, lambda ps: ref_all[ps], w.dtype, "gn", "GroupNorm, 2.18e9 elements")
    del dx, y
    free()


def test_attention_module_beyond_2_31_elements(cuda_device):
    """The attention module (q/k/v GEMM, then the attention with the output
    projection fused in): per position, so the repeated block applies."""
    w = BASE
    names = ("attn_x", "w_qkv", "b_qkv", "w_out", "b_out")
    x, wq, bq, wo, bo = (synth.make(w, t) for t in names)
    dx = big(x, w.dtype)
    out = vi.temporal_attention(dx, *(to_device(a, w.dtype) for a in (wq, bq, wo, bo)), N=w.N,
                                heads=w.heads)
    vi.take_device_errors()
    check(out, lambda ps: oracle.temporal_attention(x, wq, bq, wo, bo, w.F, w.N, w.heads, w.d,
                                                    positions=ps),
          w.dtype, "attn", "attention module, 2.18e9 elements")
    del dx, out
    free()
