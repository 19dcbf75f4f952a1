"""GPU parity of global-statistics GroupNorm against the fp64 oracle.

Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
write-up), GroupNorm-module paragraph.  Small cases element by element (vector
path with groups straddling a 16-byte vector, scalar path for groups narrower
than a vector, in place); the five workloads at full size, with the global
statistics over the whole tensor and outputs checked on sampled positions."""
import numpy as np
import pytest
import torch

import clip_temporal_modules_b200 as vi
import oracle
import synth
from parity import assert_close, from_device, sample_positions, to_device

pytestmark = pytest.mark.gpu


def run_case(w: synth.Workload, positions=None, in_place=False):
    x, g, b = (synth.make(w, t) for t in ("gn_x", "gn_gamma", "gn_beta"))
    dx, dg, db = (to_device(a, w.dtype) for a in (x, g, b))
    out = dx if in_place else None
    y = vi.groupnorm_global(dx, dg, db, out, N=w.N, groups=w.groups, eps=w.eps)
    torch.cuda.synchronize()
    vi.take_device_errors()
    got = from_device(y)
    ref, _, _ = oracle.groupnorm_global(x, g, b, w.F, w.N, w.groups, w.eps, positions=positions)
    if positions is not None:
        got = got[positions]
    return assert_close(got, ref, w.dtype, "gn", w.name)


def W(name, dtype, F, N, P, C, groups, eps=1e-5):
    return synth.Workload(name, dtype, F=F, N=N, P=P, C=C, heads=1, d=C, groups=groups, eps=eps)


SMALL = [
    synth.WORKLOADS[0],
    W("bf16_C320_G32", "bf16", 64, 4, 7, 320, 32),      # 10 channels per group: straddles
    W("bf16_C640_G32", "bf16", 48, 3, 5, 640, 32),
    W("bf16_C1280_G32", "bf16", 32, 2, 3, 1280, 32),
    W("bf16_C64_G32_scalar", "bf16", 32, 4, 5, 64, 32),  # 2 channels per group: scalar path
    W("bf16_C24_G3", "bf16", 16, 2, 3, 24, 3),
    W("f32_C36_G6", "f32", 24, 3, 4, 36, 6),
    W("f32_C64_G32_scalar", "f32", 16, 4, 3, 64, 32),
    W("bf16_C320_G1_eps0", "bf16", 16, 1, 5, 320, 1, eps=0.0),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_small_elementwise(cuda_device, w):
    run_case(w)


@pytest.mark.parametrize("w", SMALL[1:3], ids=lambda w: w.name)
def test_in_place(cuda_device, w):
    run_case(w, in_place=True)


@pytest.mark.parametrize("w", synth.WORKLOADS[1:], ids=lambda w: w.name)
def test_full_size_sampled_positions(cuda_device, w):
    run_case(w, positions=sample_positions(w.P))


def test_repeated_calls_are_identical(cuda_device):
    """The scratch ticket resets itself: back-to-back calls give the same bits."""
    w = SMALL[1]
    x, g, b = (to_device(synth.make(w, t), w.dtype) for t in ("gn_x", "gn_gamma", "gn_beta"))
    ys = [vi.groupnorm_global(x, g, b, N=w.N, groups=w.groups) for _ in range(3)]
    torch.cuda.synchronize()
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[0], ys[2])


def test_constant_group_gives_beta(cuda_device):
    w = W("bf16_const", "bf16", 32, 2, 3, 320, 32)
    x = synth.make(w, "gn_x")
    x.reshape(-1, 320)[:, 20:30] = synth.f32_to_bf16(np.array([2.5], np.float32))[0]
    g, b = synth.make(w, "gn_gamma"), synth.make(w, "gn_beta")
    y = vi.groupnorm_global(to_device(x, "bf16"), to_device(g, "bf16"), to_device(b, "bf16"),
                            N=w.N, groups=32)
    got = from_device(y).reshape(-1, 320)[:, 20:30]
    beta = synth.bf16_to_f32(b)[20:30].astype(np.float64)
    np.testing.assert_array_equal(got, np.broadcast_to(beta, got.shape))
