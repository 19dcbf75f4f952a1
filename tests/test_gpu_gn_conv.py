"""GPU parity of the fused GroupNorm -> temporal conv against the fp64 oracle.

Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
write-up), GroupNorm-module and conv-module paragraphs: the ResNet module
normalises with global statistics and then convolves along frames, with the
neighbouring clips' frames as padding and zeros at the video ends.  The call
computes the conv of the GroupNorm output; the oracle composes its two pinned
modules in fp64 (no rounding in between).  The kernel folds the GroupNorm
scale into bf16 weights and its mean and shift into exact bias tables, so it
is also checked on groups whose mean is large against their spread, where a
fold that rounded the mean term would lose accuracy.  Tolerance: 2e-2, or
half a bf16 ulp of the result + 1e-3 where that is larger (|y| >= 8)."""
import numpy as np
import pytest
import torch

import clip_temporal_modules_b200 as vi
import oracle
import synth
from parity import (assert_close, from_device, half_ulp_bf16, sample_positions, to_device,
                    tolerance)

pytestmark = pytest.mark.gpu


def inputs(w):
    names = ("gn_x", "gn_gamma", "gn_beta", "conv_w", "conv_b")
    return [synth.make(w, t) for t in names]


def run_case(w, positions=None):
    x, g, bt, wt, b = inputs(w)
    dev = [to_device(a, w.dtype) for a in (x, g, bt, wt, b)]
    y = vi.groupnorm_conv(*dev, N=w.N, groups=w.groups, eps=w.eps)
    torch.cuda.synchronize()
    vi.take_device_errors()
    got = from_device(y)
    ref = oracle.groupnorm_conv(x, g, bt, wt, b, w.F, w.N, w.groups, w.eps, w.k,
                                positions=positions, intermediate="f64")
    if positions is not None:
        got = got[positions]
    return assert_close(got, ref, w.dtype, "gn", w.name)


def W(name, F, N, P, C, groups, k=3):
    return synth.Workload(name, "bf16", F=F, N=N, P=P, C=C, heads=1, d=C, groups=groups, k=k)


SMALL = [
    W("gnconv_F48_C64_G8", 48, 3, 5, 64, 8),
    W("gnconv_F200_C320_G32_ragged", 200, 8, 3, 320, 32),
    W("gnconv_F256_C640_G32", 256, 16, 2, 640, 32),
    W("gnconv_F40_C320_G32_k5", 40, 5, 3, 320, 32, k=5),
    W("gnconv_F24_C128_G4_k1", 24, 3, 2, 128, 4, k=1),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_small_elementwise(cuda_device, w):
    run_case(w)


@pytest.mark.parametrize("name", ["bf16_F1024_P2560_C320", "bf16_F2304_P160_C1280"])
def test_full_size_sampled_positions(cuda_device, name):
    w = synth.BY_NAME[name]
    run_case(w, positions=sample_positions(w.P, count=2))


def test_matches_groupnorm_then_conv_calls(cuda_device):
    """The fused call and the two bf16 calls composed are each within the bf16
    tolerance of the exact composition, so they agree within the sum of the
    two tolerances (they round different intermediates: W a, or the
    normalised tensor, so one bf16 ulp apart is possible)."""
    w = SMALL[1]
    xs, gs, bts, wts, bs = inputs(w)
    x, g, bt, wt, b = (to_device(a, w.dtype) for a in (xs, gs, bts, wts, bs))
    fused = vi.groupnorm_conv(x, g, bt, wt, b, N=w.N, groups=w.groups, eps=w.eps)
    z = vi.groupnorm_global(x, g, bt, N=w.N, groups=w.groups, eps=w.eps)
    two = vi.temporal_conv(z, wt, b, N=w.N)
    torch.cuda.synchronize()
    ref = oracle.groupnorm_conv(xs, gs, bts, wts, bs, w.F, w.N, w.groups, w.eps, w.k,
                                intermediate="f64")
    f, t = from_device(fused), from_device(two)
    assert_close(f, ref, w.dtype, "gn", "fused")
    assert_close(t, ref, w.dtype, "gn", "two calls")
    assert np.all(np.abs(f - t) <= 2 * tolerance(w.dtype, ref, "gn"))


@pytest.mark.parametrize("tiles", [1, 2, 4])
@pytest.mark.parametrize("w", [W("gnconv_F48_C64_G8_odd_tiles", 48, 3, 5, 64, 8),
                               W("gnconv_F200_C320_G32_ragged", 200, 8, 3, 320, 32)],
                         ids=lambda w: w.name)
def test_one_and_two_tiles_per_job(cuda_device, w, tiles):
    """Both job forms of the fused conv (the transform warps normalise one or
    two x boxes per stage)."""
    from clip_temporal_modules_b200._binding import groupnorm_conv_forced_tiles
    x, g, bt, wt, b = inputs(w)
    dev = [to_device(a, w.dtype) for a in (x, g, bt, wt, b)]
    y = groupnorm_conv_forced_tiles(*dev, N=w.N, groups=w.groups, eps=w.eps, tiles=tiles)
    torch.cuda.synchronize()
    vi.take_device_errors()
    ref = oracle.groupnorm_conv(x, g, bt, wt, b, w.F, w.N, w.groups, w.eps, w.k,
                                intermediate="f64")
    assert_close(from_device(y), ref, w.dtype, "gn", w.name)


@pytest.mark.parametrize("shift", [0.0, 100.0, -300.0])
def test_groups_with_a_large_mean(cuda_device, shift):
    """x = shift + N(0.5, 2), rounded to bf16: |mean| / std up to ~200.  The
    folded weights round W a, which only scales x - m (the mean terms cancel
    exactly against bias tables built from the same rounded weights), so the
    error beyond the output's own bf16 rounding stays at the level of the two
    bf16 calls composed (about 8e-3 here at any shift).  A fold whose mean
    term used unrounded weights would err by about |m| x 2^-9 x |W a| summed
    over the 3C inputs: about 0.1 at shift 100."""
    w = W("gnconv_F200_C320_G32_shift", 200, 8, 3, 320, 32)
    x, g, bt, wt, b = inputs(w)
    xs = synth.f32_to_bf16((synth.bf16_to_f32(x) + np.float32(shift)).astype(np.float32))
    dev = [to_device(a, w.dtype) for a in (xs, g, bt, wt, b)]
    y = vi.groupnorm_conv(*dev, N=w.N, groups=w.groups, eps=w.eps)
    torch.cuda.synchronize()
    vi.take_device_errors()
    ref = oracle.groupnorm_conv(xs, g, bt, wt, b, w.F, w.N, w.groups, w.eps, w.k,
                                intermediate="f64")
    got = from_device(y)
    assert_close(got, ref, w.dtype, "gn", w.name)
    excess = np.max(np.abs(got - ref) - half_ulp_bf16(ref))
    assert excess <= 1e-2, excess
