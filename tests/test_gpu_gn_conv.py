"""GPU parity of the fused GroupNorm -> temporal conv against the fp64 oracle.

Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
write-up), GroupNorm-module and conv-module paragraphs: the ResNet module
normalises with global statistics and then convolves along frames, with the
neighbouring clips' frames as padding and zeros at the video ends.  The call
is defined as the two bf16 calls composed, so the oracle composes its two
pinned modules with the GroupNorm output rounded to bf16 (the tensor the two
calls exchange).  Tolerance: 2e-2, or half a bf16 ulp of the result + 1e-3
where that is larger (|y| >= 8), as for GroupNorm outputs."""
import pytest
import torch

import clip_temporal_modules_b200 as vi
import oracle
import synth
from parity import assert_close, from_device, sample_positions, to_device

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
                                positions=positions, intermediate="bf16")
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
    """Same bf16 rounding of the normalised tensor as the two separate calls."""
    w = SMALL[1]
    x, g, bt, wt, b = (to_device(a, w.dtype) for a in inputs(w))
    fused = vi.groupnorm_conv(x, g, bt, wt, b, N=w.N, groups=w.groups, eps=w.eps)
    z = vi.groupnorm_global(x, g, bt, N=w.N, groups=w.groups, eps=w.eps)
    two = vi.temporal_conv(z, wt, b, N=w.N)
    torch.cuda.synchronize()
    d = (fused.float() - two.float()).abs().max().item()
    assert d <= 2e-2, d


def test_unsupported_channel_count_is_reported(cuda_device):
    """C not a multiple of 64 has no fused kernel: VI_ERR_UNSUPPORTED, nothing launched."""
    w = W("gnconv_C40", 16, 2, 2, 40, 8)
    x, g, bt, wt, b = (to_device(a, w.dtype) for a in inputs(w))
    with pytest.raises(vi.ViError) as e:
        vi.groupnorm_conv(x, g, bt, wt, b, N=w.N, groups=w.groups)
    assert e.value.status == -3


@pytest.mark.parametrize("tiles", [1, 2])
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
                                intermediate="bf16")
    assert_close(from_device(y), ref, w.dtype, "gn", w.name)
