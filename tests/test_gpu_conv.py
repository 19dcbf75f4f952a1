"""GPU parity of the clip-padded temporal conv against the fp64 oracle.

Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
write-up), conv-module paragraph.  Small cases element by element (several
tiles, ragged frame and channel tails, k = 1, 3, 5); the five workloads at full
size on sampled positions (all frames and channels of each)."""
import pytest
import torch

import clip_temporal_modules_b200 as vi
import oracle
import synth
from parity import assert_close, from_device, sample_positions, to_device

pytestmark = pytest.mark.gpu


def run_case(w: synth.Workload, positions=None):
    x, wt, b = (synth.make(w, t) for t in ("conv_x", "conv_w", "conv_b"))
    dx, dw, db = (to_device(a, w.dtype) for a in (x, wt, b))
    y = vi.temporal_conv(dx, dw, db, N=w.N)
    torch.cuda.synchronize()
    vi.take_device_errors()
    got = from_device(y)
    ref = oracle.temporal_conv(x, wt, b, w.F, w.N, w.k, positions=positions)
    if positions is not None:
        got = got[positions]
    return assert_close(got, ref, w.dtype, "conv", w.name)


def W(name, dtype, F, N, P, C, k=3):
    return synth.Workload(name, dtype, F=F, N=N, P=P, C=C, heads=1, d=C, k=k)


SMALL = [
    synth.WORKLOADS[0],
    W("bf16_F48_C64", "bf16", 48, 3, 5, 64),
    W("bf16_F200_C320_ragged", "bf16", 200, 8, 3, 320),      # frame tail of 72 rows
    W("bf16_F256_C640", "bf16", 256, 16, 2, 640),
    W("bf16_F72_C192_slab96", "bf16", 72, 3, 3, 192),      # 96-channel slabs: 64 + 32 chunks
    W("bf16_F64_C256_slab128", "bf16", 64, 4, 2, 256),     # 128-channel slabs
    W("bf16_F40_C136_k5", "bf16", 40, 5, 3, 136, k=5),       # channel tail, wider halo
    W("bf16_F24_C64_k1", "bf16", 24, 3, 2, 64, k=1),
    W("f32_F40_C36_k5", "f32", 40, 4, 2, 36, k=5),
    W("f32_F16_C64_one_clip", "f32", 16, 1, 3, 64),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_small_elementwise(cuda_device, w):
    run_case(w)


@pytest.mark.parametrize("w", synth.WORKLOADS[1:], ids=lambda w: w.name)
def test_full_size_sampled_positions(cuda_device, w):
    run_case(w, positions=sample_positions(w.P, count=2))


def test_result_does_not_depend_on_clip_count(cuda_device):
    """Neighbour padding makes every N give the unpartitioned conv (bit-identical)."""
    w = W("bf16_F128_C320", "bf16", 128, 8, 3, 320)
    x, wt, b = (to_device(synth.make(w, t), w.dtype) for t in ("conv_x", "conv_w", "conv_b"))
    ys = [vi.temporal_conv(x, wt, b, N=n) for n in (1, 2, 8, 64)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y, ys[0])


@pytest.mark.parametrize("tiles", [1, 2, 4])
@pytest.mark.parametrize("w", [W("bf16_F48_C64_odd_tiles", "bf16", 48, 3, 5, 64),
                               W("bf16_F200_C320_ragged", "bf16", 200, 8, 3, 320),
                               W("bf16_F24_C320_k1", "bf16", 24, 3, 3, 320, k=1)],
                         ids=lambda w: w.name)
def test_one_and_two_tiles_per_job(cuda_device, w, tiles):
    """Every job form of the tensor-core conv: one 128-frame tile per job, two
    sharing every weight stage, or a CTA pair with two tiles per CTA (M = 256,
    each CTA holding half the weight rows); odd tile counts leave zero tiles."""
    from clip_temporal_modules_b200._binding import conv_forced_tiles
    x, wt, b = (synth.make(w, t) for t in ("conv_x", "conv_w", "conv_b"))
    dx, dw, db = (to_device(a, w.dtype) for a in (x, wt, b))
    y = conv_forced_tiles(dx, dw, db, N=w.N, tiles=tiles)
    torch.cuda.synchronize()
    vi.take_device_errors()
    ref = oracle.temporal_conv(x, wt, b, w.F, w.N, w.k)
    assert_close(from_device(y), ref, w.dtype, "conv", w.name)
