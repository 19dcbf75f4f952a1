"""The per-shard kernels of clip parallelism on one GPU: W shards of a video
are emulated in one process (each shard's halo-padded storage is cut from the
whole tensor, which is what the exchange delivers: see test_clip_parallel.py),
run through vi_dual_attn_shard / vi_temporal_conv_shard / vi_groupnorm_shard_*,
and stitched back.  The interior and boundary parts of a shard together give
the whole-shard call.  Attention must equal the one-GPU call bit for bit (same
keys in the same order); the conv and GroupNorm must match the one-GPU calls
and the fp64 oracle within the bf16 tolerances (the conv's CTAs and the
statistics merge may sum in another order).

Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
write-up), clip-parallelism, attention-, conv- and GroupNorm-module paragraphs."""
import numpy as np
import pytest
import torch

import clip_temporal_modules_b200 as vi
from clip_temporal_modules_b200._binding import (dual_attn_shard, groupnorm_shard_apply,
                                                 groupnorm_shard_stats, temporal_conv_shard)
from clip_temporal_modules_b200.clip_parallel import (PART_BOUNDARY, PART_INTERIOR, ClipParallel,
                                                      ShardLayout, extended_from_full,
                                                      global_frame_index)
import oracle
import synth
from parity import assert_close, from_device, to_device

pytestmark = pytest.mark.gpu

CASES = [dict(F=256, N=16, P=5, heads=2, world=4, n_pre=8, n_post=8, n_global=16),
         dict(F=256, N=16, P=3, heads=5, world=2, n_pre=3, n_post=5, n_global=7),
         dict(F=128, N=8, P=4, heads=1, world=8, n_pre=8, n_post=8, n_global=0)]


def _w(c, name="cp"):
    return synth.Workload(name, "bf16", F=c["F"], N=c["N"], P=c["P"], C=64 * c["heads"],
                          heads=c["heads"], d=64, n_pre=c["n_pre"], n_post=c["n_post"],
                          n_global=c["n_global"])


@pytest.mark.parametrize("c", CASES, ids=lambda c: f"W{c['world']}_ng{c['n_global']}")
def test_sharded_attention_equals_one_gpu(cuda_device, c):
    w = _w(c)
    q, k, v = (to_device(synth.make(w, t), w.dtype) for t in ("q", "k", "v"))
    whole = vi.dual_attn(q, k, v, N=w.N, heads=w.heads, n_pre=w.n_pre, n_post=w.n_post,
                         n_global=w.n_global)
    gidx = global_frame_index(w.F, w.n_global)
    kg, vg = k[:, gidx].contiguous(), v[:, gidx].contiguous()
    parts, split = [], []
    for r in range(c["world"]):
        lay = ShardLayout(w.F, w.N, c["world"], r)
        f0, f1 = lay.f0, lay.f0 + lay.F_loc
        args = (q[:, f0:f1].contiguous(), extended_from_full(k, f0, f1, 8),
                extended_from_full(v, f0, f1, 8), kg, vg)
        kw = dict(N_loc=lay.N_loc, clip0=lay.clip0, N=w.N, heads=w.heads, n_pre=w.n_pre,
                  n_post=w.n_post, n_global=w.n_global)
        parts.append(dual_attn_shard(*args, **kw))
        o = torch.full_like(args[0], float("nan"))
        dual_attn_shard(*args, o, part=PART_INTERIOR, **kw)
        dual_attn_shard(*args, o, part=PART_BOUNDARY, **kw)
        split.append(o)
    torch.cuda.synchronize()
    vi.take_device_errors()
    got = torch.cat(parts, dim=1)
    assert torch.equal(got.view(torch.int16), whole.view(torch.int16))
    assert torch.equal(torch.cat(split, dim=1).view(torch.int16), whole.view(torch.int16))


@pytest.mark.parametrize("F,world,k", [(256, 4, 3), (256, 2, 5), (256, 8, 1), (1024, 2, 3),
                                       (576, 2, 3)])
def test_sharded_conv_matches_one_gpu_and_oracle(cuda_device, F, world, k):
    """Shards of one, two and several frame blocks, a ragged last block
    (F_loc = 288), and the interior + boundary split."""
    w = synth.Workload("cp_conv", "bf16", F=F, N=F // 16, P=3, C=320, heads=5, d=64, k=k)
    x, wt, b = (synth.make(w, t) for t in ("conv_x", "conv_w", "conv_b"))
    dx, dw, db = (to_device(a, w.dtype) for a in (x, wt, b))
    whole = vi.temporal_conv(dx, dw, db, N=w.N)
    parts, split = [], []
    for r in range(world):
        lay = ShardLayout(w.F, w.N, world, r)
        xe = extended_from_full(dx, lay.f0, lay.f0 + lay.F_loc, k // 2)
        parts.append(temporal_conv_shard(xe, dw, db))
        y = torch.full((w.P, lay.F_loc, w.C), float("nan"), dtype=dx.dtype, device=dx.device)
        temporal_conv_shard(xe, dw, db, y, part=PART_INTERIOR)
        temporal_conv_shard(xe, dw, db, y, part=PART_BOUNDARY)
        split.append(y)
    torch.cuda.synchronize()
    vi.take_device_errors()
    ref = oracle.temporal_conv(x, wt, b, w.F, w.N, k)
    for got in (from_device(torch.cat(parts, dim=1)), from_device(torch.cat(split, dim=1))):
        assert np.max(np.abs(got - from_device(whole))) <= 2e-2
        assert_close(got, ref, w.dtype, "conv", "sharded conv")


@pytest.mark.parametrize("world", [2, 4])
def test_sharded_groupnorm_matches_one_gpu_and_oracle(cuda_device, world):
    w = synth.Workload("cp_gn", "bf16", F=256, N=16, P=6, C=320, heads=5, d=64)
    x, g, bt = (synth.make(w, t) for t in ("gn_x", "gn_gamma", "gn_beta"))
    dx, dg, dbt = (to_device(a, w.dtype) for a in (x, g, bt))
    whole = vi.groupnorm_global(dx, dg, dbt, N=w.N, groups=w.groups)
    lays = [ShardLayout(w.F, w.N, world, r) for r in range(world)]
    shards = [dx[:, l.f0:l.f0 + l.F_loc].contiguous() for l in lays]
    stats = torch.stack([groupnorm_shard_stats(s, groups=w.groups) for s in shards])
    parts = [groupnorm_shard_apply(s, stats, dg, dbt) for s in shards]
    torch.cuda.synchronize()
    vi.take_device_errors()
    got = from_device(torch.cat(parts, dim=1))
    ref, mean, var = oracle.groupnorm_global(x, g, bt, w.F, w.N, w.groups, w.eps)
    st = stats.cpu().numpy()
    # merged statistics against the oracle's fp64 ones (the kernels accumulate
    # runs of 32 elements in fp32 before folding into fp64)
    np.testing.assert_allclose(st[:, :, 0].mean(axis=0), mean, rtol=0, atol=1e-6)
    pooled = (st[:, :, 1] + (st[:, :, 0] - st[:, :, 0].mean(axis=0)) ** 2).mean(axis=0)
    np.testing.assert_allclose(pooled, var, rtol=1e-6, atol=0)
    assert np.max(np.abs(got - from_device(whole))) <= 2e-2
    assert_close(got, ref, w.dtype, "gn", "sharded GroupNorm")


@pytest.mark.parametrize("C,groups", [(320, 32), (64, 32)])
def test_shard_stats_into_gathered_slots(cuda_device, C, groups):
    """Each shard's statistics written into its slot of one [W][groups][2]
    tensor (what an all-gather delivers) equal the separately returned ones
    bit for bit, and the apply pass on them matches the one-GPU call.  C=320
    takes the ring path, whose apply threads merge the shards' records
    themselves; C=64 with 32 groups (2 channels per group) the scalar path,
    which merges in a kernel of its own."""
    world = 4
    w = synth.Workload("cp_gn_slots", "bf16", F=256, N=16, P=5, C=C, heads=C // 64, d=64,
                       groups=groups)
    x, g, bt = (synth.make(w, t) for t in ("gn_x", "gn_gamma", "gn_beta"))
    dx, dg, dbt = (to_device(a, w.dtype) for a in (x, g, bt))
    whole = vi.groupnorm_global(dx, dg, dbt, N=w.N, groups=w.groups)
    lays = [ShardLayout(w.F, w.N, world, r) for r in range(world)]
    shards = [dx[:, l.f0:l.f0 + l.F_loc].contiguous() for l in lays]
    gathered = torch.full((world, w.groups, 2), float("nan"), dtype=torch.float64,
                          device=dx.device)
    for i, sh in enumerate(shards):
        groupnorm_shard_stats(sh, groups=w.groups, out=gathered[i])
    single = torch.stack([groupnorm_shard_stats(sh, groups=w.groups) for sh in shards])
    parts = [groupnorm_shard_apply(sh, gathered, dg, dbt) for sh in shards]
    torch.cuda.synchronize()
    vi.take_device_errors()
    assert torch.equal(gathered, single)
    got = from_device(torch.cat(parts, dim=1))
    ref, _, _ = oracle.groupnorm_global(x, g, bt, w.F, w.N, w.groups, w.eps)
    assert np.max(np.abs(got - from_device(whole))) <= 2e-2
    assert_close(got, ref, w.dtype, "gn", "sharded GroupNorm from gathered slots")


def test_shard_stats_out_slot_is_checked(cuda_device):
    x = torch.zeros((2, 16, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        groupnorm_shard_stats(x, groups=32, out=torch.empty((32, 3), dtype=torch.float64,
                                                            device="cuda"))
    with pytest.raises(ValueError):
        groupnorm_shard_stats(x, groups=32, out=torch.empty((32, 2), dtype=torch.float32,
                                                            device="cuda"))


def _single_rank_run(t, w, stream=None):
    cp = ClipParallel(w.F, w.N, heads=w.heads, groups=w.groups)
    k = w.k // 2
    a = cp.dual_attn(t["q"], ClipParallel.padded(t["k"], 8), ClipParallel.padded(t["v"], 8),
                     stream=stream)
    y = cp.temporal_conv(ClipParallel.padded(t["conv_x"], k), t["conv_w"], t["conv_b"],
                         stream=stream)
    z = cp.groupnorm(t["gn_x"], t["gn_gamma"], t["gn_beta"], stream=stream)
    return a, y, z


def test_clip_parallel_single_rank_equals_whole_video_calls(cuda_device):
    """ClipParallel without a process group (one rank): its exchange degenerates
    to zero halos and all frames, and each module equals the one-GPU call."""
    w = _w(CASES[0])
    t = {n: to_device(synth.make(w, n), w.dtype) for n in
         ("q", "k", "v", "conv_x", "conv_w", "conv_b", "gn_x", "gn_gamma", "gn_beta")}
    a, y, z = _single_rank_run(t, w)
    torch.cuda.synchronize()
    vi.take_device_errors()
    assert torch.equal(a, vi.dual_attn(t["q"], t["k"], t["v"], N=w.N, heads=w.heads))
    yy = vi.temporal_conv(t["conv_x"], t["conv_w"], t["conv_b"], N=w.N)
    assert (y.float() - yy.float()).abs().max().item() <= 2e-2
    zz = vi.groupnorm_global(t["gn_x"], t["gn_gamma"], t["gn_beta"], N=w.N, groups=w.groups)
    assert (z.float() - zz.float()).abs().max().item() <= 2e-2


def test_clip_parallel_on_a_caller_stream(cuda_device):
    """With a caller's stream every allocation, copy, exchange and kernel is
    ordered on it: the inputs are produced on that stream just before the
    calls, and the results equal those on the default stream."""
    w = _w(CASES[0])
    host = {n: synth.make(w, n) for n in
            ("q", "k", "v", "conv_x", "conv_w", "conv_b", "gn_x", "gn_gamma", "gn_beta")}
    ref = _single_rank_run({n: to_device(a, w.dtype) for n, a in host.items()}, w)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        # produced on s, consumed on s: nothing orders them against the default stream
        t = {n: to_device(a, w.dtype) * 1 for n, a in host.items()}
    got = _single_rank_run(t, w, stream=s)
    s.synchronize()
    vi.take_device_errors()
    assert torch.equal(got[0], ref[0])
    for g, r in zip(got[1:], ref[1:]):
        assert (g.float() - r.float()).abs().max().item() <= 2e-2
