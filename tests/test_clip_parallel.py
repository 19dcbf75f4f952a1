"""The exchange of clip parallelism (frames sharded over ranks), on CPU with
gloo: every rank must receive, in place in its halo-padded storage, exactly
the frames the one-GPU layout has next to its shard (zeros past the video
ends), the video's global frames, and every shard's GroupNorm statistics in
rank order; and the frame blocks that need no halo must be launched before
the halo exchange completes.

Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
write-up), clip-parallelism paragraphs (neighbour context and global frames
exchanged between devices before the temporal modules run)."""
import os
import socket
import time

import pytest
import torch
import torch.multiprocessing as mp

from clip_temporal_modules_b200.clip_parallel import (PART_BOUNDARY, PART_INTERIOR, ClipParallel,
                                                      ShardLayout, extended_from_full,
                                                      global_frame_index)


def test_layout_and_global_frames():
    lay = ShardLayout(F=128, N=8, world=4, rank=2)
    assert (lay.F_loc, lay.N_loc, lay.f0, lay.clip0) == (32, 2, 64, 4)
    assert global_frame_index(128, 16) == list(range(0, 128, 8))
    assert global_frame_index(100, 16) == [6 * j for j in range(16)]
    assert global_frame_index(64, 0) == []
    with pytest.raises(ValueError):
        ShardLayout(F=128, N=8, world=3, rank=0)


def test_extended_from_full_pads_with_zeros_at_the_ends():
    full = torch.arange(2 * 10 * 3, dtype=torch.float32).reshape(2, 10, 3) + 1
    e = extended_from_full(full, 0, 5, 2)
    assert e.shape == (2, 9, 3)
    assert torch.all(e[:, :2] == 0) and torch.equal(e[:, 2:9], full[:, 0:7])
    e = extended_from_full(full, 5, 10, 2)
    assert torch.equal(e[:, :7], full[:, 3:10]) and torch.all(e[:, 7:] == 0)


def test_padded_storage_puts_the_shard_between_zero_halos():
    x = torch.randn(3, 16, 4)
    p = ClipParallel.padded(x, 2)
    assert p.shape == (3, 20, 4)
    assert torch.equal(p[:, 2:18], x) and torch.all(p[:, :2] == 0) and torch.all(p[:, 18:] == 0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _spawn(target, world, *extra):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q) + extra) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    return dict(q.get(timeout=5) for _ in range(world))


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        F, N, P, C, ng = 64, 16, 3, 8, 16
        g = torch.Generator().manual_seed(7)
        full = torch.randn(P, F, C, generator=g)                # the same on every rank
        cp = ClipParallel(F, N, n_global=ng)
        lay = cp.lay
        f0, f1 = lay.f0, lay.f0 + lay.F_loc
        x = full[:, f0:f1].contiguous()
        ok = True
        for h in (1, 2, 8):
            xp = ClipParallel.padded(x, h)
            ok &= cp.halo(xp, h) is xp                         # in place
            ok &= torch.equal(xp, extended_from_full(full, f0, f1, h))
        ok &= torch.equal(cp.global_frames(x), full[:, global_frame_index(F, ng)])
        xp = ClipParallel.padded(x, 8)
        ok &= torch.equal(cp.global_frames(xp, 8), full[:, global_frame_index(F, ng)])
        stats = torch.full((4, 2), float(rank), dtype=torch.float64)
        got = cp.gather_stats(stats)
        ok &= got.shape == (world, 4, 2) and all(bool(torch.all(got[r] == r)) for r in range(world))
        q.put((rank, bool(ok)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_exchange_delivers_the_one_gpu_neighbourhood_gloo(world):
    assert _spawn(_rank_main, world) == {r: True for r in range(world)}


class _Recorder:
    """Stand-in for the shard kernels: records each launch's part and time
    and the halo rows it would read at that moment."""

    def __init__(self):
        self.log = []

    def conv(self, x_pad, w, b, out, *, part):
        self.log.append(("conv", part, time.monotonic(), x_pad.clone()))

    def attn(self, q, k_pad, v_pad, kg, vg, out, *, lay, heads, n_pre, n_post, n_global, part):
        self.log.append(("attn", part, time.monotonic(), k_pad.clone()))


def _overlap_main(rank, world, port, q, delay):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        F, N, P, C = 64, 4, 2, 8
        full = torch.randn(P, F, C, generator=torch.Generator().manual_seed(3))
        rec = _Recorder()
        cp = ClipParallel(F, N, n_global=0, kernels=rec)
        lay = cp.lay
        f0, f1 = lay.f0, lay.f0 + lay.F_loc
        x = ClipParallel.padded(full[:, f0:f1].contiguous(), 1)
        kv = ClipParallel.padded(full[:, f0:f1].contiguous(), 8)
        w = torch.zeros(C, C, 3)
        if rank == 1:
            time.sleep(delay)                 # the neighbour joins the exchange late
        t0 = time.monotonic()
        cp.temporal_conv(x, w, torch.zeros(C))
        t1 = time.monotonic()
        cp.dual_attn(full[:, f0:f1].contiguous(), kv, kv.clone())
        res = {"t0": t0, "t1": t1,
               "log": [(name, part, t, bool(torch.equal(
                   snap, extended_from_full(full, f0, f1, 1 if name == "conv" else 8))))
                       for name, part, t, snap in rec.log]}
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


def test_interior_launch_does_not_wait_for_the_halo_exchange_gloo():
    """Rank 1 joins the halo exchange `delay` seconds late.  Rank 0 must launch
    its interior blocks at once (before its halo rows have arrived), and its
    boundary blocks only once the halo rows are in place."""
    delay = 1.0
    res = _spawn(_overlap_main, 2, delay)[0]
    log = res["log"]
    assert [(n, p) for n, p, _, _ in log] == [("conv", PART_INTERIOR), ("conv", PART_BOUNDARY),
                                             ("attn", PART_INTERIOR), ("attn", PART_BOUNDARY)]
    (_, _, t_int, halo_in_at_interior), (_, _, t_bnd, halo_in_at_boundary) = log[0], log[1]
    assert t_int - res["t0"] < 0.5 * delay        # not held back by the late neighbour
    assert t_bnd - res["t0"] >= 0.5 * delay       # held back until the halo arrived
    assert not halo_in_at_interior and halo_in_at_boundary
    assert log[3][3]                             # attention's boundary saw its halos too
