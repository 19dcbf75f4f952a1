"""The exchange of clip parallelism (frames sharded over ranks), on CPU with
gloo: every rank must receive exactly the frames the one-GPU layout would
have next to its shard (zeros past the video ends), the video's global frames,
and every shard's GroupNorm statistics in rank order.

Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
write-up), clip-parallelism paragraphs (neighbour context and global frames
exchanged between devices before the temporal modules run)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from clip_temporal_modules_b200.clip_parallel import (ClipParallel, ShardLayout,
                                                      extended_from_full, global_frame_index)


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


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


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
        x = full[:, lay.f0:lay.f0 + lay.F_loc].contiguous()
        ok = True
        for h in (1, 2, 8):
            ok &= torch.equal(cp.halo(x, h), extended_from_full(full, lay.f0, lay.f0 + lay.F_loc, h))
        ok &= torch.equal(cp.global_frames(x), full[:, global_frame_index(F, ng)])
        stats = torch.full((4, 2), float(rank), dtype=torch.float64)
        got = cp.gather_stats(stats)
        ok &= got.shape == (world, 4, 2) and all(bool(torch.all(got[r] == r)) for r in range(world))
        q.put((rank, bool(ok)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_exchange_delivers_the_one_gpu_neighbourhood_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = dict(q.get(timeout=5) for _ in range(world))
    assert res == {r: True for r in range(world)}
