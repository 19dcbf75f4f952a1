"""Clip parallelism over several GPUs: a video cut along frames, one shard per rank.

"Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com write-up),
clip-parallelism paragraphs: each device holds some clips of the video; before
its temporal modules run it receives the frames its clips need from the
neighbouring devices (the end of the previous clip, the start of the next one)
and the globally sampled frames; GroupNorm statistics are exchanged.  This
module is that exchange, written with torch.distributed (NCCL between GPUs;
gloo works for the exchange alone, on CPU tensors), around the per-shard
kernels of libvi (vi_dual_attn_shard, vi_temporal_conv_shard,
vi_groupnorm_shard_stats / _apply).

Rank r holds frames [r F/W, (r+1) F/W) of every position, a whole number of
clips.  The exchanges, per call:
  halo       each rank sends its first h frames to rank r-1 and its last h
             frames to rank r+1 (h = 8 for attention, k/2 for the conv); the
             ranks at the video ends pad with zeros
  global     every rank contributes the global frames j floor(F/n_global) it
             owns; an all_gather gives every rank all of them
  GroupNorm  an all_gather of every shard's per-group (mean, var)
The exchange is done before the kernels run (no overlap with the own-clip
compute in this version).  The results equal the one-GPU calls on the whole
video.
"""
from __future__ import annotations

from dataclasses import dataclass

ATTN_HALO = 8            # frames of context on each side the attention kernel reads


@dataclass(frozen=True)
class ShardLayout:
    """Which frames and clips of an F-frame, N-clip video rank `rank` of `world` holds."""
    F: int
    N: int
    world: int
    rank: int

    def __post_init__(self):
        if self.F % self.N or self.N % self.world:
            raise ValueError("clips must divide frames and ranks must divide clips")

    @property
    def F_loc(self) -> int:
        return self.F // self.world

    @property
    def N_loc(self) -> int:
        return self.N // self.world

    @property
    def f0(self) -> int:
        return self.rank * self.F_loc

    @property
    def clip0(self) -> int:
        return self.rank * self.N_loc


def global_frame_index(F: int, n_global: int):
    """Frames sampled over the whole video: j * floor(F / n_global), j < n_global."""
    if n_global == 0:
        return []
    gs = F // n_global
    return [j * gs for j in range(n_global)]


def extended_from_full(full, f0: int, f1: int, h: int):
    """Reference of the halo exchange: frames [f0 - h, f1 + h) of a whole
    [P][F][C] tensor, with zeros outside [0, F).  Used by the tests as the
    definition of what the exchange must deliver."""
    import torch
    P, F, C = full.shape
    out = torch.zeros((P, f1 - f0 + 2 * h, C), dtype=full.dtype, device=full.device)
    a, b = max(f0 - h, 0), min(f1 + h, F)
    out[:, a - (f0 - h):b - (f0 - h)] = full[:, a:b]
    return out


class ClipParallel:
    """Per-rank driver of the temporal modules of a video sharded along frames.

    Tensors are this rank's [P][F_loc][C] shards (bf16 CUDA tensors for the
    module calls; the exchange methods also take CPU tensors under gloo)."""

    def __init__(self, F: int, N: int, *, heads: int = 1, n_pre: int = 8, n_post: int = 8,
                 n_global: int = 16, groups: int = 32, eps: float = 1e-5, group=None):
        import torch.distributed as dist
        self.group = group
        world = dist.get_world_size(group) if dist.is_initialized() else 1
        rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.lay = ShardLayout(F, N, world, rank)
        self.heads, self.n_pre, self.n_post, self.n_global = heads, n_pre, n_post, n_global
        self.groups, self.eps = groups, eps
        gidx = global_frame_index(F, n_global)
        f0, f1 = self.lay.f0, self.lay.f0 + self.lay.F_loc
        self.owned = [(j, g - f0) for j, g in enumerate(gidx) if f0 <= g < f1]

    # ---- exchanges ---------------------------------------------------------------
    def halo(self, x, h: int):
        """[P][F_loc][C] -> [P][F_loc + 2h][C] with the neighbours' frames (zeros at the ends)."""
        import torch
        import torch.distributed as dist
        lay = self.lay
        if h > lay.F_loc:
            raise ValueError("halo wider than a shard")
        P, F_loc, C = x.shape
        ext = torch.zeros((P, F_loc + 2 * h, C), dtype=x.dtype, device=x.device)
        ext[:, h:h + F_loc] = x
        if h == 0 or lay.world == 1:
            return ext
        send_lo = x[:, :h].contiguous()               # -> rank - 1, its post-halo
        send_hi = x[:, F_loc - h:].contiguous()       # -> rank + 1, its pre-halo
        recv_lo = torch.empty_like(send_lo)           # <- rank - 1, my pre-halo
        recv_hi = torch.empty_like(send_hi)           # <- rank + 1, my post-halo
        peer = lambda r: dist.get_global_rank(self.group, r) if self.group is not None else r  # noqa: E731
        ops = []
        if lay.rank > 0:
            ops += [dist.P2POp(dist.isend, send_lo, peer(lay.rank - 1), self.group),
                    dist.P2POp(dist.irecv, recv_lo, peer(lay.rank - 1), self.group)]
        if lay.rank < lay.world - 1:
            ops += [dist.P2POp(dist.isend, send_hi, peer(lay.rank + 1), self.group),
                    dist.P2POp(dist.irecv, recv_hi, peer(lay.rank + 1), self.group)]
        for req in dist.batch_isend_irecv(ops):
            req.wait()
        if lay.rank > 0:
            ext[:, :h] = recv_lo
        if lay.rank < lay.world - 1:
            ext[:, h + F_loc:] = recv_hi
        return ext

    def global_frames(self, x):
        """[P][F_loc][C] -> [P][n_global][C]: the video's global frames, on every rank."""
        import torch
        import torch.distributed as dist
        P, _, C = x.shape
        mine = torch.zeros((P, self.n_global, C), dtype=x.dtype, device=x.device)
        for j, fl in self.owned:
            mine[:, j] = x[:, fl]
        if self.lay.world == 1:
            return mine
        parts = [torch.empty_like(mine) for _ in range(self.lay.world)]
        dist.all_gather(parts, mine, group=self.group)
        out = torch.empty_like(mine)
        F_loc = self.lay.F_loc
        for j, g in enumerate(global_frame_index(self.lay.F, self.n_global)):
            out[:, j] = parts[g // F_loc][:, j]
        return out

    def gather_stats(self, stats):
        """This shard's [groups][2] statistics -> every shard's, [W][groups][2]."""
        import torch
        import torch.distributed as dist
        if self.lay.world == 1:
            return stats.unsqueeze(0).contiguous()
        parts = [torch.empty_like(stats) for _ in range(self.lay.world)]
        dist.all_gather(parts, stats.contiguous(), group=self.group)
        return torch.stack(parts).contiguous()

    # ---- modules -------------------------------------------------------------------
    def dual_attn(self, q, k, v, stream=None):
        from ._binding import dual_attn_shard
        lay = self.lay
        k_ext, v_ext = self.halo(k, ATTN_HALO), self.halo(v, ATTN_HALO)
        kg = self.global_frames(k) if self.n_global else None
        vg = self.global_frames(v) if self.n_global else None
        return dual_attn_shard(q, k_ext, v_ext, kg, vg, N_loc=lay.N_loc, clip0=lay.clip0,
                               N=lay.N, heads=self.heads, n_pre=self.n_pre, n_post=self.n_post,
                               n_global=self.n_global, stream=stream)

    def temporal_conv(self, x, w, b, stream=None):
        from ._binding import temporal_conv_shard
        return temporal_conv_shard(self.halo(x, w.shape[2] // 2), w, b, stream=stream)

    def groupnorm(self, x, gamma, beta, stream=None):
        from ._binding import groupnorm_shard_apply, groupnorm_shard_stats
        stats = groupnorm_shard_stats(x, groups=self.groups, stream=stream)
        return groupnorm_shard_apply(x, self.gather_stats(stats), gamma, beta, eps=self.eps,
                                     stream=stream)
