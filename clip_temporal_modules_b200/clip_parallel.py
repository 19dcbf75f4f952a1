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
clips.  The tensors whose neighbour frames a module reads (k and v of the
attention, x of the conv) are kept in halo-padded storage, [P][F_loc + 2h][C]
with the shard at rows [h, h + F_loc): the exchange writes only the halo
rows, so no call copies the shard.  Per call:
  global     every rank puts the global frames j floor(F/n_global) it owns
             into a zero [P][n_global][C] tensor; one all_reduce (a sum in
             which each frame has exactly one non-zero term, so it is exact)
             gives every rank all of them, for k and v together
  halo       each rank sends its first h frames to rank r-1 and its last h
             frames to rank r+1 and receives the matching rows (zeros at the
             video ends, where no rank sends)
  GroupNorm  an all_gather of every shard's per-group (mean, var)
Overlap: the exchanges are posted asynchronously; the frame blocks that read
no halo row (VI_PART_INTERIOR) are launched as soon as the global frames are
in, before the halos have arrived, and the boundary blocks after.  On GPUs
everything is ordered on one CUDA stream (the caller's, if given): NCCL works
on its own stream and the waits are stream waits, so the host never blocks.
The results equal the one-GPU calls on the whole video.
"""
from __future__ import annotations

import contextlib
from dataclasses import dataclass

ATTN_HALO = 8            # frames of context on each side the attention kernel reads
PART_ALL, PART_INTERIOR, PART_BOUNDARY = 0, 1, 2


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


class LibviKernels:
    """The per-shard compute: libvi's shard calls (argument marshalling only)."""

    def attn(self, q, k_pad, v_pad, kg, vg, out, *, lay, heads, n_pre, n_post, n_global, part):
        from ._binding import dual_attn_shard
        dual_attn_shard(q, k_pad, v_pad, kg, vg, out, N_loc=lay.N_loc, clip0=lay.clip0,
                        N=lay.N, heads=heads, n_pre=n_pre, n_post=n_post, n_global=n_global,
                        part=part)

    def conv(self, x_pad, w, b, out, *, part):
        from ._binding import temporal_conv_shard
        temporal_conv_shard(x_pad, w, b, out, part=part)

    def gn_stats(self, x, *, groups):
        from ._binding import groupnorm_shard_stats
        return groupnorm_shard_stats(x, groups=groups)

    def gn_apply(self, x, stats, gamma, beta, out, *, eps):
        from ._binding import groupnorm_shard_apply
        return groupnorm_shard_apply(x, stats, gamma, beta, out, eps=eps)


class _Halo:
    """A posted halo exchange of one padded tensor; finish() waits for it
    (a stream wait under NCCL) and writes the received rows in place."""

    def __init__(self, x_pad, h, reqs, recv_lo, recv_hi, sends=()):
        self.x_pad, self.h, self.reqs = x_pad, h, reqs
        self.recv_lo, self.recv_hi = recv_lo, recv_hi
        self.sends = sends                     # kept alive until the sends are done

    def finish(self):
        for r in self.reqs:
            r.wait()
        h, F_pad = self.h, self.x_pad.shape[1]
        if self.recv_lo is not None:
            self.x_pad[:, :h].copy_(self.recv_lo)
        if self.recv_hi is not None:
            self.x_pad[:, F_pad - h:].copy_(self.recv_hi)
        self.reqs, self.sends = [], ()


class ClipParallel:
    """Per-rank driver of the temporal modules of a video sharded along frames.

    q, the GroupNorm input and the outputs are this rank's [P][F_loc][C]
    shards; k, v (attention) and x (conv) are halo-padded [P][F_loc + 2h][C]
    (see `padded`).  bf16 CUDA tensors for the module calls; the exchange
    methods also take CPU tensors under gloo.  `kernels` computes a shard
    (libvi by default)."""

    def __init__(self, F: int, N: int, *, heads: int = 1, n_pre: int = 8, n_post: int = 8,
                 n_global: int = 16, groups: int = 32, eps: float = 1e-5, group=None,
                 kernels=None):
        import torch.distributed as dist
        self.group = group
        world = dist.get_world_size(group) if dist.is_initialized() else 1
        rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.lay = ShardLayout(F, N, world, rank)
        self.heads, self.n_pre, self.n_post, self.n_global = heads, n_pre, n_post, n_global
        self.groups, self.eps = groups, eps
        self.kernels = kernels if kernels is not None else LibviKernels()
        gidx = global_frame_index(F, n_global)
        f0, f1 = self.lay.f0, self.lay.f0 + self.lay.F_loc
        owned = [(j, g - f0) for j, g in enumerate(gidx) if f0 <= g < f1]
        self.own_slots = [j for j, _ in owned]          # positions in the global list
        self.own_frames = [fl for _, fl in owned]       # shard-local frame indices
        self._index_cache = {}

    # ---- storage -------------------------------------------------------------------
    @staticmethod
    def padded(x, h: int):
        """Halo-padded storage of a dense shard: [P][F_loc][C] -> [P][F_loc + 2h][C],
        the shard at rows [h, h + F_loc), the halo rows zero.  One copy, for a
        caller whose shard is dense; keep the result as the shard's storage."""
        import torch
        P, F_loc, C = x.shape
        out = torch.zeros((P, F_loc + 2 * h, C), dtype=x.dtype, device=x.device)
        out[:, h:h + F_loc] = x
        return out

    def _peer(self, r: int) -> int:
        import torch.distributed as dist
        return dist.get_global_rank(self.group, r) if self.group is not None else r

    # ---- exchanges -----------------------------------------------------------------
    def start_halo(self, x_pad, h: int) -> _Halo:
        """Post the exchange of the h frames on each side of a padded shard."""
        import torch.distributed as dist
        lay = self.lay
        P, F_pad, C = x_pad.shape
        F_loc = F_pad - 2 * h
        if h > F_loc:
            raise ValueError("halo wider than a shard")
        if h == 0 or lay.world == 1:
            return _Halo(x_pad, h, [], None, None)
        ops, recv_lo, recv_hi, send_lo, send_hi = [], None, None, None, None
        if lay.rank > 0:                       # my first h frames <-> rank-1's last h
            send_lo = x_pad[:, h:2 * h].contiguous()
            recv_lo = x_pad.new_empty((P, h, C))
            ops += [dist.P2POp(dist.isend, send_lo, self._peer(lay.rank - 1), self.group),
                    dist.P2POp(dist.irecv, recv_lo, self._peer(lay.rank - 1), self.group)]
        if lay.rank < lay.world - 1:           # my last h frames <-> rank+1's first h
            send_hi = x_pad[:, F_loc:F_loc + h].contiguous()
            recv_hi = x_pad.new_empty((P, h, C))
            ops += [dist.P2POp(dist.isend, send_hi, self._peer(lay.rank + 1), self.group),
                    dist.P2POp(dist.irecv, recv_hi, self._peer(lay.rank + 1), self.group)]
        return _Halo(x_pad, h, dist.batch_isend_irecv(ops), recv_lo, recv_hi, (send_lo, send_hi))

    def start_global(self, tensors, h: int = 0):
        """Post the gather of the video's global frames of each [P][F_loc (+2h)][C]
        tensor (shard at rows [h, h + F_loc)).  Returns (work, stacked) where
        stacked[i] is tensor i's [P][n_global][C] once work is waited on."""
        import torch
        import torch.distributed as dist
        x0 = tensors[0]
        P, _, C = x0.shape
        stacked = x0.new_zeros((len(tensors), P, self.n_global, C))
        if self.own_frames:
            key = (str(x0.device), h)
            if key not in self._index_cache:     # built once per device and halo width
                self._index_cache[key] = (
                    torch.tensor([f + h for f in self.own_frames], device=x0.device),
                    torch.tensor(self.own_slots, device=x0.device))
            src, dst = self._index_cache[key]
            for i, t in enumerate(tensors):
                stacked[i].index_copy_(1, dst, t.index_select(1, src))
        if self.lay.world == 1:
            return None, stacked
        return dist.all_reduce(stacked, group=self.group, async_op=True), stacked

    def halo(self, x_pad, h: int):
        """Exchange the halo rows of a padded shard in place (blocking form)."""
        ex = self.start_halo(x_pad, h)
        ex.finish()
        return x_pad

    def global_frames(self, x, h: int = 0):
        """[P][F_loc (+2h)][C] -> [P][n_global][C]: the video's global frames, on every rank."""
        work, stacked = self.start_global([x], h)
        if work is not None:
            work.wait()
        return stacked[0]

    def gather_stats(self, stats):
        """This shard's [groups][2] statistics -> every shard's, [W][groups][2]."""
        import torch
        import torch.distributed as dist
        stats = stats.contiguous()
        if self.lay.world == 1:
            return stats.unsqueeze(0)
        out = torch.empty((self.lay.world * stats.shape[0],) + tuple(stats.shape[1:]),
                          dtype=stats.dtype, device=stats.device)
        dist.all_gather_into_tensor(out, stats, group=self.group)   # shards along dim 0
        return out.view((self.lay.world,) + tuple(stats.shape))

    # ---- modules -------------------------------------------------------------------
    @staticmethod
    def _on(stream):
        """Order everything (allocations, copies, collectives, kernels) on `stream`."""
        if stream is None:
            return contextlib.nullcontext()
        import torch
        return torch.cuda.stream(stream)

    def dual_attn(self, q, k_pad, v_pad, out=None, stream=None):
        """Attention of this shard; k_pad, v_pad halo-padded with h = 8."""
        import torch
        kw = dict(lay=self.lay, heads=self.heads, n_pre=self.n_pre, n_post=self.n_post,
                  n_global=self.n_global)
        with self._on(stream):
            out = torch.empty_like(q) if out is None else out
            work, kv_g = (self.start_global([k_pad, v_pad], ATTN_HALO) if self.n_global
                          else (None, None))
            hk, hv = self.start_halo(k_pad, ATTN_HALO), self.start_halo(v_pad, ATTN_HALO)
            if work is not None:
                work.wait()
            kg, vg = (kv_g[0], kv_g[1]) if kv_g is not None else (None, None)
            self.kernels.attn(q, k_pad, v_pad, kg, vg, out, part=PART_INTERIOR, **kw)
            hk.finish()
            hv.finish()
            self.kernels.attn(q, k_pad, v_pad, kg, vg, out, part=PART_BOUNDARY, **kw)
        return out

    def temporal_conv(self, x_pad, w, b, out=None, stream=None):
        """Conv of this shard; x_pad halo-padded with h = k // 2."""
        import torch
        h = w.shape[2] // 2
        with self._on(stream):
            P, F_pad, C = x_pad.shape
            if out is None:
                out = torch.empty((P, F_pad - 2 * h, C), dtype=x_pad.dtype, device=x_pad.device)
            hx = self.start_halo(x_pad, h)
            self.kernels.conv(x_pad, w, b, out, part=PART_INTERIOR)
            hx.finish()
            self.kernels.conv(x_pad, w, b, out, part=PART_BOUNDARY)
        return out

    def groupnorm(self, x, gamma, beta, out=None, stream=None):
        """GroupNorm of this shard with the statistics of the whole video."""
        with self._on(stream):
            stats = self.kernels.gn_stats(x, groups=self.groups)
            return self.kernels.gn_apply(x, self.gather_stats(stats), gamma, beta, out,
                                         eps=self.eps)
