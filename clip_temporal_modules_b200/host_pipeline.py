"""Temporal modules on host-resident tensors, with copies overlapped with compute.

The three temporal modules of a clip-parallel video U-Net step (dual-domain
attention, neighbour-padded temporal conv, GroupNorm with global statistics;
"Video-Infinity: Distributed Long Video Generation", clip-parallelism
paragraphs) take latents that may live in host memory, e.g. when a serving
process stages them between denoising steps.  Moving them over PCIe costs far
more than the kernels, so this executor cuts the work into chunks of positions
and runs three CUDA streams:

  copy-in   host -> device: the GroupNorm input first (its statistics need the
            whole tensor), then q, k, v and the conv input chunk by chunk
  compute   GroupNorm once its input is resident, then attention and conv of
            each chunk as soon as that chunk has arrived
  copy-out  device -> host: each result chunk as soon as it is computed

Attention and the conv are independent per position (frames are contiguous per
position in the [P][F][C] layout), so a chunk of positions is a contiguous
slice.  Chunked attention equals the whole-tensor call bit for bit; the conv
may differ in the last bf16 bit, because which CTA takes a tile (and so the
order in which it sums its K-blocks in fp32) depends on the call's size.
Host->device and device->host copies use separate copy engines, so the step
costs about the larger of the two transfer volumes instead of their sum.

Host tensors must be pinned (page-locked) for the copies to be asynchronous.
"""
from __future__ import annotations

from dataclasses import dataclass

from ._binding import dual_attn, groupnorm_global, temporal_conv

_INPUTS = ("q", "k", "v", "conv_x", "conv_w", "conv_b", "gn_x", "gn_gamma", "gn_beta")
_OUTPUTS = ("out", "y", "z")


def chunk_bounds(P: int, chunks: int):
    """[p0, p1) ranges cutting P positions into `chunks` near-equal parts, in order."""
    chunks = max(1, min(int(chunks), P))
    base, extra = divmod(P, chunks)
    out, p0 = [], 0
    for i in range(chunks):
        p1 = p0 + base + (1 if i < extra else 0)
        out.append((p0, p1))
        p0 = p1
    return out


@dataclass(frozen=True)
class StepShape:
    """Shape of one step: latent [P][F][C], N clips, attention heads and context."""
    F: int
    N: int
    P: int
    C: int
    heads: int
    n_pre: int = 8
    n_post: int = 8
    n_global: int = 16
    k: int = 3
    groups: int = 32
    eps: float = 1e-5


class HostPipeline:
    """Runs attention, conv and GroupNorm on pinned host tensors of one shape.

    Device buffers for every input and output are allocated once, at
    construction, on `device`; `run` may be called repeatedly.  `chunks` is the
    number of position chunks the copies and the per-position modules are cut
    into (clamped to P).
    """

    def __init__(self, shape: StepShape, device, dtype, chunks: int = 8):
        import torch
        self.s = shape
        self.device = torch.device(device)
        self.dtype = dtype
        self.chunks = max(1, min(int(chunks), shape.P))
        act = (shape.P, shape.F, shape.C)
        mk = lambda sz: torch.empty(sz, dtype=dtype, device=self.device)  # noqa: E731
        self.d = {n: mk(act) for n in ("q", "k", "v", "conv_x", "gn_x", "out", "y", "z")}
        self.d["conv_w"] = mk((shape.C, shape.C, shape.k))
        for n in ("conv_b", "gn_gamma", "gn_beta"):
            self.d[n] = mk((shape.C,))
        self.s_in = torch.cuda.Stream(self.device)
        self.s_comp = torch.cuda.Stream(self.device)
        self.s_out = torch.cuda.Stream(self.device)
        self.bounds = chunk_bounds(shape.P, self.chunks)

    def _check(self, tensors: dict, names, shapes_from) -> None:
        for n in names:
            t = tensors[n]
            ref = shapes_from[n]
            if t.device.type != "cpu" or not t.is_pinned():
                raise ValueError(f"{n}: expected a pinned host tensor")
            if t.dtype != self.dtype or tuple(t.shape) != tuple(ref.shape) or not t.is_contiguous():
                raise ValueError(f"{n}: expected contiguous {self.dtype} of shape {tuple(ref.shape)}")

    def run(self, host_in: dict, host_out: dict) -> None:
        """One step: host_in (pinned inputs) -> host_out (pinned outputs out, y, z).

        Returns once everything is enqueued; the caller synchronises (for
        example torch.cuda.synchronize()) before reading host_out.
        """
        import torch
        self._check(host_in, _INPUTS, self.d)
        self._check(host_out, _OUTPUTS, self.d)
        s, d = self.s, self.d
        cur = torch.cuda.current_stream(self.device)
        for st in (self.s_in, self.s_comp, self.s_out):
            st.wait_stream(cur)            # the device buffers' previous users are done

        ev_gn_in = torch.cuda.Event()
        ev_chunk_in = [torch.cuda.Event() for _ in self.bounds]
        ev_gn_done = torch.cuda.Event()
        ev_chunk_done = [torch.cuda.Event() for _ in self.bounds]

        with torch.cuda.stream(self.s_in):
            for n in ("gn_x", "gn_gamma", "gn_beta", "conv_w", "conv_b"):
                d[n].copy_(host_in[n], non_blocking=True)
            ev_gn_in.record(self.s_in)
            for (p0, p1), ev in zip(self.bounds, ev_chunk_in):
                for n in ("q", "k", "v", "conv_x"):
                    d[n][p0:p1].copy_(host_in[n][p0:p1], non_blocking=True)
                ev.record(self.s_in)

        with torch.cuda.stream(self.s_comp):
            self.s_comp.wait_event(ev_gn_in)
            groupnorm_global(d["gn_x"], d["gn_gamma"], d["gn_beta"], d["z"], N=s.N,
                             groups=s.groups, eps=s.eps, stream=self.s_comp)
            ev_gn_done.record(self.s_comp)
            for (p0, p1), ev_in, ev_done in zip(self.bounds, ev_chunk_in, ev_chunk_done):
                self.s_comp.wait_event(ev_in)
                dual_attn(d["q"][p0:p1], d["k"][p0:p1], d["v"][p0:p1], d["out"][p0:p1], N=s.N,
                          heads=s.heads, n_pre=s.n_pre, n_post=s.n_post, n_global=s.n_global,
                          stream=self.s_comp)
                temporal_conv(d["conv_x"][p0:p1], d["conv_w"], d["conv_b"], d["y"][p0:p1],
                              N=s.N, stream=self.s_comp)
                ev_done.record(self.s_comp)

        with torch.cuda.stream(self.s_out):
            self.s_out.wait_event(ev_gn_done)
            host_out["z"].copy_(d["z"], non_blocking=True)
            for (p0, p1), ev in zip(self.bounds, ev_chunk_done):
                self.s_out.wait_event(ev)
                for n in ("out", "y"):
                    host_out[n][p0:p1].copy_(d[n][p0:p1], non_blocking=True)

        for st in (self.s_in, self.s_comp, self.s_out):
            cur.wait_stream(st)            # the caller's stream sees the whole step

    @staticmethod
    def h2d_bytes(host_in: dict) -> int:
        return int(sum(host_in[n].numel() * host_in[n].element_size() for n in _INPUTS))

    @staticmethod
    def d2h_bytes(host_out: dict) -> int:
        return int(sum(host_out[n].numel() * host_out[n].element_size() for n in _OUTPUTS))
