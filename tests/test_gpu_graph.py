"""The three module calls captured in a CUDA graph and replayed.

Every call only enqueues stream-ordered work (kernels, a memset, allocations
from the library's stream-ordered pool), so a step can be captured once and
replayed without host overhead.  The first calls run eagerly (they set kernel
attributes and create the pool); the replays must equal the eager results."""
import numpy as np
import pytest
import torch

import clip_temporal_modules_b200 as vi
import synth
from parity import to_device

pytestmark = pytest.mark.gpu


def test_step_replays_from_a_cuda_graph(cuda_device):
    w = synth.Workload("graph_bf16_F256_P16_C320", "bf16", F=256, N=16, P=16, C=320, heads=5,
                       d=64)
    d = {n: to_device(synth.make(w, n), w.dtype) for n in
         ("q", "k", "v", "conv_x", "conv_w", "conv_b", "gn_x", "gn_gamma", "gn_beta")}
    out = {n: torch.empty_like(d["q"]) for n in ("a", "y", "z")}

    def step(stream):
        vi.dual_attn(d["q"], d["k"], d["v"], out["a"], N=w.N, heads=w.heads, stream=stream)
        vi.temporal_conv(d["conv_x"], d["conv_w"], d["conv_b"], out["y"], N=w.N, stream=stream)
        vi.groupnorm_global(d["gn_x"], d["gn_gamma"], d["gn_beta"], out["z"], N=w.N,
                            groups=w.groups, stream=stream)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step(s)                                  # eager: first-use setup happens here
    s.synchronize()
    eager = {n: t.clone() for n, t in out.items()}

    g = torch.cuda.CUDAGraph()
    n0 = vi.launch_count()
    with torch.cuda.graph(g, stream=s):
        step(s)
    captured = vi.launch_count() - n0
    assert captured == 5                         # attention, pack + conv, stats + apply
    for t in out.values():
        t.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    vi.take_device_errors()
    for n in out:
        assert np.array_equal(out[n].cpu().view(torch.int16).numpy(),
                              eager[n].cpu().view(torch.int16).numpy()), n
    del g


def test_attention_module_replays_from_a_cuda_graph(cuda_device):
    """The attention module (q/k/v GEMM, then the attention with the output
    projection fused in, a persistent kernel) captured with a caller-owned
    workspace and replayed: the replays equal the eager result bit for bit."""
    w = synth.Workload("graph_bf16_F256_P16_C320", "bf16", F=256, N=16, P=16, C=320, heads=5,
                       d=64)
    x, wq, bq, wo, bo = (to_device(synth.make(w, n), w.dtype)
                         for n in ("attn_x", "w_qkv", "b_qkv", "w_out", "b_out"))
    out = torch.empty_like(x)
    n = int(vi.lib().vi_temporal_attention_workspace_bytes(w.F, w.P, w.C))
    ws = torch.empty(n // 2, dtype=torch.bfloat16, device=x.device)

    def step(stream):
        vi.temporal_attention(x, wq, bq, wo, bo, out, ws, N=w.N, heads=w.heads, stream=stream)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step(s)
    s.synchronize()
    eager = out.clone()

    g = torch.cuda.CUDAGraph()
    n0 = vi.launch_count()
    with torch.cuda.graph(g, stream=s):
        step(s)
    assert vi.launch_count() - n0 == 3           # weight pack, q/k/v GEMM, fused attention
    out.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    vi.take_device_errors()
    assert np.array_equal(out.cpu().view(torch.int16).numpy(),
                          eager.cpu().view(torch.int16).numpy())
    del g
