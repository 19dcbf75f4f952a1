"""The host-buffer executor: position chunking (CPU) and equality with the
whole-tensor calls (GPU).  Attention is computed per (position, clip block,
head) and GroupNorm runs on the whole tensor, so those two must match the plain
calls bit for bit; the conv's CTAs sum their K-blocks starting at an offset
that depends on which CTA takes a tile, so a different chunking may change the
fp32 summation order: it must match within the bf16 parity tolerance."""
import numpy as np
import pytest
import torch

import synth
from clip_temporal_modules_b200.host_pipeline import chunk_bounds


@pytest.mark.parametrize("P,chunks", [(10, 3), (2560, 8), (5, 8), (1, 1), (7, 7)])
def test_chunk_bounds_cover_positions_in_order(P, chunks):
    b = chunk_bounds(P, chunks)
    assert b[0][0] == 0 and b[-1][1] == P
    assert all(p1 > p0 for p0, p1 in b)
    assert all(b[i][1] == b[i + 1][0] for i in range(len(b) - 1))
    sizes = [p1 - p0 for p0, p1 in b]
    assert max(sizes) - min(sizes) <= 1
    assert len(b) == min(chunks, P)


@pytest.mark.gpu
@pytest.mark.parametrize("chunks", [1, 3])
def test_pipeline_equals_whole_tensor_calls(cuda_device, chunks):
    import clip_temporal_modules_b200 as vi
    w = synth.Workload("pipe_bf16_F128_P10_C320", "bf16", F=128, N=8, P=10, C=320, heads=5, d=64)
    host = {}
    for n in ("q", "k", "v", "conv_x", "conv_w", "conv_b", "gn_x", "gn_gamma", "gn_beta"):
        host[n] = torch.from_numpy(synth.make(w, n)).view(torch.bfloat16).pin_memory()
    out = {n: torch.empty_like(host["q"]).pin_memory() for n in ("out", "y", "z")}
    shape = vi.StepShape(F=w.F, N=w.N, P=w.P, C=w.C, heads=w.heads)
    pipe = vi.HostPipeline(shape, "cuda", torch.bfloat16, chunks=chunks)
    pipe.run(host, out)
    torch.cuda.synchronize()
    vi.take_device_errors()
    d = {n: t.cuda() for n, t in host.items()}
    ref_out = vi.dual_attn(d["q"], d["k"], d["v"], N=w.N, heads=w.heads)
    ref_y = vi.temporal_conv(d["conv_x"], d["conv_w"], d["conv_b"], N=w.N)
    ref_z = vi.groupnorm_global(d["gn_x"], d["gn_gamma"], d["gn_beta"], N=w.N, groups=w.groups)
    torch.cuda.synchronize()
    for got, ref in ((out["out"], ref_out), (out["z"], ref_z)):
        assert np.array_equal(got.view(torch.int16).numpy(), ref.cpu().view(torch.int16).numpy())
    diff = (out["y"].float() - ref_y.cpu().float()).abs().max().item()
    assert diff <= 2e-2


@pytest.mark.gpu
def test_pipeline_rejects_pageable_host_tensors(cuda_device):
    import clip_temporal_modules_b200 as vi
    shape = vi.StepShape(F=16, N=1, P=2, C=64, heads=1)
    pipe = vi.HostPipeline(shape, "cuda", torch.bfloat16)
    t = torch.zeros(2, 16, 64, dtype=torch.bfloat16)
    host = {n: t for n in ("q", "k", "v", "conv_x", "gn_x")}
    host.update(conv_w=torch.zeros(64, 64, 3, dtype=torch.bfloat16),
                conv_b=torch.zeros(64, dtype=torch.bfloat16),
                gn_gamma=torch.zeros(64, dtype=torch.bfloat16),
                gn_beta=torch.zeros(64, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        pipe.run(host, {n: t for n in ("out", "y", "z")})
