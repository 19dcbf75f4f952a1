"""Several host threads calling the library at once, each on its own CUDA
stream: the per-device state the library sets up on first use (memory pool,
kernel attributes, cached device properties) and the argument checks must be
safe to reach concurrently, and every thread must get the single-threaded
result (ctypes releases the GIL during each call, so the calls overlap)."""
import threading

import numpy as np
import pytest
import torch

import clip_temporal_modules_b200 as vi
import synth
from parity import to_device

pytestmark = pytest.mark.gpu


def _inputs(seed):
    w = synth.Workload("thr_bf16_F128_P8_C320", "bf16", F=128, N=8, P=8, C=320, heads=5, d=64,
                       seed=seed)
    return w, {n: to_device(synth.make(w, n), w.dtype) for n in
               ("q", "k", "v", "conv_x", "conv_w", "conv_b", "gn_x", "gn_gamma", "gn_beta",
                "attn_x", "w_qkv", "b_qkv", "w_out", "b_out")}


def _step(w, d, stream):
    with torch.cuda.stream(stream):
        a = vi.dual_attn(d["q"], d["k"], d["v"], N=w.N, heads=w.heads, stream=stream)
        y = vi.temporal_conv(d["conv_x"], d["conv_w"], d["conv_b"], N=w.N, stream=stream)
        z = vi.groupnorm_global(d["gn_x"], d["gn_gamma"], d["gn_beta"], N=w.N, groups=w.groups,
                                stream=stream)
        # the attention module: q/k/v GEMM, then the persistent fused kernel
        m = vi.temporal_attention(d["attn_x"], d["w_qkv"], d["b_qkv"], d["w_out"], d["b_out"],
                                  N=w.N, heads=w.heads, stream=stream)
    stream.synchronize()
    return [t.cpu().view(torch.int16).numpy() for t in (a, y, z, m)]


def test_concurrent_host_threads_match_serial_results(cuda_device):
    cases = [_inputs(seed) for seed in range(4)]
    serial = [_step(w, d, torch.cuda.Stream()) for w, d in cases]
    got = [None] * len(cases)
    errors = []

    def run(i):
        try:
            torch.cuda.set_device(0)
            w, d = cases[i]
            for _ in range(5):
                got[i] = _step(w, d, torch.cuda.Stream())
        except Exception as e:          # reported below, on the main thread
            errors.append(e)

    threads = [threading.Thread(target=run, args=(i,)) for i in range(len(cases))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not errors, errors
    vi.take_device_errors()
    for i in range(len(cases)):
        # attention and GroupNorm are deterministic; the conv's and the
        # module's summation orders depend only on their grids, which are the
        # same for every call here
        for g, s in zip(got[i], serial[i]):
            assert np.array_equal(g, s)
