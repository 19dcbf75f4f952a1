"""Randomised pins of the oracle over many small shapes (hypothesis): the
clip-padded conv against the library's unpartitioned conv1d, the global-stat
GroupNorm against the library's group_norm on the whole tensor, and the
dual-domain attention against a dense softmax weighted by key multiplicities.
The fixed-shape pins in the other test files cover the special cases; these
sweep clip counts, ragged channel counts and context sizes."""
import numpy as np
import torch
from hypothesis import assume, given, settings
from hypothesis import strategies as st

import oracle
import synth

SETTINGS = settings(max_examples=25, deadline=None, derandomize=True)


@st.composite
def clip_shapes(draw, max_l=6):
    N = draw(st.integers(1, 5))
    L = draw(st.integers(1, max_l))
    P = draw(st.integers(1, 3))
    return N * L, N, L, P


@SETTINGS
@given(shape=clip_shapes(), C=st.integers(1, 9), k=st.sampled_from([1, 3, 5]),
       seed=st.integers(0, 2 ** 20))
def test_conv_equals_library_conv1d(shape, C, k, seed):
    F, N, L, P = shape
    assume(k // 2 <= L)                      # the halo comes from the neighbouring clip only
    x = synth.normal((P, F, C), 1, 0.0, 1.0, seed=seed, dtype="f32")
    w = synth.normal((C, C, k), 2, 0.0, 0.4, seed=seed, dtype="f32")
    b = synth.normal((C,), 3, 0.0, 1.0, seed=seed, dtype="f32")
    y = oracle.temporal_conv(x, w, b, F, N, k)
    xt = torch.from_numpy(x.astype(np.float64)).permute(0, 2, 1)
    ref = torch.nn.functional.conv1d(xt, torch.from_numpy(w.astype(np.float64)),
                                     torch.from_numpy(b.astype(np.float64)), padding=k // 2)
    np.testing.assert_allclose(y, ref.permute(0, 2, 1).numpy(), rtol=0, atol=1e-11)


@SETTINGS
@given(shape=clip_shapes(), G=st.integers(1, 4), cg=st.integers(1, 4),
       seed=st.integers(0, 2 ** 20))
def test_groupnorm_equals_library_group_norm(shape, G, cg, seed):
    F, N, L, P = shape
    assume(P * F * cg > 1)                   # the library needs more than one value per group
    C = G * cg
    x = synth.normal((P, F, C), 4, 0.3, 1.7, seed=seed, dtype="f32")
    g = synth.normal((C,), 5, 1.0, 0.3, seed=seed, dtype="f32")
    bt = synth.normal((C,), 6, 0.0, 0.3, seed=seed, dtype="f32")
    y, _, _ = oracle.groupnorm_global(x, g, bt, F, N, G, 1e-5)
    xt = torch.from_numpy(x.astype(np.float64)).reshape(P * F, C).T.reshape(1, C, P * F)
    ref = torch.nn.functional.group_norm(xt, G, torch.from_numpy(g.astype(np.float64)),
                                         torch.from_numpy(bt.astype(np.float64)), 1e-5)
    ref = ref.reshape(C, P * F).T.reshape(P, F, C).numpy()
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-10)


@SETTINGS
@given(shape=clip_shapes(max_l=5), heads=st.integers(1, 2), d=st.integers(1, 6),
       ctx=st.tuples(st.integers(0, 5), st.integers(0, 5)), ng=st.integers(0, 6),
       seed=st.integers(0, 2 ** 20))
def test_attention_equals_multiplicity_weighted_dense_softmax(shape, heads, d, ctx, ng, seed):
    F, N, L, P = shape
    n_pre, n_post = (min(ctx[0], L), min(ctx[1], L)) if N > 1 else ctx
    ng = min(ng, F)
    C = heads * d
    q, k, v = (synth.normal((P, F, C), t, 0.0, 1.0, seed=seed, dtype="f32") for t in (7, 8, 9))
    out = oracle.dual_attn(q, k, v, F, N, heads, d, n_pre, n_post, ng)
    M = np.zeros((F, F))
    for i in range(N):
        for j in oracle.key_frames(i, F, N, n_pre, n_post, ng):
            M[i * L:(i + 1) * L, j] += 1
    for p in range(P):
        for h in range(heads):
            sl = slice(h * d, (h + 1) * d)
            s = q[p, :, sl].astype(np.float64) @ k[p, :, sl].astype(np.float64).T / np.sqrt(d)
            s = np.where(M > 0, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            wgt = M * np.exp(s)
            ref = (wgt @ v[p, :, sl].astype(np.float64)) / wgt.sum(axis=1, keepdims=True)
            np.testing.assert_allclose(out[p, :, sl], ref, rtol=0, atol=1e-11)
