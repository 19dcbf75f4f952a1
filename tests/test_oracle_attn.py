"""Pins of the oracle's dual-domain attention to facts outside the oracle.

Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
write-up), attention-module paragraph (dual-domain attention: own clip, local
neighbours C_pre/C_post, uniformly sampled global frames C_global).
"""
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "attn_key_frames.txt")


def golden_cases():
    cases = []
    with open(GOLDEN) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, frames = line.split(":")
            F, N, n_pre, n_post, n_global, i = map(int, head.split())
            cases.append(((F, N, n_pre, n_post, n_global), i, [int(t) for t in frames.split()]))
    return cases


def golden_table():
    table = {}
    for cfg, i, frames in golden_cases():
        table.setdefault(cfg, {})[i] = frames
    return table


@pytest.mark.parametrize("cfg,i,frames", golden_cases())
def test_key_frames_match_hand_derived(cfg, i, frames):
    F, N, n_pre, n_post, n_global = cfg
    got = oracle.key_frames(i, F, N, n_pre, n_post, n_global)
    assert sorted(got) == sorted(frames)


def _rand(shape, tid, dtype="f32", mean=0.0, std=1.0):
    return synth.normal(shape, tid, mean, std, seed=123, dtype=dtype)


def _weights_from_golden(F, N, cfg_lists):
    """Multiplicity matrix M[f][j] = copies of frame j in the key list of f's clip."""
    L = F // N
    M = np.zeros((F, F))
    for i, frames in cfg_lists.items():
        for f in range(i * L, (i + 1) * L):
            for j in frames:
                M[f, j] += 1
    return M


FULL_GOLDEN = [c for c in golden_table().items() if c[0][0] <= 32 and len(c[1]) == c[0][1]]


@pytest.mark.parametrize("cfg,lists", FULL_GOLDEN)
def test_random_inputs_match_multiplicity_mask_formulation(cfg, lists):
    """Softmax over the key multiset == dense attention weighted by multiplicities.

    An independent formulation: dense F x F scores, each key weighted by how
    often it appears in the (hand-derived) list of the query's clip.
    """
    F, N, n_pre, n_post, n_global = cfg
    heads, d, P = 2, 8, 3
    C = heads * d
    q, k, v = (_rand((P, F, C), t) for t in (11, 12, 13))
    out = oracle.dual_attn(q, k, v, F, N, heads, d, n_pre, n_post, n_global)
    M = _weights_from_golden(F, N, lists)
    for p in range(P):
        for h in range(heads):
            sl = slice(h * d, (h + 1) * d)
            s = q[p, :, sl].astype(np.float64) @ k[p, :, sl].astype(np.float64).T / np.sqrt(d)
            s = s - s.max(axis=1, keepdims=True)
            w = M * np.exp(s)
            ref = (w @ v[p, :, sl].astype(np.float64)) / w.sum(axis=1, keepdims=True)
            np.testing.assert_allclose(out[p, :, sl], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("cfg,lists", FULL_GOLDEN)
def test_zero_query_gives_multiset_mean(cfg, lists):
    """q = 0 makes every score 0: the output is the mean of V over the key multiset.

    With V one-hot in the frame index, the output row is the multiset's
    histogram divided by its size, which reads back the key list exactly
    (multiplicities and absent ends included).
    """
    F, N, n_pre, n_post, n_global = cfg
    d = F
    P = 1
    q = np.zeros((P, F, d), np.float32)
    k = _rand((P, F, d), 21)
    v = np.zeros((P, F, d), np.float32)
    v[0, np.arange(F), np.arange(F)] = 1.0
    out = oracle.dual_attn(q, k, v, F, N, 1, d, n_pre, n_post, n_global)
    L = F // N
    for i, frames in lists.items():
        hist = np.bincount(frames, minlength=F) / len(frames)
        for f in range(i * L, (i + 1) * L):
            np.testing.assert_allclose(out[0, f], hist, rtol=0, atol=1e-15)


def test_orthonormal_key_probe_selects_members_only():
    """q = beta e_t with one-hot keys selects frame t iff t is in the clip's key list."""
    F, N, n_pre, n_post, n_global = 12, 3, 2, 1, 3
    lists = golden_table()[(F, N, n_pre, n_post, n_global)]
    d, L = 16, F // N
    k = np.zeros((1, F, d), np.float32)
    k[0, np.arange(F), np.arange(F)] = 1.0
    v = k.copy()
    for t in range(F):
        q = np.zeros((1, F, d), np.float32)
        q[0, :, t] = 200.0 * np.sqrt(d)      # score 200 for frame t, 0 elsewhere
        out = oracle.dual_attn(q, k, v, F, N, 1, d, n_pre, n_post, n_global)
        for i, frames in lists.items():
            for f in range(i * L, (i + 1) * L):
                if t in frames:
                    expect = np.zeros(d)
                    expect[t] = 1.0
                else:
                    expect = np.bincount(frames, minlength=d) / len(frames)
                np.testing.assert_allclose(out[0, f], expect, rtol=0, atol=1e-12)


def test_constant_v_returns_v():
    F, N, heads, d, P = 32, 4, 2, 16, 2
    C = heads * d
    q, k = _rand((P, F, C), 31), _rand((P, F, C), 32)
    row = _rand((C,), 33)
    v = np.broadcast_to(row, (P, F, C)).astype(np.float32)
    out = oracle.dual_attn(q, k, v, F, N, heads, d, 8, 8, 16)
    np.testing.assert_allclose(out, np.broadcast_to(row.astype(np.float64), out.shape),
                               rtol=0, atol=1e-12)


def _sdpa(qh, kh, vh):
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    return torch.nn.functional.scaled_dot_product_attention(t(qh), t(kh), t(vh)).numpy()


def test_one_clip_no_global_is_full_temporal_attention():
    """N = 1 and n_global = 0: plain softmax attention over all F frames (library SDPA)."""
    F, heads, d, P = 24, 3, 16, 2
    C = heads * d
    q, k, v = (_rand((P, F, C), t) for t in (41, 42, 43))
    out = oracle.dual_attn(q, k, v, F, 1, heads, d, 0, 0, 0)
    for p in range(P):
        for h in range(heads):
            sl = slice(h * d, (h + 1) * d)
            ref = _sdpa(q[p, :, sl], k[p, :, sl], v[p, :, sl])
            np.testing.assert_allclose(out[p, :, sl], ref, rtol=0, atol=1e-12)


def test_no_context_is_independent_per_clip_attention():
    """n_pre = n_post = n_global = 0: each clip attends only to itself (library SDPA)."""
    F, N, heads, d, P = 24, 4, 2, 8, 2
    C, L = heads * d, 24 // 4
    q, k, v = (_rand((P, F, C), t) for t in (51, 52, 53))
    out = oracle.dual_attn(q, k, v, F, N, heads, d, 0, 0, 0)
    for p in range(P):
        for h in range(heads):
            sl = slice(h * d, (h + 1) * d)
            for i in range(N):
                fr = slice(i * L, (i + 1) * L)
                ref = _sdpa(q[p, fr, sl], k[p, fr, sl], v[p, fr, sl])
                np.testing.assert_allclose(out[p, fr, sl], ref, rtol=0, atol=1e-12)


def test_bf16_inputs_are_widened_exactly():
    """bf16 bit patterns give the same result as their exact fp32 values."""
    F, N, heads, d, P = 32, 4, 1, 64, 2
    C = heads * d
    qb, kb, vb = (_rand((P, F, C), t, dtype="bf16") for t in (61, 62, 63))
    out_b = oracle.dual_attn(qb, kb, vb, F, N, heads, d)
    out_f = oracle.dual_attn(*(synth.bf16_to_f32(a) for a in (qb, kb, vb)), F, N, heads, d)
    np.testing.assert_array_equal(out_b, out_f)


def test_position_subset_equals_full_slice():
    F, N, heads, d, P = 32, 4, 2, 8, 5
    C = heads * d
    q, k, v = (_rand((P, F, C), t) for t in (71, 72, 73))
    full = oracle.dual_attn(q, k, v, F, N, heads, d)
    sub = oracle.dual_attn(q, k, v, F, N, heads, d, positions=[4, 1])
    np.testing.assert_array_equal(sub, full[[4, 1]])


def test_attention_module_equals_library_composition():
    """Projections + dual attention + output projection; with one clip and no
    global frames this is Linear -> per-head SDPA -> Linear (library, fp64)."""
    F, heads, d, P = 16, 2, 8, 2
    C = heads * d
    x = _rand((P, F, C), 81)
    w_qkv, b_qkv = _rand((3 * C, C), 82, std=0.25), _rand((3 * C,), 83)
    w_out, b_out = _rand((C, C), 84, std=0.25), _rand((C,), 85)
    got = oracle.temporal_attention(x, w_qkv, b_qkv, w_out, b_out, F, 1, heads, d, 0, 0, 0,
                                    intermediate="f64")
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    xt = t(x)
    qkv = torch.nn.functional.linear(xt, t(w_qkv), t(b_qkv))          # [P][F][3C]
    q, k, v = qkv[..., :C], qkv[..., C:2 * C], qkv[..., 2 * C:]
    hs = lambda a: a.reshape(P, F, heads, d).permute(0, 2, 1, 3)
    a = torch.nn.functional.scaled_dot_product_attention(hs(q), hs(k), hs(v))
    a = a.permute(0, 2, 1, 3).reshape(P, F, C)
    ref = torch.nn.functional.linear(a, t(w_out), t(b_out)).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-11)
    sub = oracle.temporal_attention(x, w_qkv, b_qkv, w_out, b_out, F, 1, heads, d, 0, 0, 0,
                                    positions=[1], intermediate="f64")
    np.testing.assert_array_equal(sub, got[[1]])
