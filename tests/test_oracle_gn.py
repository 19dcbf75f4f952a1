"""Pins of the oracle's global-statistics GroupNorm.

Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
write-up), GroupNorm-module paragraph: clip group means are aggregated into a
global mean, each clip then measures its spread about that global mean and
these are aggregated into a global std.  The result must equal GroupNorm of
the whole, unpartitioned latent, which the library computes independently.
"""
import numpy as np
import pytest
import torch

import oracle
import synth


def _rand(shape, tid, mean=0.0, std=1.0, dtype="f32"):
    return synth.normal(shape, tid, mean, std, seed=5, dtype=dtype)


def _torch_gn(x, gamma, beta, groups, eps):
    """GroupNorm of the whole latent, batch 1, channels first (library)."""
    P, F, C = x.shape
    xt = torch.from_numpy(np.asarray(x, np.float64)).reshape(P * F, C).T.reshape(1, C, P * F)
    y = torch.nn.functional.group_norm(xt, groups, torch.from_numpy(np.asarray(gamma, np.float64)),
                                       torch.from_numpy(np.asarray(beta, np.float64)), eps)
    return y.reshape(C, P * F).T.reshape(P, F, C).numpy()


@pytest.mark.parametrize("F,N", [(16, 1), (16, 2), (16, 4), (16, 16), (24, 3)])
@pytest.mark.parametrize("C,groups", [(8, 8), (20, 2), (12, 4)])
def test_global_stats_equal_whole_tensor_groupnorm(F, N, C, groups):
    P = 3
    x = _rand((P, F, C), 1, 0.5, np.sqrt(2.0))
    gamma, beta = _rand((C,), 2, 1.0, 0.3), _rand((C,), 3, 0.0, 0.3)
    y, mean, var = oracle.groupnorm_global(x, gamma, beta, F, N, groups, 1e-5)
    np.testing.assert_allclose(y, _torch_gn(x, gamma, beta, groups, 1e-5), rtol=0, atol=1e-12)
    xg = x.astype(np.float64).reshape(P * F, groups, C // groups)
    np.testing.assert_allclose(mean, xg.mean(axis=(0, 2)), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(var, xg.var(axis=(0, 2)), rtol=1e-12, atol=1e-14)


def test_constant_group_gives_beta():
    F, N, P, C, G = 8, 2, 2, 8, 4
    x = _rand((P, F, C), 4)
    x[:, :, 2:4] = 3.25                  # group 1 constant
    gamma, beta = _rand((C,), 5, 1.0, 0.3), _rand((C,), 6)
    y, _, var = oracle.groupnorm_global(x, gamma, beta, F, N, G, 1e-5)
    assert var[1] == 0.0
    np.testing.assert_array_equal(y[:, :, 2:4], np.broadcast_to(beta[2:4].astype(np.float64),
                                                                 (P, F, 2)))


def test_unit_affine_moments():
    """gamma = 1, beta = 0: each group has mean 0 and variance var/(var+eps)."""
    F, N, P, C, G, eps = 16, 4, 3, 16, 4, 1e-2
    x = _rand((P, F, C), 7, 0.5, 2.0)
    y, _, var = oracle.groupnorm_global(x, np.ones(C, np.float32), np.zeros(C, np.float32),
                                        F, N, G, eps)
    yg = y.reshape(P * F, G, C // G)
    np.testing.assert_allclose(yg.mean(axis=(0, 2)), 0.0, atol=1e-12)
    np.testing.assert_allclose(yg.var(axis=(0, 2)), var / (var + eps), rtol=1e-12)


def test_invariant_to_affine_change_of_input():
    F, N, P, C, G = 16, 4, 2, 8, 2
    x = _rand((P, F, C), 8)
    gamma, beta = _rand((C,), 9, 1.0, 0.3), _rand((C,), 10)
    y1, _, _ = oracle.groupnorm_global(x, gamma, beta, F, N, G, 0.0)
    y2, _, _ = oracle.groupnorm_global((3.0 * x + 7.0).astype(np.float32), gamma, beta, F, N, G,
                                       0.0)
    np.testing.assert_allclose(y2, y1, rtol=0, atol=1e-5)


def test_bf16_inputs_are_widened_exactly():
    F, N, P, C, G = 16, 4, 2, 16, 4
    xb = _rand((P, F, C), 11, 0.5, 1.4, "bf16")
    gb, bb = _rand((C,), 12, 1.0, 0.3, "bf16"), _rand((C,), 13, 0.0, 0.3, "bf16")
    yb, mb, vb = oracle.groupnorm_global(xb, gb, bb, F, N, G)
    yf, mf, vf = oracle.groupnorm_global(*(synth.bf16_to_f32(a) for a in (xb, gb, bb)), F, N, G)
    np.testing.assert_array_equal(yb, yf)
    np.testing.assert_array_equal(mb, mf)


def test_position_subset_equals_full_slice():
    F, N, P, C, G = 8, 2, 4, 8, 2
    x = _rand((P, F, C), 14)
    gamma, beta = _rand((C,), 15, 1.0, 0.3), _rand((C,), 16)
    full, _, _ = oracle.groupnorm_global(x, gamma, beta, F, N, G)
    sub, _, _ = oracle.groupnorm_global(x, gamma, beta, F, N, G, positions=[2, 0])
    np.testing.assert_array_equal(sub, full[[2, 0]])


def test_pooled_statistics_of_equal_shards_equal_the_whole():
    """The merge the shard calls use (mean of means; mean of var + squared
    deviation of the shard mean) gives the statistics of the whole tensor when
    the shards are equal in size -- checked against the oracle's GroupNorm
    statistics of the whole tensor and of each shard."""
    F, N, P, C, G = 64, 8, 3, 16, 4
    x = synth.normal((P, F, C), 31, 0.5, 1.4, seed=9, dtype="f32")
    g = np.ones(C, np.float32)
    b = np.zeros(C, np.float32)
    _, mean, var = oracle.groupnorm_global(x, g, b, F, N, G, want_y=False)
    for W in (2, 4, 8):
        Fl = F // W
        parts = [oracle.groupnorm_global(np.ascontiguousarray(x[:, r * Fl:(r + 1) * Fl]), g, b,
                                         Fl, N // W, G, want_y=False)[1:] for r in range(W)]
        m = np.stack([p[0] for p in parts])
        v = np.stack([p[1] for p in parts])
        pooled_mean = m.mean(axis=0)
        pooled_var = (v + (m - pooled_mean) ** 2).mean(axis=0)
        np.testing.assert_allclose(pooled_mean, mean, rtol=0, atol=1e-12)
        np.testing.assert_allclose(pooled_var, var, rtol=1e-12, atol=0)
