"""Pins of the oracle's clip-padded temporal convolution.

Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
write-up), conv-module paragraph: each clip is padded with the last n frames
of the previous clip and the first n frames of the next, n the receptive
field of the conv.  With zeros at the video ends this must equal the
unpartitioned zero-padded conv1d, which the library computes independently.
"""
import numpy as np
import pytest
import torch

import oracle
import synth


def _rand(shape, tid, std=1.0, dtype="f32"):
    return synth.normal(shape, tid, 0.0, std, seed=7, dtype=dtype)


def _torch_conv(x, w, b, k):
    """Unpartitioned Conv1d over frames, zero padding k//2 (library)."""
    xt = torch.from_numpy(np.asarray(x, np.float64)).permute(0, 2, 1)   # [P][C][F]
    y = torch.nn.functional.conv1d(xt, torch.from_numpy(np.asarray(w, np.float64)),
                                   torch.from_numpy(np.asarray(b, np.float64)), padding=k // 2)
    return y.permute(0, 2, 1).numpy()


@pytest.mark.parametrize("F,N,k", [(16, 1, 3), (16, 2, 3), (16, 4, 3), (24, 8, 3), (16, 4, 5),
                                   (12, 3, 1), (20, 4, 5)])
def test_clip_padded_conv_equals_unpartitioned_conv1d(F, N, k):
    P, C = 3, 12
    x = _rand((P, F, C), 1)
    w = _rand((C, C, k), 2, std=0.3)
    b = _rand((C,), 3)
    y = oracle.temporal_conv(x, w, b, F, N, k)
    np.testing.assert_allclose(y, _torch_conv(x, w, b, k), rtol=0, atol=1e-12)


def test_centre_tap_identity_gives_x_plus_b():
    F, N, P, C = 16, 4, 2, 8
    x, b = _rand((P, F, C), 4), _rand((C,), 5)
    w = np.zeros((C, C, 3), np.float32)
    w[np.arange(C), np.arange(C), 1] = 1.0
    y = oracle.temporal_conv(x, w, b, F, N, 3)
    np.testing.assert_allclose(y, x.astype(np.float64) + b, rtol=0, atol=0)


def test_first_tap_shift_reads_previous_frame_and_zero_at_start():
    """Tap 0 = identity: y[f] = x[f-1] + b, and y[0] = b (zero pad before the video)."""
    F, N, P, C = 16, 4, 2, 8
    x, b = _rand((P, F, C), 6), _rand((C,), 7)
    w = np.zeros((C, C, 3), np.float32)
    w[np.arange(C), np.arange(C), 0] = 1.0
    y = oracle.temporal_conv(x, w, b, F, N, 3)
    np.testing.assert_array_equal(y[:, 0, :], np.broadcast_to(b.astype(np.float64), (P, C)))
    np.testing.assert_array_equal(y[:, 1:, :], x[:, :-1, :].astype(np.float64) + b)


def test_last_tap_shift_reads_next_frame_and_zero_at_end():
    F, N, P, C = 16, 4, 2, 8
    x, b = _rand((P, F, C), 8), _rand((C,), 9)
    w = np.zeros((C, C, 3), np.float32)
    w[np.arange(C), np.arange(C), 2] = 1.0
    y = oracle.temporal_conv(x, w, b, F, N, 3)
    np.testing.assert_array_equal(y[:, -1, :], np.broadcast_to(b.astype(np.float64), (P, C)))
    np.testing.assert_array_equal(y[:, :-1, :], x[:, 1:, :].astype(np.float64) + b)


def test_channel_mixing_orientation():
    """W[co, ci, 1] routes input channel ci to output channel co (not the transpose)."""
    F, N, P, C = 8, 2, 1, 4
    x = _rand((P, F, C), 10)
    w = np.zeros((C, C, 3), np.float32)
    w[0, 3, 1] = 1.0                       # out channel 0 <- in channel 3
    b = np.zeros(C, np.float32)
    y = oracle.temporal_conv(x, w, b, F, N, 3)
    np.testing.assert_array_equal(y[0, :, 0], x[0, :, 3].astype(np.float64))
    np.testing.assert_array_equal(y[0, :, 1:], 0.0)


def test_linearity_in_x():
    F, N, P, C = 16, 4, 2, 8
    x1, x2 = _rand((P, F, C), 11), _rand((P, F, C), 12)
    w, b = _rand((C, C, 3), 13, std=0.3), _rand((C,), 14)
    a = 0.75
    y1 = oracle.temporal_conv(x1, w, b, F, N) - b
    y2 = oracle.temporal_conv(x2, w, b, F, N) - b
    y12 = oracle.temporal_conv((a * x1 + x2).astype(np.float32), w, b, F, N) - b
    np.testing.assert_allclose(y12, a * y1 + y2, rtol=0, atol=1e-5)


def test_bf16_inputs_are_widened_exactly():
    F, N, P, C = 16, 4, 2, 16
    xb, wb, bb = _rand((P, F, C), 15, dtype="bf16"), _rand((C, C, 3), 16, 0.3, "bf16"), \
        _rand((C,), 17, dtype="bf16")
    yb = oracle.temporal_conv(xb, wb, bb, F, N)
    yf = oracle.temporal_conv(*(synth.bf16_to_f32(a) for a in (xb, wb, bb)), F, N)
    np.testing.assert_array_equal(yb, yf)


def test_position_subset_equals_full_slice():
    F, N, P, C = 16, 4, 5, 8
    x, w, b = _rand((P, F, C), 18), _rand((C, C, 3), 19, 0.3), _rand((C,), 20)
    full = oracle.temporal_conv(x, w, b, F, N)
    np.testing.assert_array_equal(oracle.temporal_conv(x, w, b, F, N, positions=[3, 0]),
                                  full[[3, 0]])


def test_groupnorm_then_conv_equals_library_composition():
    """GroupNorm (whole-tensor statistics) then conv1d, both from the library."""
    F, N, P, C, G, k = 16, 4, 3, 16, 4, 3
    x = synth.normal((P, F, C), 21, 0.5, 1.4, seed=7, dtype="f32")
    gamma = synth.normal((C,), 22, 1.0, 0.3, seed=7, dtype="f32")
    beta = synth.normal((C,), 23, 0.0, 0.3, seed=7, dtype="f32")
    w, b = _rand((C, C, k), 24, std=0.3), _rand((C,), 25)
    got = oracle.groupnorm_conv(x, gamma, beta, w, b, F, N, G, 1e-5, k)
    xt = torch.from_numpy(x.astype(np.float64)).reshape(P * F, C).T.reshape(1, C, P * F)
    z = torch.nn.functional.group_norm(xt, G, torch.from_numpy(gamma.astype(np.float64)),
                                       torch.from_numpy(beta.astype(np.float64)), 1e-5)
    z = z.reshape(C, P * F).T.reshape(P, F, C).numpy()
    np.testing.assert_allclose(got, _torch_conv(z, w, b, k), rtol=0, atol=1e-12)
    sub = oracle.groupnorm_conv(x, gamma, beta, w, b, F, N, G, 1e-5, k, positions=[2, 0])
    np.testing.assert_array_equal(sub, got[[2, 0]])


def test_round_bf16_is_nearest_even():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -8 + 2 ** -20])
    np.testing.assert_array_equal(oracle.round_bf16(v), [1.0, 1.0, 1.0 + 2 ** -6, -2.5,
                                                         1.0 + 2 ** -7])
