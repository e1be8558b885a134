"""Pins for the oracle's causal short convolution and its history rewind
(oracle_short_conv), each against something other than the oracle itself: NumPy's
convolution and SciPy's logistic function, the streaming property a rewound history must
have, closed forms of the history, and special filters whose output is known."""
import numpy as np
import pytest
from scipy.special import expit

from oracle import gdn_oracle as orc


def _rand(B, T, C, K, seed):
    r = np.random.default_rng(seed)
    return (r.standard_normal((B, T, C)), r.standard_normal((C, K)) * 0.5,
            r.standard_normal((B, K - 1, C)))


def _silu(z):
    return z * expit(z)


@pytest.mark.parametrize("K", [2, 3, 4])
def test_matches_numpy_convolution(K):
    B, T, C = 2, 9, 5
    x, w, h = _rand(B, T, C, K, seed=K)
    y, _, _ = orc.short_conv_channels(x, w, h)
    for b in range(B):
        for c in range(C):
            stream = np.concatenate([h[b, :, c], x[b, :, c]])
            # np.convolve flips its second argument: flipping w back gives sum_i w[i] xc[t + i]
            z = np.convolve(stream, w[c, ::-1], mode="valid")
            np.testing.assert_allclose(y[b, :, c], _silu(z), rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("T,L1", [(8, 0), (8, 1), (8, 2), (8, 5), (8, 8), (2, 1), (2, 0), (1, 1)])
def test_rewound_history_continues_the_accepted_stream(T, L1):
    # Block 1 accepted up to L1, then block 2 from the rewound history, must give exactly the
    # outputs of one pass over [x1[:L1], x2] from the first history.
    K, C = 4, 6
    x1, w, h0 = _rand(1, T, C, K, seed=10 + T + L1)
    x2 = np.random.default_rng(99).standard_normal((1, 5, C))
    _, h1, bad = orc.short_conv_channels(x1, w, h0, np.array([L1], dtype=np.int32))
    assert bad == 0
    y2, h2, _ = orc.short_conv_channels(x2, w, h1)
    joined = np.concatenate([x1[:, :L1], x2], axis=1)
    yj, hj, _ = orc.short_conv_channels(joined, w, h0)
    np.testing.assert_allclose(y2, yj[:, L1:], rtol=1e-13, atol=1e-14)
    np.testing.assert_array_equal(h2, hj)


def test_history_closed_forms():
    K, T, C = 4, 8, 3
    x, w, h = _rand(3, T, C, K, seed=5)
    _, hn, bad = orc.short_conv_channels(x, w, h, np.array([0, 8, 2], dtype=np.int32))
    assert bad == 0
    np.testing.assert_array_equal(hn[0], h[0])                          # rollback: unchanged
    np.testing.assert_array_equal(hn[1], x[1, T - (K - 1):])            # all accepted: last K-1 inputs
    np.testing.assert_array_equal(hn[2], np.concatenate([h[2, 2:], x[2, :2]]))   # oldest first
    _, hall, _ = orc.short_conv_channels(x, w, h)                       # no counts: all T accepted
    np.testing.assert_array_equal(hall, x[:, T - (K - 1):])


def test_out_of_range_count_keeps_history():
    x, w, h = _rand(3, 8, 4, 4, seed=6)
    _, hn, bad = orc.short_conv_channels(x, w, h, np.array([-1, 9, 3], dtype=np.int32))
    assert bad == 2
    np.testing.assert_array_equal(hn[:2], h[:2])


def test_tap_order():
    # w = e_{K-1}: only the current input; w = e_0: the input K-1 steps back (from the history
    # for the first K-1 tokens).
    K, T, C = 4, 6, 3
    x, _, h = _rand(2, T, C, K, seed=7)
    cur = np.zeros((C, K)); cur[:, K - 1] = 1.0
    old = np.zeros((C, K)); old[:, 0] = 1.0
    y, _, _ = orc.short_conv_channels(x, cur, h)
    np.testing.assert_allclose(y, _silu(x), rtol=1e-14, atol=1e-15)
    y, _, _ = orc.short_conv_channels(x, old, h)
    stream = np.concatenate([h, x], axis=1)
    np.testing.assert_allclose(y, _silu(stream[:, :T]), rtol=1e-14, atol=1e-15)


def test_silu_values():
    # silu(0) = 0; silu(z) - silu(-z) = z; silu(z) -> z for large z
    x = np.array([[[0.0, 3.0, -3.0, 40.0]]])
    w = np.ones((4, 1))
    y, _, _ = orc.short_conv_channels(x, w, np.zeros((1, 0, 4)))
    assert y[0, 0, 0] == 0.0
    assert abs((y[0, 0, 1] - y[0, 0, 2]) - 3.0) < 1e-14
    assert abs(y[0, 0, 3] - 40.0) < 1e-12


def test_channel_order_q_k_v():
    # each of q', k', v' depends only on its own channels, in the order q | k | v
    r = np.random.default_rng(8)
    B, T, Hk, Hv, dk, dv, K = 2, 4, 2, 4, 8, 8, 4
    q, k = r.standard_normal((B, T, Hk, dk)), r.standard_normal((B, T, Hk, dk))
    v = r.standard_normal((B, T, Hv, dv))
    C = 2 * Hk * dk + Hv * dv
    w, h = r.standard_normal((C, K)), r.standard_normal((B, K - 1, C))
    q1, k1, v1, _, _ = orc.short_conv(q, k, v, w, h)
    q2, k2, v2, _, _ = orc.short_conv(q, k * 2.0, v + 1.0, w, h)
    np.testing.assert_array_equal(q1, q2)
    assert not np.allclose(k1, k2) and not np.allclose(v1, v2)
    # q head g, column j is channel g * d_k + j
    y, _, _ = orc.short_conv_channels(q.reshape(B, T, -1), w[:Hk * dk], h[:, :, :Hk * dk])
    np.testing.assert_array_equal(q1, y.reshape(q.shape))
