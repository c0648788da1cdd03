"""Pins for the oracle's short causal convolution (CPU only).

ATMA ("Long-Context Language Modeling via Polar Attention and Gated-Delta Compression Memory",
Sec. 3) applies depthwise causal convolutions to q, k and v; the plain reading is
y_t[c] = sum_{j<W} w[c, j] x_{t-j}[c] with the history before t = 0 from a carried state.  Pinned by
a hand-worked example, the impulse response, causality, linearity and the carried state (a split
sequence gives the whole sequence's result).
"""
import numpy as np

import oracle


def test_hand_worked():
    # channel 0: x = 0,2,4,...,10, w = (1, 1/2, 1/4): y_2 = 4 + 2/2 + 0/4 = 5, y_3 = 6 + 4/2 + 2/4 = 8.5
    # channel 1: x = 1,3,5,...,11, w = (2, 0, 1):     y_0 = 2, y_2 = 10 + 0 + 1 = 11, y_5 = 22 + 7 = 29
    x = np.arange(12, dtype=np.float32).reshape(1, 6, 2)
    w = np.array([[1, 0.5, 0.25], [2, 0, 1]])
    y, st = oracle.causal_conv(x, w)
    assert np.array_equal(y[0, :, 0], [0, 2, 5, 8.5, 12, 15.5])
    assert np.array_equal(y[0, :, 1], [2, 6, 11, 17, 23, 29])
    assert np.array_equal(st[0], [[8, 9], [10, 11]])


def test_impulse_response_is_the_weights():
    rng = np.random.default_rng(61)
    C, W, T = 5, 4, 9
    w = rng.standard_normal((C, W))
    x = np.zeros((1, T, C), np.float32)
    x[0, 2] = 1.0
    y, _ = oracle.causal_conv(x, w)
    for t in range(T):
        expect = w[:, t - 2] if 0 <= t - 2 < W else np.zeros(C)
        assert np.array_equal(y[0, t], expect)


def test_causal_and_linear():
    rng = np.random.default_rng(62)
    B, T, C, W = 2, 20, 6, 3
    w = rng.standard_normal((C, W))
    x1 = rng.standard_normal((B, T, C)).astype(np.float32)
    x2 = rng.standard_normal((B, T, C)).astype(np.float32)
    y1, _ = oracle.causal_conv(x1, w)
    x3 = x1.copy()
    x3[:, 12:] += 5.0  # changing the future leaves the past unchanged
    y3, _ = oracle.causal_conv(x3, w)
    assert np.array_equal(y1[:, :12], y3[:, :12]) and not np.array_equal(y1[:, 12:], y3[:, 12:])
    y2, _ = oracle.causal_conv(x2, w)
    y12, _ = oracle.causal_conv(x1.astype(np.float64) + 2 * x2, w)
    np.testing.assert_allclose(y12, y1 + 2 * y2, rtol=0, atol=1e-12)


def test_carried_state_splits_the_sequence():
    rng = np.random.default_rng(63)
    B, T, C, W = 2, 17, 4, 4
    w = rng.standard_normal((C, W))
    x = rng.standard_normal((B, T, C)).astype(np.float32)
    s0 = rng.standard_normal((B, W - 1, C))
    y, s = oracle.causal_conv(x, w, s0)
    ya, sa = oracle.causal_conv(x[:, :2], w, s0)  # fewer tokens than the window
    yb, sb = oracle.causal_conv(x[:, 2:], w, sa)
    assert np.array_equal(np.concatenate([ya, yb], axis=1), y) and np.array_equal(sb, s)
    y1, s1 = oracle.causal_conv(x[:, :0], w, s0)
    assert y1.shape == (B, 0, C) and np.array_equal(s1, s0)
