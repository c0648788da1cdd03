"""CPU pins of the oracle's packed-sequence helper (oracle.forward_varlen): the recurrence runs
on each sequence alone, from its own initial state, so packing changes nothing but the layout."""
import numpy as np

import oracle
from gdn_inputs import as_f32_numpy, forward_inputs, varlen_inputs


def np32(t):
    return None if t is None else as_f32_numpy(t)


def test_equal_lengths_match_the_batched_forward():
    B, T, H, d = 3, 20, 2, 8
    inp = forward_inputs(B, T, H, d, d, "f32", seed=5, s0_std=0.3)
    ref_o, ref_S = oracle.forward(*(np32(inp[n]) for n in ("q", "k", "v", "log_alpha", "beta")),
                                  np32(inp["S0"]).astype(np.float64))
    packed = {n: np32(inp[n]).reshape((B * T,) + tuple(inp[n].shape[2:])) for n in ("q", "k", "v", "log_alpha", "beta")}
    o, S = oracle.forward_varlen(packed["q"], packed["k"], packed["v"], packed["log_alpha"], packed["beta"],
                                 [0, T, 2 * T, 3 * T], np32(inp["S0"]).astype(np.float64))
    assert np.array_equal(o.reshape(B, T, H, d), ref_o)
    assert np.array_equal(S, ref_S)


def test_sequences_do_not_see_each_other():
    """Changing every input of sequence 1 leaves sequence 0's and 2's results unchanged."""
    inp = varlen_inputs([7, 5, 9], 2, 4, 4, "f32", seed=9, s0_std=0.2)
    args = [np32(inp[n]) for n in ("q", "k", "v", "log_alpha", "beta")]
    o1, S1 = oracle.forward_varlen(*args, inp["cu_seqlens"], np32(inp["S0"]))
    a, b = inp["cu_seqlens"][1], inp["cu_seqlens"][2]
    args2 = [x.copy() for x in args]
    for x in args2:
        x[a:b] = x[a:b][::-1] * 0.5
    o2, S2 = oracle.forward_varlen(*args2, inp["cu_seqlens"], np32(inp["S0"]))
    assert np.array_equal(o1[:a], o2[:a]) and np.array_equal(o1[b:], o2[b:])
    assert np.array_equal(S1[0], S2[0]) and np.array_equal(S1[2], S2[2])
    assert not np.array_equal(S1[1], S2[1])


def test_empty_sequences_keep_their_initial_state():
    inp = varlen_inputs([4, 0, 3, 0], 1, 4, 4, "f32", seed=11, s0_std=0.5)
    args = [np32(inp[n]) for n in ("q", "k", "v", "log_alpha", "beta")]
    o, S = oracle.forward_varlen(*args, inp["cu_seqlens"], np32(inp["S0"]))
    assert np.array_equal(S[1], np32(inp["S0"])[1]) and np.array_equal(S[3], np32(inp["S0"])[3])
    o0, S0z = oracle.forward_varlen(*args, inp["cu_seqlens"], None)
    assert not S0z[1].any() and not S0z[3].any()
