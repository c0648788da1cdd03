"""Pins for the oracle's grouped heads (CPU only).

Query head h reads the memory of key-value head h // G (G = Hq / Hkv); each memory is written by
its own k, v and gates with the Sec. 3.3 recurrence of "ATMA: Long-Context Language Modeling via
Polar Attention and Gated-Delta Compression Memory" (whose attention layers have 8 query and 2
key-value heads, Sec. 3).  Pinned against the already-pinned plain forward: G = 1 is the plain
forward; any G equals the plain forward on k, v, gates and S0 repeated for every query head of a
group; outputs are linear in q; the decode step is the forward over one token.
"""
import numpy as np
import pytest

import oracle as oracle_pkg
from test_oracle import rand_inputs, rand_unit


def grouped_inputs(rng, B, T, Hq, Hkv, dk, dv):
    q = rand_unit(rng, (B, T, Hq, dk))
    k = rand_unit(rng, (B, T, Hkv, dk))
    v = rng.standard_normal((B, T, Hkv, dv)).astype(np.float32)
    be = (1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, Hkv))))).astype(np.float32)
    la = (-np.log1p(np.exp(rng.standard_normal((B, T, Hkv))))).astype(np.float32)
    S0 = rng.standard_normal((B, Hkv, dv, dk)) * 0.5
    return q, k, v, la, be, S0


def pin_grouped_single_group_is_plain(orc):
    rng = np.random.default_rng(41)
    q, k, v, la, be, S0 = rand_inputs(rng, 2, 9, 3, 8, 5)
    a = orc.forward_grouped(q, k, v, la, be, S0)
    b = orc.forward(q, k, v, la, be, S0)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def pin_grouped_equals_repeated_plain(orc):
    """Repeating k, v, gates and S0 for every query head of a group gives the plain forward the
    same outputs; its final states are the group's memory, G times."""
    rng = np.random.default_rng(42)
    B, T, Hq, Hkv, dk, dv = 2, 11, 8, 2, 8, 6
    q, k, v, la, be, S0 = grouped_inputs(rng, B, T, Hq, Hkv, dk, dv)
    G = Hq // Hkv
    out, Sf = orc.forward_grouped(q, k, v, la, be, S0)
    rep = lambda x, ax: np.repeat(x, G, axis=ax)  # noqa: E731
    ref_o, ref_S = orc.forward(q, rep(k, 2), rep(v, 2), rep(la, 2), rep(be, 2), rep(S0, 1))
    assert np.array_equal(out, ref_o)
    assert np.array_equal(rep(Sf, 1), ref_S)


def pin_grouped_linear_in_q(orc):
    rng = np.random.default_rng(43)
    q1, k, v, la, be, S0 = grouped_inputs(rng, 1, 7, 4, 2, 8, 5)
    q2 = rand_unit(rng, q1.shape)
    o1, _ = orc.forward_grouped(q1, k, v, la, be, S0)
    o2, _ = orc.forward_grouped(q2, k, v, la, be, S0)
    o3, _ = orc.forward_grouped((q1 + 2 * q2).astype(np.float32), k, v, la, be, S0)
    np.testing.assert_allclose(o3, o1 + 2 * o2, rtol=0, atol=1e-6 * np.abs(o3).max())


def pin_grouped_decode(orc):
    rng = np.random.default_rng(44)
    q, k, v, la, be, S0 = grouped_inputs(rng, 2, 3, 6, 3, 8, 4)
    out, Sf = orc.forward_grouped(q, k, v, la, be, S0)
    S = S0.copy()
    for t in range(3):
        o, S = orc.forward_grouped(q[:, t:t + 1], k[:, t:t + 1], v[:, t:t + 1], la[:, t:t + 1], be[:, t:t + 1], S)
        assert np.array_equal(o[:, 0], out[:, t])
    assert np.array_equal(S, Sf)


GROUPED_PINS = [pin_grouped_single_group_is_plain, pin_grouped_equals_repeated_plain, pin_grouped_linear_in_q,
                pin_grouped_decode]


@pytest.fixture(scope="module")
def orc():
    return oracle_pkg.get()


@pytest.mark.parametrize("pin", GROUPED_PINS, ids=[p.__name__ for p in GROUPED_PINS])
def test_pin(orc, pin):
    pin(orc)


def test_module_decode_helper_updates_state_in_place():
    rng = np.random.default_rng(45)
    q, k, v, la, be, S0 = grouped_inputs(rng, 1, 1, 4, 2, 8, 4)
    S = S0.copy()
    o = oracle_pkg.decode_step_grouped(q[:, 0], k[:, 0], v[:, 0], la[:, 0], be[:, 0], S)
    ro, rS = oracle_pkg.forward_grouped(q, k, v, la, be, S0)
    assert np.array_equal(o, ro[:, 0]) and np.array_equal(S, rS)
