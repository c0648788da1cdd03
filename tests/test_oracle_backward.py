"""Pins for the oracle's backward (reverse mode) of the gated-delta recurrence (CPU only).

The recurrence is "ATMA: Long-Context Language Modeling via Polar Attention and Gated-Delta
Compression Memory", Sec. 3.3.  Its reverse mode is pinned against things other than itself:
central finite differences of the forward oracle, a closed form of the frozen-state case
(alpha = 1, beta = 0), linearity in the incoming gradients, and the chain rule across a split
of the sequence.  Each pin is a plain function of an ``Oracle`` so that
``test_oracle_mutants.py`` runs them against planted mistakes too.
"""
import numpy as np
import pytest

import oracle as oracle_pkg
from test_oracle import rand_inputs, rel_err


def loss(orc, q, k, v, la, be, S0, dO, dSf):
    out, Sf = orc.forward(q, k, v, la, be, S0)
    return float((out * dO).sum() + (Sf * dSf).sum())


def fd_grad(orc, args, name, dO, dSf, n_samples, rng):
    """Central differences at n_samples random positions of input `name`, with the step taken as
    the exact difference of the perturbed values (float32 inputs are perturbed by 2^-10)."""
    a = dict(args)
    x = a[name]
    idx = rng.choice(x.size, size=min(n_samples, x.size), replace=False)
    out = []
    for i in idx:
        xp, xm = x.copy(), x.copy()
        flat_p, flat_m = xp.reshape(-1), xm.reshape(-1)
        h = 1e-6 if x.dtype == np.float64 else 2.0 ** -10
        flat_p[i] = flat_p[i] + h
        flat_m[i] = flat_m[i] - h
        step = float(flat_p[i]) - float(flat_m[i])
        lp = loss(orc, **{**a, name: xp}, dO=dO, dSf=dSf)
        lm = loss(orc, **{**a, name: xm}, dO=dO, dSf=dSf)
        out.append((i, (lp - lm) / step))
    return out


def pin_backward_finite_differences(orc):
    """Every gradient agrees with central differences of the forward oracle."""
    rng = np.random.default_rng(31)
    B, T, H, dk, dv = 1, 6, 2, 4, 3
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    dO = rng.standard_normal((B, T, H, dv))
    dSf = rng.standard_normal((B, H, dv, dk))
    g = dict(zip(("q", "k", "v", "la", "be", "S0"), orc.backward(q, k, v, la, be, S0, dO, dSf)))
    args = dict(q=q, k=k, v=v, la=la, be=be, S0=S0)
    for name in ("q", "k", "v", "la", "be", "S0"):
        for i, fd in fd_grad(orc, args, name, dO, dSf, 12, rng):
            an = g[name].reshape(-1)[i]
            assert abs(an - fd) <= 2e-5 * max(1.0, abs(fd)), (name, i, an, fd)


def pin_backward_frozen_state(orc):
    """alpha = 1, beta = 0: S_t = S0, so dq_t = S0^T do_t, dv = dk = 0,
    dS0 = dS_T + sum_t do_t q_t^T, dlog_alpha_t = <G_t, S0> and dbeta_t = (v_t - S0 k_t) . G_t k_t
    with G_t = dS_T + sum_{t' >= t} do_t' q_t'^T."""
    rng = np.random.default_rng(32)
    B, T, H, dk, dv = 1, 5, 2, 4, 3
    q, k, v, _, _, S0 = rand_inputs(rng, B, T, H, dk, dv)
    la = np.zeros((B, T, H), np.float32)
    be = np.zeros((B, T, H), np.float32)
    dO = rng.standard_normal((B, T, H, dv))
    dSf = rng.standard_normal((B, H, dv, dk))
    gq, gk, gv, gla, gbe, gS0 = orc.backward(q, k, v, la, be, S0, dO, dSf)
    q64, k64, v64 = (x.astype(np.float64) for x in (q, k, v))
    assert rel_err(gq, np.einsum("bhrc,bthr->bthc", S0, dO)) < 1e-13
    assert not gv.any() and not gk.any()
    for h in range(H):
        G = dSf[0, h].copy()
        for t in range(T - 1, -1, -1):
            G += np.outer(dO[0, t, h], q64[0, t, h])
            assert abs(gla[0, t, h] - (G * S0[0, h]).sum()) < 1e-12 * max(1, abs(gla[0, t, h]))
            db = (v64[0, t, h] - S0[0, h] @ k64[0, t, h]) @ (G @ k64[0, t, h])
            assert abs(gbe[0, t, h] - db) < 1e-12 * max(1, abs(db))
        assert rel_err(gS0[0, h], G) < 1e-13


def pin_backward_linearity(orc):
    """The gradients are linear in (dL/dout, dL/dS_final)."""
    rng = np.random.default_rng(33)
    B, T, H, dk, dv = 2, 7, 2, 8, 5
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    d1, d2 = rng.standard_normal((2, B, T, H, dv))
    s1, s2 = rng.standard_normal((2, B, H, dv, dk))
    g1 = orc.backward(q, k, v, la, be, S0, d1, s1)
    g2 = orc.backward(q, k, v, la, be, S0, d2, s2)
    g3 = orc.backward(q, k, v, la, be, S0, 3 * d1 + d2, 3 * s1 + s2)
    for a, b, c in zip(g1, g2, g3):
        assert rel_err(c, 3 * a + b) < 1e-12


def pin_backward_split(orc):
    """Chain rule across a split at T1: the backward of the second part (from the state at T1)
    hands dS0 to the backward of the first part as its dS_final."""
    rng = np.random.default_rng(34)
    B, T, H, dk, dv, T1 = 1, 9, 2, 6, 4, 4
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    dO = rng.standard_normal((B, T, H, dv))
    dSf = rng.standard_normal((B, H, dv, dk))
    full = orc.backward(q, k, v, la, be, S0, dO, dSf)
    sl1, sl2 = (slice(None), slice(0, T1)), (slice(None), slice(T1, T))
    _, S1 = orc.forward(q[sl1], k[sl1], v[sl1], la[sl1], be[sl1], S0)
    second = orc.backward(q[sl2], k[sl2], v[sl2], la[sl2], be[sl2], S1, dO[sl2], dSf)
    first = orc.backward(q[sl1], k[sl1], v[sl1], la[sl1], be[sl1], S0, dO[sl1], second[5])
    for i in range(5):
        assert rel_err(np.concatenate([first[i], second[i]], axis=1), full[i]) < 1e-12
    assert rel_err(first[5], full[5]) < 1e-12


def pin_backward_chunked(orc):
    """The chunkwise adjoint (the algebra the CUDA kernel uses) equals the token-by-token reverse mode for
    chunk lengths 1 .. 64, with a ragged last chunk."""
    rng = np.random.default_rng(36)
    B, T, H, dk, dv = 1, 23, 2, 8, 5
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    dO = rng.standard_normal((B, T, H, dv))
    dSf = rng.standard_normal((B, H, dv, dk))
    ref = orc.backward(q, k, v, la, be, S0, dO, dSf)
    for C in (1, 2, 3, 7, 16, 64):
        got = orc.backward_chunked(q, k, v, la, be, S0, dO, dSf, chunk=C)
        for a, b in zip(got, ref):
            assert rel_err(a, b) < 1e-10, C


BWD_PINS = [pin_backward_finite_differences, pin_backward_frozen_state, pin_backward_linearity,
            pin_backward_split, pin_backward_chunked]


@pytest.fixture(scope="module")
def orc():
    return oracle_pkg.get()


@pytest.mark.parametrize("pin", BWD_PINS, ids=[p.__name__ for p in BWD_PINS])
def test_pin(orc, pin):
    pin(orc)


def test_empty_sequence(orc):
    rng = np.random.default_rng(35)
    q, k, v, la, be, S0 = rand_inputs(rng, 1, 0, 2, 4, 3)
    dSf = rng.standard_normal((1, 2, 3, 4))
    g = orc.backward(q, k, v, la, be, S0, np.zeros((1, 0, 2, 3)), dSf)
    assert g[0].shape == (1, 0, 2, 4) and np.array_equal(g[5], dSf)
