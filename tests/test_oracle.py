"""Pins for the float64 oracle (CPU only).

The oracle is checked against things other than itself: a hand-worked
example, closed forms of special cases, the state bound of the paper's
Appendix A.2, brute force over explicit matrix products, algebraic
invariants, and an independent chunkwise derivation.  Every pin is a plain
function of an ``Oracle`` so that ``test_oracle_mutants.py`` can re-run the
same pins against deliberately broken copies of the oracle source and check
that each planted mistake is caught.

Source for every pin: "ATMA: Long-Context Language Modeling via Polar
Attention and Gated-Delta Compression Memory", Sec. 3.3 (the gated-delta
memory equation) and App. A.2 (bounded recurrent state).
"""
import json
import os

import numpy as np
import pytest

import oracle as oracle_pkg

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ----------------------------------------------------------------------------- helpers
def rand_unit(rng, shape):
    x = rng.standard_normal(shape)
    x /= np.linalg.norm(x, axis=-1, keepdims=True)
    return x.astype(np.float32)


def exact_unit(rng, shape):
    """Rows of norm exactly 1 in float32: m = 4 (or 1) entries of +-1/sqrt(m) at random places."""
    *lead, d = shape
    m = 4 if d >= 4 else 1
    out = np.zeros(shape, np.float32)
    flat = out.reshape(-1, d)
    for row in flat:
        idx = rng.choice(d, size=m, replace=False)
        row[idx] = rng.choice([-1.0, 1.0], size=m) / np.sqrt(m)
    return out


def rand_inputs(rng, B, T, H, dk, dv, s0=True):
    q = rand_unit(rng, (B, T, H, dk))
    k = rand_unit(rng, (B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv)).astype(np.float32)
    beta = (1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))).astype(np.float32)
    log_alpha = (-np.log1p(np.exp(rng.standard_normal((B, T, H))))).astype(np.float32)
    S0 = rng.standard_normal((B, H, dv, dk)) * 0.5 if s0 else None
    return q, k, v, log_alpha, beta, S0


def rel_err(a, b):
    scale = max(np.abs(b).max(), 1e-300)
    return np.abs(a - b).max() / scale


# ----------------------------------------------------------------------------- pins
def pin_hand_worked(orc):
    """Four tokens evaluated by hand from the Sec. 3.3 equation (tests/golden/hand_worked_d2.json)."""
    g = json.load(open(os.path.join(GOLDEN, "hand_worked_d2.json")))
    T = len(g["alpha"])
    q = np.array(g["q"], np.float32).reshape(1, T, 1, 2)
    k = np.array(g["k"], np.float32).reshape(1, T, 1, 2)
    v = np.array(g["v"], np.float32).reshape(1, T, 1, 2)
    la = np.log(np.array(g["alpha"])).astype(np.float32).reshape(1, T, 1)
    be = np.array(g["beta"], np.float32).reshape(1, T, 1)
    out, Sf = orc.forward(q, k, v, la, be)
    np.testing.assert_allclose(out.reshape(T, 2), np.array(g["out"]), rtol=0, atol=1e-6)
    np.testing.assert_allclose(Sf.reshape(2, 2), np.array(g["S_final"]), rtol=0, atol=1e-6)


def pin_identity_gates(orc):
    """alpha = 1, beta = 0: the state never changes, so S_T = S0 exactly and o_t = S0 q_t."""
    rng = np.random.default_rng(1)
    B, T, H, dk, dv = 2, 9, 3, 8, 6
    q, k, v, _, _, S0 = rand_inputs(rng, B, T, H, dk, dv)
    la = np.zeros((B, T, H), np.float32)
    be = np.zeros((B, T, H), np.float32)
    out, Sf = orc.forward(q, k, v, la, be, S0)
    assert np.array_equal(Sf, S0)
    expect = np.einsum("bhrc,bthc->bthr", S0, q.astype(np.float64))
    assert rel_err(out, expect) < 1e-14


def pin_unit_write(orc):
    """alpha = 1, beta = 1, ||k|| = 1 exactly: S_t k_t = v_t for any history (since (I - k k^T) k = 0).
    With q_t = k_t the output is o_t = v_t."""
    rng = np.random.default_rng(2)
    B, T, H, dk, dv = 2, 12, 2, 16, 7
    k = exact_unit(rng, (B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv)).astype(np.float32)
    S0 = rng.standard_normal((B, H, dv, dk))
    la = np.zeros((B, T, H), np.float32)
    be = np.ones((B, T, H), np.float32)
    out, _ = orc.forward(k, k, v, la, be, S0)
    assert rel_err(out, v.astype(np.float64)) < 1e-13


def pin_reset(orc):
    """alpha = 0 (log_alpha = -inf) erases the past: S_t = beta_t v_t k_t^T, o_t = beta_t (k_t . q_t) v_t."""
    rng = np.random.default_rng(3)
    B, T, H, dk, dv = 1, 6, 2, 8, 5
    q, k, v, _, beta, S0 = rand_inputs(rng, B, T, H, dk, dv)
    la = np.full((B, T, H), -np.inf, np.float32)
    out, Sf = orc.forward(q, k, v, la, beta, S0)
    kq = np.einsum("bthc,bthc->bth", k.astype(np.float64), q.astype(np.float64))
    expect = beta[..., None].astype(np.float64) * kq[..., None] * v.astype(np.float64)
    assert rel_err(out, expect) < 1e-14
    Sexp = np.einsum("bh,bhr,bhc->bhrc", beta[:, -1].astype(np.float64), v[:, -1].astype(np.float64),
                     k[:, -1].astype(np.float64))
    assert rel_err(Sf, Sexp) < 1e-14


def _orthonormal_case(rng, T, dk, dv, exact):
    """Keys k_t = s_t e_{i_t}: (I - beta k k^T) only scales column i_t by (1 - beta), so
    column i_t evolves as S[:, i] <- alpha ((1 - beta) S[:, i]) + beta s v and every other
    column as S[:, j] <- alpha S[:, j].  Outputs use q_t = e_{j_t}: o_t = S_t[:, j_t]."""
    idx = rng.integers(0, dk, size=T)
    sgn = rng.choice([-1.0, 1.0], size=T)
    qi = rng.integers(0, dk, size=T)
    k = np.zeros((1, T, 1, dk), np.float32)
    q = np.zeros((1, T, 1, dk), np.float32)
    k[0, np.arange(T), 0, idx] = sgn
    q[0, np.arange(T), 0, qi] = 1.0
    if exact:   # dyadic values with few bits: every operation is exact in double
        la = np.zeros((1, T, 1), np.float32)
        be = rng.choice([0.25, 0.5, 0.75, 1.0], size=(1, T, 1)).astype(np.float32)
        v = (rng.integers(-64, 65, size=(1, T, 1, dv)) / 16.0).astype(np.float32)
        S0 = rng.integers(-64, 65, size=(1, 1, dv, dk)) / 16.0
    else:
        la = (-rng.uniform(0.0, 1.0, size=(1, T, 1))).astype(np.float32)
        be = rng.uniform(0.0, 1.0, size=(1, T, 1)).astype(np.float32)
        v = rng.standard_normal((1, T, 1, dv)).astype(np.float32)
        S0 = rng.standard_normal((1, 1, dv, dk))
    S = S0[0, 0].copy()
    outs = np.zeros((T, dv))
    for t in range(T):
        a, b, i = np.exp(np.float64(la[0, t, 0])), np.float64(be[0, t, 0]), idx[t]
        col = a * (1.0 - b) * S[:, i] + b * sgn[t] * v[0, t, 0].astype(np.float64)
        S = a * S
        S[:, i] = col
        outs[t] = S[:, qi[t]]
    return q, k, v, la, be, S0, outs, S


def pin_orthonormal_keys(orc):
    rng = np.random.default_rng(4)
    q, k, v, la, be, S0, outs, S = _orthonormal_case(rng, 40, 8, 5, exact=False)
    out, Sf = orc.forward(q, k, v, la, be, S0)
    assert rel_err(out[0, :, 0], outs) < 1e-13
    assert rel_err(Sf[0, 0], S) < 1e-13


def pin_orthonormal_keys_exact(orc):
    """Same closed form with alpha = 1 and dyadic data: bit-exact equality."""
    rng = np.random.default_rng(5)
    q, k, v, la, be, S0, outs, S = _orthonormal_case(rng, 24, 6, 4, exact=True)
    out, Sf = orc.forward(q, k, v, la, be, S0)
    assert np.array_equal(out[0, :, 0], outs)
    assert np.array_equal(Sf[0, 0], S)


def pin_state_bound(orc):
    """App. A.2: with ||k_t|| = 1, ||v_t|| <= V, 0 <= beta_t <= 1, 0 <= alpha_t <= abar < 1,
    ||S_t||_F <= abar^t ||S_0||_F + V / (1 - abar) at every t."""
    rng = np.random.default_rng(6)
    T, dk, dv, abar, V = 300, 16, 16, 0.9, 3.0
    k = exact_unit(rng, (T, 1, 1, dk))
    q = rand_unit(rng, (T, 1, 1, dk))
    v = rng.standard_normal((T, 1, 1, dv))
    v = (v / np.linalg.norm(v, axis=-1, keepdims=True) * V * rng.uniform(0.5, 1.0, (T, 1, 1, 1))).astype(np.float32)
    la = np.log(rng.uniform(0.0, abar, (T, 1, 1))).astype(np.float32)
    be = rng.uniform(0.0, 1.0, (T, 1, 1)).astype(np.float32)
    S = rng.standard_normal((1, 1, dv, dk)) * 20.0
    n0 = np.linalg.norm(S)
    vmax = np.linalg.norm(v.astype(np.float64), axis=-1).max()
    assert vmax <= V * (1 + 1e-6)
    for t in range(T):
        orc.decode_step(q[t], k[t], v[t], la[t], be[t], S)
        bound = abar ** (t + 1) * n0 + V / (1 - abar)
        assert np.linalg.norm(S) <= bound * (1 + 1e-9), (t, np.linalg.norm(S), bound)


def pin_dense_product(orc):
    """Brute force: explicit factors alpha_t (I - beta_t k_t k_t^T), products from scratch, T <= 8."""
    rng = np.random.default_rng(7)
    for dk, dv, T in [(3, 5, 8), (4, 4, 7), (6, 2, 5), (5, 3, 1)]:
        q, k, v, la, be, S0 = rand_inputs(rng, 1, T, 1, dk, dv)
        out, Sf = orc.forward(q, k, v, la, be, S0)
        od, Sd = orc.dense_product(q[0, :, 0], k[0, :, 0], v[0, :, 0], la[0, :, 0], be[0, :, 0], S0[0, 0])
        assert rel_err(out[0, :, 0], od) < 1e-12
        assert rel_err(Sf[0, 0], Sd) < 1e-12


def pin_chunked(orc):
    """The chunkwise (UT-transform) form equals the token recurrence for any chunk length."""
    rng = np.random.default_rng(8)
    B, T, H, dk, dv = 2, 70, 2, 8, 6
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    ref, Sref = orc.forward(q, k, v, la, be, S0)
    for C in (1, 2, 3, 16, 64, 70, 128):
        out, Sf = orc.forward_chunked(q, k, v, la, be, S0, chunk=C)
        assert rel_err(out, ref) < 1e-10, C
        assert rel_err(Sf, Sref) < 1e-10, C


def pin_segment_transfer(orc):
    """A run of tokens maps the state affinely: S_end = S_start M + Bseg, for any S_start."""
    rng = np.random.default_rng(9)
    T, dk, dv = 45, 8, 5
    q, k, v, la, be, _ = rand_inputs(rng, 1, T, 1, dk, dv, s0=False)
    M, Bs = orc.segment_transfer(k[0, :, 0], v[0, :, 0], la[0, :, 0], be[0, :, 0], chunk=16)
    for _ in range(3):
        S0 = rng.standard_normal((1, 1, dv, dk))
        _, Sf = orc.forward(q, k, v, la, be, S0)
        assert rel_err(S0[0, 0] @ M + Bs, Sf[0, 0]) < 1e-11


def pin_linearity(orc):
    """Outputs and final state are affine in S0 and linear in V: f(S0, V1 + V2) = f(S0, V1) + f(0, V2)."""
    rng = np.random.default_rng(10)
    B, T, H, dk, dv = 1, 20, 2, 8, 8
    q, k, _, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    v1 = (rng.integers(-2048, 2049, size=(B, T, H, dv)) / 1024.0).astype(np.float32)
    v2 = (rng.integers(-2048, 2049, size=(B, T, H, dv)) / 1024.0).astype(np.float32)
    o12, S12 = orc.forward(q, k, v1 + v2, la, be, S0)
    o1, S1 = orc.forward(q, k, v1, la, be, S0)
    o2, S2 = orc.forward(q, k, v2, la, be, None)
    assert rel_err(o12, o1 + o2) < 1e-12
    assert rel_err(S12, S1 + S2) < 1e-12


def pin_split(orc):
    """Continuation: forward(T) == forward(T1) then forward(T - T1) from its final state,
    and == T single-token decode steps."""
    rng = np.random.default_rng(11)
    B, T, H, dk, dv = 2, 17, 2, 8, 4
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    ref, Sref = orc.forward(q, k, v, la, be, S0)
    T1 = 6
    oa, Sa = orc.forward(q[:, :T1], k[:, :T1], v[:, :T1], la[:, :T1], be[:, :T1], S0)
    ob, Sb = orc.forward(q[:, T1:], k[:, T1:], v[:, T1:], la[:, T1:], be[:, T1:], Sa)
    assert rel_err(np.concatenate([oa, ob], axis=1), ref) < 1e-13
    assert rel_err(Sb, Sref) < 1e-13
    S = S0.copy()
    for t in range(T):
        o = orc.decode_step(q[:, t], k[:, t], v[:, t], la[:, t], be[:, t], S)
        assert rel_err(o, ref[:, t]) < 1e-13
    assert rel_err(S, Sref) < 1e-13


def pin_permutation(orc):
    """(batch, head) problems are independent: permuting heads and batches permutes the results."""
    rng = np.random.default_rng(12)
    B, T, H, dk, dv = 3, 10, 4, 8, 6
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    ref, Sref = orc.forward(q, k, v, la, be, S0)
    pb, ph = rng.permutation(B), rng.permutation(H)

    def perm(x, hax):
        return np.ascontiguousarray(np.take(np.take(x, pb, axis=0), ph, axis=hax))

    out, Sf = orc.forward(perm(q, 2), perm(k, 2), perm(v, 2), perm(la, 2), perm(be, 2), perm(S0, 1))
    assert np.array_equal(out, perm(ref, 2))
    assert np.array_equal(Sf, perm(Sref, 1))


def pin_empty(orc):
    """T = 0: no outputs, the final state is the initial state (or zero)."""
    rng = np.random.default_rng(13)
    q, k, v, la, be, S0 = rand_inputs(rng, 2, 0, 2, 4, 3)
    out, Sf = orc.forward(q, k, v, la, be, S0)
    assert out.shape == (2, 0, 2, 3) and np.array_equal(Sf, S0)
    _, Sz = orc.forward(q, k, v, la, be, None)
    assert not Sz.any()


PINS = [pin_hand_worked, pin_identity_gates, pin_unit_write, pin_reset, pin_orthonormal_keys,
        pin_orthonormal_keys_exact, pin_state_bound, pin_dense_product, pin_chunked,
        pin_segment_transfer, pin_linearity, pin_split, pin_permutation, pin_empty]


@pytest.fixture(scope="module")
def orc():
    return oracle_pkg.get()


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(orc, pin):
    pin(orc)


def test_threads_do_not_change_results(orc):
    rng = np.random.default_rng(14)
    q, k, v, la, be, S0 = rand_inputs(rng, 2, 33, 3, 8, 8)
    a = orc.forward(q, k, v, la, be, S0, nthreads=1)
    b = orc.forward(q, k, v, la, be, S0, nthreads=4)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
