"""Pins for the oracle's input stage and its raw-input forward / decode (CPU only).

The memory reads unit-norm queries and keys ("ATMA: Long-Context Language
Modeling via Polar Attention and Gated-Delta Compression Memory", App. A.2
takes ||q_t|| = ||k_t|| = 1) and gates alpha_t, beta_t in (0, 1) (Sec. 3.3).
The input stage forms them from raw projections: x / sqrt(|x|^2 + 1e-12),
log alpha = -softplus(x_alpha), beta = sigmoid(x_beta).  The pins below check
the stage and the raw forward against a hand-worked example, known values of
softplus and sigmoid, identities between them, scale invariance, and the
already-pinned forward on inputs that the stage leaves unchanged.  Each pin
is a plain function of an ``Oracle`` so that ``test_oracle_mutants.py`` runs
them against planted mistakes too.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle as oracle_pkg
from test_oracle import exact_unit, rel_err

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def pin_raw_hand_worked(orc):
    """Two tokens with raw q, k and gate logits, evaluated by hand (tests/golden/hand_worked_raw_d2.json)."""
    g = json.load(open(os.path.join(GOLDEN, "hand_worked_raw_d2.json")))
    T = len(g["x_alpha"])
    q = np.array(g["q"], np.float32).reshape(1, T, 1, 2)
    k = np.array(g["k"], np.float32).reshape(1, T, 1, 2)
    v = np.array(g["v"], np.float32).reshape(1, T, 1, 2)
    xa = np.array(g["x_alpha"], np.float32).reshape(1, T, 1)
    xb = np.array(g["x_beta"], np.float32).reshape(1, T, 1)
    S0 = np.array(g["S0"], np.float64).reshape(1, 1, 2, 2)
    out, Sf = orc.forward(q, k, v, xa, xb, S0, raw=True)
    np.testing.assert_allclose(out.reshape(T, 2), np.array(g["out"]), rtol=0, atol=1e-6)
    np.testing.assert_allclose(Sf.reshape(2, 2), np.array(g["S_final"]), rtol=0, atol=1e-6)


def pin_input_stage_values(orc):
    """Known values: (3,4)/5, (0,-5)/5, a zero row stays zero; softplus(0) = ln 2,
    softplus(ln 3) = ln 4, softplus(-10) = ln(1 + e^-10); sigmoid(0) = 1/2, sigmoid(+-ln 3) = 3/4, 1/4."""
    q = np.array([[3, 4], [0, -5], [0, 0], [1, 0]], np.float32)
    k = np.array([[0, 2], [0, 0], [-6, 8], [0, 3]], np.float32)
    ln3 = np.float32(math.log(3.0))
    xa = np.array([0.0, ln3, -10.0, 20.0], np.float32)
    xb = np.array([0.0, ln3, -ln3, 0.0], np.float32)
    qn, kn, la, be = orc.input_stage(q, k, xa, xb)
    np.testing.assert_allclose(qn, [[0.6, 0.8], [0, -1], [0, 0], [1, 0]], rtol=0, atol=1e-12)
    np.testing.assert_allclose(kn, [[0, 1], [0, 0], [-0.6, 0.8], [0, 1]], rtol=0, atol=1e-12)
    # ln 3 is rounded to float32: softplus moves by at most 3/4 of that rounding (< 1e-7)
    np.testing.assert_allclose(la[:2], [-math.log(2.0), -math.log(4.0)], rtol=0, atol=1e-7)
    np.testing.assert_allclose(la[2], -4.5398899216870535e-05, rtol=1e-12)   # ln(1 + e^-10)
    np.testing.assert_allclose(la[3], -20.000000002061153, rtol=1e-14)       # 20 + ln(1 + e^-20)
    np.testing.assert_allclose(be, [0.5, 0.75, 0.25, 0.5], rtol=0, atol=1e-7)


def pin_gate_identities(orc):
    """For every x: alpha(x) + beta(x) = 1 (exp(-softplus(x)) = sigmoid(-x)), softplus(x) - softplus(-x) = x,
    beta increasing and log alpha decreasing in x, both gates inside (0, 1)."""
    x = np.linspace(-30, 30, 241).astype(np.float32)
    z = np.zeros((x.size, 1), np.float32)
    _, _, la, be = orc.input_stage(z, z, x, x)
    _, _, la_neg, _ = orc.input_stage(z, z, -x, -x)
    np.testing.assert_allclose(np.exp(la) + be, 1.0, rtol=0, atol=1e-15)
    np.testing.assert_allclose(la_neg - la, x.astype(np.float64), rtol=0, atol=1e-12)
    assert np.all(np.diff(be) > 0) and np.all(np.diff(la) < 0)
    assert np.all(la < 0) and np.all((be > 0) & (be < 1))


def pin_unit_norm(orc):
    """Non-zero rows come out with norm 1 (to the eps), in the direction of the input."""
    rng = np.random.default_rng(21)
    x = (rng.standard_normal((50, 16)) * np.exp(rng.uniform(-3, 3, (50, 1)))).astype(np.float32)
    qn, kn, _, _ = orc.input_stage(x, x[::-1].copy(), np.zeros(50, np.float32), np.zeros(50, np.float32))
    norms = np.sqrt((x.astype(np.float64) ** 2).sum(-1))
    np.testing.assert_allclose(np.linalg.norm(qn, axis=-1), 1.0, rtol=1e-10)
    np.testing.assert_allclose(qn * norms[:, None], x, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(kn, qn[::-1], rtol=0, atol=0)


def pin_raw_scale_invariance(orc):
    """Scaling q or k rows by positive powers of two leaves the raw forward unchanged (to the eps)."""
    rng = np.random.default_rng(22)
    B, T, H, dk, dv = 1, 11, 2, 8, 5
    q = rng.standard_normal((B, T, H, dk)).astype(np.float32)
    k = rng.standard_normal((B, T, H, dk)).astype(np.float32)
    v = rng.standard_normal((B, T, H, dv)).astype(np.float32)
    xa = rng.standard_normal((B, T, H)).astype(np.float32)
    xb = rng.standard_normal((B, T, H)).astype(np.float32)
    S0 = rng.standard_normal((B, H, dv, dk))
    o1, s1 = orc.forward(q, k, v, xa, xb, S0, raw=True)
    o2, s2 = orc.forward(q * 8, k * 2, v, xa, xb, S0, raw=True)
    assert rel_err(o2, o1) < 1e-10 and rel_err(s2, s1) < 1e-10


def pin_raw_matches_forward(orc):
    """On rows of norm exactly 1 the stage leaves q, k unchanged, so the raw forward is the (pinned)
    forward with the gates the stage produces."""
    rng = np.random.default_rng(23)
    B, T, H, dk, dv = 2, 13, 2, 8, 6
    q = exact_unit(rng, (B, T, H, dk))
    k = exact_unit(rng, (B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv)).astype(np.float32)
    xa = (rng.standard_normal((B, T, H)) * 2).astype(np.float32)
    xb = (rng.standard_normal((B, T, H)) * 2).astype(np.float32)
    S0 = rng.standard_normal((B, H, dv, dk))
    _, _, la, be = orc.input_stage(q, k, xa, xb)
    o_raw, s_raw = orc.forward(q, k, v, xa, xb, S0, raw=True)
    o_ref, s_ref = orc.forward(q, k, v, la.astype(np.float32), be.astype(np.float32), S0)
    # the gates are rounded to float32 for the plain forward
    assert rel_err(o_raw, o_ref) < 1e-5 and rel_err(s_raw, s_ref) < 1e-5


def pin_raw_decode(orc):
    """Raw decode steps, one token at a time, give the raw forward's outputs and final state."""
    rng = np.random.default_rng(24)
    T, B, H, dk, dv = 4, 2, 3, 8, 5
    q = rng.standard_normal((B, T, H, dk)).astype(np.float32)
    k = rng.standard_normal((B, T, H, dk)).astype(np.float32)
    v = rng.standard_normal((B, T, H, dv)).astype(np.float32)
    xa = rng.standard_normal((B, T, H)).astype(np.float32)
    xb = rng.standard_normal((B, T, H)).astype(np.float32)
    S0 = rng.standard_normal((B, H, dv, dk))
    out, Sf = orc.forward(q, k, v, xa, xb, S0, raw=True)
    S = S0.copy()
    for t in range(T):
        o = orc.decode_step(q[:, t].copy(), k[:, t].copy(), v[:, t].copy(), xa[:, t].copy(), xb[:, t].copy(),
                            S, raw=True)
        assert rel_err(o, out[:, t]) < 1e-13
    assert rel_err(S, Sf) < 1e-13


RAW_PINS = [pin_raw_hand_worked, pin_input_stage_values, pin_gate_identities, pin_unit_norm,
            pin_raw_scale_invariance, pin_raw_matches_forward, pin_raw_decode]


@pytest.fixture(scope="module")
def orc():
    return oracle_pkg.get()


@pytest.mark.parametrize("pin", RAW_PINS, ids=[p.__name__ for p in RAW_PINS])
def test_pin(orc, pin):
    pin(orc)


def test_raw_varlen_runs_each_sequence_alone():
    rng = np.random.default_rng(25)
    lens = [3, 0, 5]
    T, H, dk, dv = sum(lens), 2, 4, 3
    q = rng.standard_normal((T, H, dk)).astype(np.float32)
    k = rng.standard_normal((T, H, dk)).astype(np.float32)
    v = rng.standard_normal((T, H, dv)).astype(np.float32)
    xa = rng.standard_normal((T, H)).astype(np.float32)
    xb = rng.standard_normal((T, H)).astype(np.float32)
    S0 = rng.standard_normal((3, H, dv, dk))
    cu = [0, 3, 3, 8]
    out, Sf = oracle_pkg.forward_varlen_raw(q, k, v, xa, xb, cu, S0)
    for i in range(3):
        a, b = cu[i], cu[i + 1]
        if a == b:
            assert np.array_equal(Sf[i], S0[i])
            continue
        o, s = oracle_pkg.forward_raw(q[None, a:b], k[None, a:b], v[None, a:b], xa[None, a:b], xb[None, a:b],
                                      S0[i:i + 1])
        assert np.array_equal(out[a:b], o[0]) and np.array_equal(Sf[i], s[0])
