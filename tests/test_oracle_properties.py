"""Randomised agreement between the oracle's independent forms (CPU only, hypothesis).

Across random small shapes: the chunkwise forward equals the token recurrence for any chunk length;
decode steps equal the forward; the chunkwise reverse mode equals the token-by-token one; grouped
heads equal the plain forward on repeated key-value inputs.  The forms are separate code written from
the same equation ("ATMA: Long-Context Language Modeling via Polar Attention and Gated-Delta
Compression Memory", Sec. 3.3), so agreement across random shapes pins indexing and masking.
"""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle
from test_oracle import rand_inputs, rel_err

shapes = st.tuples(st.integers(1, 2), st.integers(0, 19), st.integers(1, 3), st.sampled_from([1, 2, 4, 8]),
                   st.sampled_from([1, 3, 4]), st.integers(1, 9), st.integers(0, 2 ** 31 - 1))


@settings(max_examples=40, deadline=None)
@given(shapes)
def test_chunked_forward_and_decode_agree_with_the_recurrence(sh):
    B, T, H, dk, dv, C, seed = sh
    rng = np.random.default_rng(seed)
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    o, S = oracle.forward(q, k, v, la, be, S0)
    oc, Sc = oracle.forward_chunked(q, k, v, la, be, S0, chunk=C)
    assert rel_err(oc, o) < 1e-10 if o.size else True
    assert rel_err(Sc, S) < 1e-10
    Sd = S0.copy()
    for t in range(T):
        od = oracle.decode_step(q[:, t].copy(), k[:, t].copy(), v[:, t].copy(), la[:, t].copy(), be[:, t].copy(), Sd)
        assert rel_err(od, o[:, t]) < 1e-12
    assert rel_err(Sd, S) < 1e-12


@settings(max_examples=25, deadline=None)
@given(shapes)
def test_chunked_reverse_mode_agrees_with_the_token_reverse_mode(sh):
    B, T, H, dk, dv, C, seed = sh
    rng = np.random.default_rng(seed)
    q, k, v, la, be, S0 = rand_inputs(rng, B, T, H, dk, dv)
    dO = rng.standard_normal((B, T, H, dv))
    dSf = rng.standard_normal((B, H, dv, dk))
    ref = oracle.backward(q, k, v, la, be, S0, dO, dSf)
    got = oracle.get().backward_chunked(q, k, v, la, be, S0, dO, dSf, chunk=C)
    for a, b in zip(got, ref):
        if b.size:
            assert rel_err(a, b) < 1e-9


@settings(max_examples=25, deadline=None)
@given(st.integers(1, 2), st.integers(0, 12), st.integers(1, 3), st.integers(1, 4), st.integers(0, 2 ** 31 - 1))
def test_grouped_heads_equal_repeated_key_value_heads(B, T, Hkv, G, seed):
    rng = np.random.default_rng(seed)
    dk, dv = 4, 3
    q, _, _, _, _, _ = rand_inputs(rng, B, T, Hkv * G, dk, dv)
    _, k, v, la, be, S0 = rand_inputs(rng, B, T, Hkv, dk, dv)
    o, S = oracle.forward_grouped(q, k, v, la, be, S0)
    rep = lambda x, ax: np.repeat(x, G, axis=ax)  # noqa: E731
    ro, rS = oracle.forward(q, rep(k, 2), rep(v, 2), rep(la, 2), rep(be, 2), rep(S0, 1))
    assert np.array_equal(o, ro) and np.array_equal(rep(S, 1), rS)
