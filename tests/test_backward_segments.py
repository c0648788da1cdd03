"""CPU check of the algebra the reverse segments of the tensor-core backward rest on (not of its
kernels), on the float64 oracle alone.

The memory is the Sec. 3.3 recurrence of "ATMA: Long-Context Language Modeling via Polar Attention and
Gated-Delta Compression Memory".  A run of tokens maps the state affinely, S_end = S_start M + B.  The
reverse mode over that run therefore maps the adjoint of the state leaving it to the adjoint of the
state entering it affinely too, dS_start = dS_end M^T + B', where B' is the run's own term: it depends
on the run's output adjoints and inputs, not on the state.  The backward cuts long sequences into
segments on that basis: it forms each segment's (B', M^T), chains them from dS_final, and then walks
every segment from its own entry adjoint.
"""
import numpy as np

import oracle
from gdn_inputs import as_f32_numpy, forward_inputs

NAMES = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0")


def rel_err(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def problem(T, d, seed, alpha_mu=-2.0):
    inp = forward_inputs(1, T, 1, d, d, "f32", seed=seed, s0_std=0.3, alpha_mu=alpha_mu)
    x = [as_f32_numpy(inp[n]) for n in ("q", "k", "v", "log_alpha", "beta")]
    S0 = as_f32_numpy(inp["S0"]).astype(np.float64)
    rng = np.random.default_rng(seed + 1)
    d_out = rng.standard_normal((1, T, 1, d))
    dS_final = rng.standard_normal((1, 1, d, d))
    return x, S0, d_out, dS_final


def test_adjoint_map_is_affine_with_the_transposed_forward_transfer():
    """dS_start(dO, E) - dS_start(dO, 0) = E M^T for several E, M the run's forward transfer; and the run's
    own term B' = dS_start(dO, 0) does not change with the state entering the run."""
    T, d = 150, 16
    # alpha close to 1, so that M stays of order one and the difference below is not lost to rounding
    (q, k, v, la, be), S0, d_out, _ = problem(T, d, seed=31, alpha_mu=-8.0)
    M, _ = oracle.get().segment_transfer(k[0, :, 0], v[0, :, 0], la[0, :, 0], be[0, :, 0], chunk=64)
    base = oracle.backward(q, k, v, la, be, S0, d_out, None)[5]
    rng = np.random.default_rng(32)
    for _ in range(3):
        E = rng.standard_normal((1, 1, d, d))
        got = oracle.backward(q, k, v, la, be, S0, d_out, E)[5]
        assert rel_err(got[0, 0] - base[0, 0], E[0, 0] @ M.T) < 1e-11
    other = oracle.backward(q, k, v, la, be, 5.0 * S0 + 1.0, d_out, None)[5]
    assert rel_err(other, base) < 1e-12


def test_segmented_reverse_walk_equals_the_whole_walk():
    """Cut at a chunk boundary and at a ragged point: walking the last run from dS_final, then the first
    run from the adjoint reached (the state entering each run from the forward), gives the whole reverse
    mode's gradients; and the entry adjoint of the last run is dS_final M2^T + B'2."""
    T, d = 170, 16
    (q, k, v, la, be), S0, d_out, dSf = problem(T, d, seed=41)
    whole = oracle.backward(q, k, v, la, be, S0, d_out, dSf)
    for cut in (128, 97):
        first = [a[:, :cut] for a in (q, k, v, la, be)]
        last = [a[:, cut:] for a in (q, k, v, la, be)]
        _, S_cut = oracle.forward(*first, S0)  # the state entering the last run
        g2 = oracle.backward(*last, S_cut, d_out[:, cut:], dSf)
        # the entry adjoint of the last run through its affine map
        M2, _ = oracle.get().segment_transfer(last[1][0, :, 0], last[2][0, :, 0], last[3][0, :, 0],
                                              last[4][0, :, 0], chunk=64)
        b2 = oracle.backward(*last, S_cut, d_out[:, cut:], None)[5]
        assert rel_err(g2[5][0, 0], dSf[0, 0] @ M2.T + b2[0, 0]) < 1e-11
        g1 = oracle.backward(*first, S0, d_out[:, :cut], g2[5])
        for i, name in enumerate(NAMES[:5]):
            joined = np.concatenate([g1[i], g2[i]], axis=1)
            assert rel_err(joined, whole[i]) < 1e-11, (cut, name)
        assert rel_err(g1[5], whole[5]) < 1e-11, cut
