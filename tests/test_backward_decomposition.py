"""CPU check of the decomposition the tensor-core reverse mode computes (not of its kernels): the
products of its two passes, written out in float64 numpy with the same stacked operands, must give
the oracle's reverse mode.

The forward is the Sec. 3.3 recurrence of "ATMA: Long-Context Language Modeling via Polar Attention
and Gated-Delta Compression Memory" in chunkwise form; pass 1 walks the chunks backwards with the
state adjoint (dU^T = dO^T P + (dS K^T) diag(dl), dR^T = dU^T T, dS <- gamma_C dS + dO^T diag(gamma) Q
- dR^T diag(beta gamma) K), pass 2 forms each chunk's gradients from S, dS' and dR: [Q;K]K^T,
[Q;K]S^T, dS'K^T, U^T = Y^T (T diag(beta))^T, [dO; dR] U^T, and [dQ; dK] = A1 [Q; K] + (scaled)
[dO; dR] S + [.; U] dS' with A1 = [[0, dP o E], [(dP o E)^T, F + F^T]].
"""
import numpy as np

import oracle
from gdn_inputs import as_f32_numpy, forward_inputs

C = 64


def chunk_terms(q, k, v, la, be, t0, n, d):
    Q = np.zeros((C, d)); K = np.zeros((C, d)); V = np.zeros((C, d))
    lg = np.zeros(C); bb = np.zeros(C)
    Q[:n], K[:n], V[:n] = q[t0:t0 + n], k[t0:t0 + n], v[t0:t0 + n]
    lg[:n] = np.maximum(la[t0:t0 + n], -40.0)
    bb[:n] = be[t0:t0 + n]
    g = np.cumsum(lg)
    E = np.exp(g[:, None] - g[None, :])
    low, lowe = np.tril(np.ones((C, C)), -1), np.tril(np.ones((C, C)))
    A = bb[:, None] * E * (K @ K.T) * low
    return dict(Q=Q, K=K, V=V, g=g, gam=np.exp(g), dl=np.exp(g[-1] - g), gC=np.exp(g[-1]), E=E, bb=bb,
                T=np.linalg.inv(np.eye(C) + A), P=E * (Q @ K.T) * lowe, low=low, lowe=lowe)


def decomposed_backward(q, k, v, la, be, S0, dO, dSf):
    """One (b, h): the two passes, float64."""
    T, d = q.shape
    nch = -(-T // C)
    parts = [chunk_terms(q, k, v, la, be, c * C, min(C, T - c * C), d) for c in range(nch)]
    S, ck = S0.copy(), []
    for x in parts:  # forward recompute: the state entering every chunk
        ck.append(S.copy())
        U = x["T"] @ (x["bb"][:, None] * (x["V"] - x["gam"][:, None] * (x["K"] @ S.T)))
        S = x["gC"] * S + U.T @ (x["dl"][:, None] * x["K"])
    dOp = np.zeros((nch * C, d)); dOp[:T] = dO
    dS, dSp, dRs = dSf.copy(), [None] * nch, [None] * nch
    dv = np.zeros((T, d))
    for c in reversed(range(nch)):  # pass 1
        x, DO = parts[c], dOp[c * C:(c + 1) * C]
        dSp[c] = dS.copy()
        dUT = DO.T @ x["P"] + (dS @ x["K"].T) * x["dl"][None, :]
        dRT = dUT @ x["T"]
        dRs[c] = dRT.T
        n = min(C, T - c * C)
        dv[c * C:c * C + n] = (x["bb"][:, None] * dRT.T)[:n]
        dS = x["gC"] * dS + DO.T @ (x["gam"][:, None] * x["Q"]) + ((-x["bb"] * x["gam"])[None, :] * dRT) @ x["K"]
    dq, dk, dla, dbeta = np.zeros((T, d)), np.zeros((T, d)), np.zeros(T), np.zeros(T)
    for c in range(nch):  # pass 2
        x, S, dSc, dR, DO = parts[c], ck[c], dSp[c], dRs[c], dOp[c * C:(c + 1) * C]
        n = min(C, T - c * C)
        QK = np.vstack([x["Q"], x["K"]])
        G, Z, D2 = QK @ x["K"].T, QK @ S.T, dSc @ x["K"].T
        dg = x["gam"] * np.sum(Z[:C] * DO, axis=1)
        X = x["gam"][:, None] * Z[C:]
        Y = x["V"] - X
        db = np.sum(dR * Y, axis=1)
        dg -= x["bb"] * np.sum(dR * X, axis=1)
        UT = Y.T @ (x["T"] * x["bb"][None, :]).T
        w = x["dl"] * np.sum(UT * D2, axis=0)
        dg -= w
        DG = np.vstack([DO, dR]) @ UT
        e_le, e_lt = x["E"] * x["lowe"], x["E"] * x["low"]
        gp = DG[:C] * e_le * G[:C]
        dg += gp.sum(1) - gp.sum(0)
        dA = -DG[C:] * x["low"]
        ek = e_lt * G[C:]
        db += np.sum(dA * ek, axis=1)
        ga = dA * x["bb"][:, None] * ek
        dg += ga.sum(1) - ga.sum(0)
        F = dA * x["bb"][:, None] * e_lt
        dPE = DG[:C] * e_le
        A1 = np.zeros((2 * C, 2 * C))
        A1[:C, C:], A1[C:, :C], A1[C:, C:] = dPE, dPE.T, F + F.T
        H1, H2, H3 = A1 @ QK, np.vstack([DO, dR]) @ S, UT.T @ dSc
        dQ = H1[:C] + x["gam"][:, None] * H2[:C]
        dK = H1[C:] - (x["bb"] * x["gam"])[:, None] * H2[C:] + x["dl"][:, None] * H3
        suffix = np.cumsum(dg[::-1])[::-1] + x["gC"] * np.sum(dSc * S) + w.sum()
        sl = slice(c * C, c * C + n)
        dq[sl], dk[sl], dla[sl], dbeta[sl] = dQ[:n], dK[:n], suffix[:n], db[:n]
    dla[la < -40.0] = 0.0
    return dq, dk, dv, dla, dbeta, dS


def test_decomposition_matches_the_oracle_reverse_mode():
    B, T, H, d = 1, 150, 1, 128  # three chunks, the last ragged
    inp = forward_inputs(B, T, H, d, d, "f32", seed=3, s0_std=0.5)
    rng = np.random.default_rng(5)
    dO = rng.standard_normal((B, T, H, d))
    dSf = rng.standard_normal((B, H, d, d))
    arr = {n: as_f32_numpy(inp[n]).astype(np.float64) for n in ("q", "k", "v", "log_alpha", "beta", "S0")}
    ref = oracle.backward(*[as_f32_numpy(inp[n]) for n in ("q", "k", "v", "log_alpha", "beta")], arr["S0"], dO, dSf,
                          nthreads=2)
    got = decomposed_backward(arr["q"][0, :, 0], arr["k"][0, :, 0], arr["v"][0, :, 0], arr["log_alpha"][0, :, 0],
                              arr["beta"][0, :, 0], arr["S0"][0, 0], dO[0, :, 0], dSf[0, 0])
    for name, a, r in zip(("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"), got, ref):
        r = np.asarray(r)
        r = r[0, 0] if name == "dS0" else r.reshape(a.shape)
        assert np.abs(a - r).max() <= 1e-12 * max(1.0, np.abs(r).max()), name
