"""Planted mistakes in the oracle must be caught by its pins (CPU only).

Each case copies the committed oracle source into a temporary folder, plants
one plausible mistake (a flipped sign, a dropped factor, a wrong operand or
index, a wrong mask), compiles the copy with gcc and runs every pin of
``test_oracle.py`` against it.  The case passes when at least one pin fails.
The committed oracle itself is never modified.
"""
import os

import pytest

import oracle as oracle_pkg
from test_oracle import PINS
from test_oracle_backward import BWD_PINS
from test_oracle_grouped import GROUPED_PINS
from test_oracle_input_stage import RAW_PINS


def _swap_output_before_update(src: str) -> str:
    """o_t = S_{t-1} q_t instead of S_t q_t: move the output loop ahead of the update."""
    out_loop = (
        "    for (int64_t r = 0; r < dv; ++r) {          /* o_t = S_t q_t */\n"
        "        double acc = 0.0;\n"
        "        for (int64_t c = 0; c < dk; ++c) acc += S[r * dk + c] * (double)q[c];\n"
        "        o[r] = acc;\n"
        "    }\n")
    assert src.count(out_loop) == 1
    src = src.replace(out_loop, "")
    anchor = "    for (int64_t r = 0; r < dv; ++r) {\n        for (int64_t c = 0; c < dk; ++c) {\n            /* alpha"
    assert src.count(anchor) == 1
    return src.replace(anchor, out_loop + anchor)


MUTANTS = {
    "delta_sign": ("const double sk = S[r * dk + c] - bt * x[r] * (double)k[c];",
                   "const double sk = S[r * dk + c] + bt * x[r] * (double)k[c];"),
    "decay_on_write": ("S[r * dk + c] = a * sk + bt * (double)v[r] * (double)k[c];",
                       "S[r * dk + c] = a * (sk + bt * (double)v[r] * (double)k[c]);"),
    "write_without_beta": ("S[r * dk + c] = a * sk + bt * (double)v[r] * (double)k[c];",
                           "S[r * dk + c] = a * sk + (double)v[r] * (double)k[c];"),
    "prediction_uses_q": ("for (int64_t c = 0; c < dk; ++c) acc += S[r * dk + c] * (double)k[c];",
                          "for (int64_t c = 0; c < dk; ++c) acc += S[r * dk + c] * (double)q[c];"),
    "output_uses_k": ("for (int64_t c = 0; c < dk; ++c) acc += S[r * dk + c] * (double)q[c];\n        o[r]",
                      "for (int64_t c = 0; c < dk; ++c) acc += S[r * dk + c] * (double)k[c];\n        o[r]"),
    "gate_not_exponentiated": ("const double a = exp((double)log_alpha);",
                               "const double a = 1.0 + (double)log_alpha;"),
    "output_before_update": _swap_output_before_update,
    "chunk_A_beta_index": ("a = beta[t] * decay[t * n + s] * kk;", "a = beta[s] * decay[t * n + s] * kk;"),
    "chunk_output_drops_diagonal": ("for (int64_t s = 0; s <= t; ++s) {\n                    double qk",
                                    "for (int64_t s = 0; s < t; ++s) {\n                    double qk"),
    "chunk_state_not_decayed": ("Snew[r * dk + c] = gamma[n - 1] * S[r * dk + c] + acc;",
                                "Snew[r * dk + c] = S[r * dk + c] + acc;"),
    "chunk_U_sign": ("U[t * dv + r] = Ut[t * dv + r] - acc;", "U[t * dv + r] = Ut[t * dv + r] + acc;"),
    "chunk_W_without_gamma": ("acc += Tinv[t * n + s] * beta[s] * gamma[s] * K[s * dk + c];",
                              "acc += Tinv[t * n + s] * beta[s] * K[s * dk + c];"),
    "chunk_inverse_sign": ("x -= A[t * n + s] * Tinv[s * n + j];", "x += A[t * n + s] * Tinv[s * n + j];"),
    "chunk_inter_without_gamma": ("o[t * dv + r] = gamma[t] * inter + intra;", "o[t * dv + r] = inter + intra;"),
    "dense_factor_sign": ("a * (((i == j) ? 1.0 : 0.0) - bt *", "a * (((i == j) ? 1.0 : 0.0) + bt *"),
    "norm_without_sqrt": ("const double inv = 1.0 / sqrt(ss + GDN_ORACLE_NORM_EPS);",
                          "const double inv = 1.0 / (ss + GDN_ORACLE_NORM_EPS);"),
    "norm_without_eps": ("const double inv = 1.0 / sqrt(ss + GDN_ORACLE_NORM_EPS);",
                         "const double inv = 1.0 / sqrt(ss);"),
    "softplus_sign": ("return -log1p(exp(x));", "return -log1p(exp(-x));"),
    "softplus_drops_one": ("return -log1p(exp(x));", "return -log(exp(x));"),
    "sigmoid_sign": ("return 1.0 / (1.0 + exp(-x));", "return 1.0 / (1.0 + exp(x));"),
    "raw_gate_not_exponentiated": ("exp(neg_softplus((double)x_alpha[gi]))", "(1.0 + neg_softplus((double)x_alpha[gi]))"),
    "raw_prediction_uses_q": ("for (int64_t c = 0; c < dk; ++c) acc += S[r * dk + c] * k[c];",
                              "for (int64_t c = 0; c < dk; ++c) acc += S[r * dk + c] * q[c];"),
    "raw_write_without_beta": ("S[r * dk + c] = a * sk + bt * (double)v[r] * k[c];",
                               "S[r * dk + c] = a * sk + (double)v[r] * k[c];"),
    "bwd_dk_sign": ("dkt[c] = -a * bt * (sgk + gx) + bt * gv;", "dkt[c] = a * bt * (sgk + gx) + bt * gv;"),
    "bwd_dk_drops_transpose_term": ("dkt[c] = -a * bt * (sgk + gx) + bt * gv;", "dkt[c] = -a * bt * sgk + bt * gv;"),
    "bwd_adjoint_without_alpha": ("G[r * dk + c] = a * (G[r * dk + c] - bt * Gk[r] * (double)kt[c]);",
                                  "G[r * dk + c] = (G[r * dk + c] - bt * Gk[r] * (double)kt[c]);"),
    "bwd_dbeta_sign": ("dbeta[gi] = vgk - a * xgk;", "dbeta[gi] = vgk + a * xgk;"),
    "bwd_dlogalpha_without_alpha": ("dlog_alpha[gi] = a * (gs - bt * xgk);", "dlog_alpha[gi] = (gs - bt * xgk);"),
    "bwd_dq_uses_previous_state": ("for (int64_t r = 0; r < dv; ++r) acc += Sn[r * dk + c] * dot[r];",
                                   "for (int64_t r = 0; r < dv; ++r) acc += Sp[r * dk + c] * dot[r];"),
    "bwd_output_grad_uses_k": ("G[r * dk + c] += dot[r] * (double)qt[c];", "G[r * dk + c] += dot[r] * (double)kt[c];"),
    "grouped_wrong_kv_head": ("k + IDX_TOK(b, t, hk, 0, T, Hkv, dk),\n                            v + IDX_TOK(b, t, hk, 0, T, Hkv, dv)",
                              "k + IDX_TOK(b, t, (hk + 1) % Hkv, 0, T, Hkv, dk),\n                            v + IDX_TOK(b, t, hk, 0, T, Hkv, dv)"),
    "grouped_reads_first_query_only": ("const float *qh = q + IDX_TOK(b, t, hk * G + g, 0, T, Hq, dk);",
                                       "const float *qh = q + IDX_TOK(b, t, hk * G, 0, T, Hq, dk);"),
    "bwdc_dR_without_transpose": ("for (int64_t t = s2; t < n; ++t) a += Tm[t * C + s2] * dU[t * dv + j];",
                                  "for (int64_t t = s2; t < n; ++t) a += Tm[s2 * C + t] * dU[t * dv + j];"),
    "bwdc_dl_gradient_sign": ("dg[s2] -= w;\n                dgl += w;", "dg[s2] += w;\n                dgl += w;"),
    "bwdc_F_without_beta": ("F[t * C + s2] = (s2 < t) ? da * bet[t] * E[t * C + s2] : 0.0;",
                            "F[t * C + s2] = (s2 < t) ? da * E[t * C + s2] : 0.0;"),
    "raw_decode_swaps_q_k": ("unit_row(q + bh * dk, qk, dk);\n        unit_row(k + bh * dk, qk + dk, dk);",
                             "unit_row(k + bh * dk, qk, dk);\n        unit_row(q + bh * dk, qk + dk, dk);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, name):
    src = open(oracle_pkg.SOURCE).read()
    m = MUTANTS[name]
    if callable(m):
        bad = m(src)
    else:
        old, new = m
        assert src.count(old) == 1, "mutation anchor not unique / missing: %s" % name
        bad = src.replace(old, new)
    assert bad != src
    c_path = os.path.join(str(tmp_path), "mutant.c")
    with open(c_path, "w") as f:
        f.write(bad)
    lib = oracle_pkg.build(src=c_path, out=os.path.join(str(tmp_path), "libmutant.so"), force=True)
    mutant = oracle_pkg.Oracle(lib)
    caught = []
    for pin in PINS + RAW_PINS + BWD_PINS + GROUPED_PINS:
        try:
            pin(mutant)
        except (AssertionError, RuntimeError, FloatingPointError, ValueError):
            caught.append(pin.__name__)
    assert caught, "no pin catches mutant %s" % name
