/*
 * gdn_oracle.c -- float64 CPU oracle for the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes
 * or calls this file; only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark load it (through oracle/__init__.py).  It
 * shares no source with the CUDA path.
 *
 * What it computes (source: "ATMA: Long-Context Language Modeling via Polar
 * Attention and Gated-Delta Compression Memory", Sec. 3.3, the gated-delta
 * memory equation), per (batch b, head h), with the paper's symbols renamed
 * gamma_t -> alpha_t, M -> S, r -> o:
 *
 *     S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = S_t q_t
 *
 * S is d_v x d_k (row index over the value dimension, column index over the
 * key dimension), held in double.  alpha_t = exp(log_alpha_t).
 *
 * Layouts (row-major, 64-bit indexing):
 *   q, k        [B, T, H, dk]      float (exact values of the caller's inputs)
 *   v, out      [B, T, H, dv]      float in, double out
 *   log_alpha,
 *   beta        [B, T, H]          float
 *   S0, S_final [B, H, dv, dk]     double; S0 may be NULL (zero state),
 *                                  S_final may be NULL (not written)
 *
 * Inputs are taken as float because every input the library accepts (fp32
 * or bf16) converts to float exactly; all arithmetic is double.
 *
 * Functions:
 *   gdn_oracle_forward          the token-by-token recurrence (the definition)
 *   gdn_oracle_decode_step      one token for every (b, h), state in place
 *   gdn_oracle_forward_chunked  the chunkwise (WY / UT-transform) form of the
 *                               same recurrence, any chunk length C >= 1; the
 *                               algebra is the one of the works the paper cites
 *                               for the memory ("Gated delta networks",
 *                               "Parallelizing linear transformers with the
 *                               delta rule over sequence length"), re-derived
 *                               from the Sec. 3.3 equation
 *   gdn_oracle_segment_transfer the affine map S_end = S_start M + Bseg of a
 *                               run of tokens, built chunk by chunk
 *   gdn_oracle_dense_product    brute force: explicit d_k x d_k factors
 *                               alpha_t (I - beta_t k_t k_t^T), tiny T only
 *   gdn_oracle_input_stage      unit-norm q, k and the gate maps from logits
 *   gdn_oracle_forward_raw,     the input stage followed by the recurrence
 *   gdn_oracle_decode_step_raw
 *   gdn_oracle_backward         reverse mode of the recurrence, token by token
 *   gdn_oracle_forward_grouped  grouped heads: query heads reading the memory of
 *                               their key-value head
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define IDX_TOK(b, t, h, d, T, H, D) ((((int64_t)(b) * (T) + (t)) * (H) + (h)) * (D) + (d))
#define IDX_GATE(b, t, h, T, H) (((int64_t)(b) * (T) + (t)) * (H) + (h))
#define IDX_STATE(b, h, H, dv, dk) (((int64_t)(b) * (H) + (h)) * (dv) * (dk))

static void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

/* One token of the Sec. 3.3 recurrence on a single state S (dv x dk).
 * S (I - beta k k^T) is evaluated as S - beta (S k) k^T, which is the same
 * matrix (associativity), so the step costs O(dv dk) instead of O(dv dk^2). */
static void recurrence_step(double *S, const float *q, const float *k, const float *v,
                            float log_alpha, float beta, double *o, double *x,
                            int64_t dk, int64_t dv) {
    const double a = exp((double)log_alpha);
    const double bt = (double)beta;
    for (int64_t r = 0; r < dv; ++r) {          /* x = S_{t-1} k_t */
        double acc = 0.0;
        for (int64_t c = 0; c < dk; ++c) acc += S[r * dk + c] * (double)k[c];
        x[r] = acc;
    }
    for (int64_t r = 0; r < dv; ++r) {
        for (int64_t c = 0; c < dk; ++c) {
            /* alpha * [S (I - beta k k^T)]_{rc} + beta v_r k_c */
            const double sk = S[r * dk + c] - bt * x[r] * (double)k[c];
            S[r * dk + c] = a * sk + bt * (double)v[r] * (double)k[c];
        }
    }
    for (int64_t r = 0; r < dv; ++r) {          /* o_t = S_t q_t */
        double acc = 0.0;
        for (int64_t c = 0; c < dk; ++c) acc += S[r * dk + c] * (double)q[c];
        o[r] = acc;
    }
}

int gdn_oracle_forward(const float *q, const float *k, const float *v,
                       const float *log_alpha, const float *beta, const double *S0,
                       double *out, double *S_final, int64_t B, int64_t T, int64_t H,
                       int64_t dk, int64_t dv, int nthreads) {
    if (B < 0 || T < 0 || H < 0 || dk < 1 || dv < 1) return 1;
    set_threads(nthreads);
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        const int64_t b = bh / H, h = bh % H;
        double *S = (double *)malloc(sizeof(double) * dv * dk);
        double *x = (double *)malloc(sizeof(double) * dv);
        double *o = (double *)malloc(sizeof(double) * dv);
        if (!S || !x || !o) {
            free(S); free(x); free(o);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        if (S0) memcpy(S, S0 + IDX_STATE(b, h, H, dv, dk), sizeof(double) * dv * dk);
        else memset(S, 0, sizeof(double) * dv * dk);
        for (int64_t t = 0; t < T; ++t) {
            recurrence_step(S, q + IDX_TOK(b, t, h, 0, T, H, dk), k + IDX_TOK(b, t, h, 0, T, H, dk),
                            v + IDX_TOK(b, t, h, 0, T, H, dv), log_alpha[IDX_GATE(b, t, h, T, H)],
                            beta[IDX_GATE(b, t, h, T, H)], o, x, dk, dv);
            if (out) memcpy(out + IDX_TOK(b, t, h, 0, T, H, dv), o, sizeof(double) * dv);
        }
        if (S_final) memcpy(S_final + IDX_STATE(b, h, H, dv, dk), S, sizeof(double) * dv * dk);
        free(S); free(x); free(o);
    }
    return failed ? 2 : 0;
}

/* Decode: one token per (b, h).  q, k [B, H, dk]; v, out [B, H, dv];
 * gates [B, H]; S [B, H, dv, dk] updated in place. */
int gdn_oracle_decode_step(const float *q, const float *k, const float *v,
                           const float *log_alpha, const float *beta, double *S,
                           double *out, int64_t B, int64_t H, int64_t dk, int64_t dv,
                           int nthreads) {
    if (B < 0 || H < 0 || dk < 1 || dv < 1) return 1;
    set_threads(nthreads);
    int failed = 0;
#pragma omp parallel for schedule(static)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        double *x = (double *)malloc(sizeof(double) * dv);
        if (!x) {
#pragma omp atomic write
            failed = 1;
            continue;
        }
        recurrence_step(S + bh * dv * dk, q + bh * dk, k + bh * dk, v + bh * dv, log_alpha[bh],
                        beta[bh], out + bh * dv, x, dk, dv);
        free(x);
    }
    return failed ? 2 : 0;
}

/* ------------------------------------------------------------------------
 * Chunkwise form.  Within a chunk of n <= C tokens with entry state S0, write
 * the Sec. 3.3 step as S_t = alpha_t S_{t-1} + u_t k_t^T with
 * u_t = beta_t (v_t - alpha_t S_{t-1} k_t).  Unrolling,
 *     S_t = gamma_t S0 + sum_{s<=t} (gamma_t / gamma_s) u_s k_s^T,
 * gamma_t = prod_{r<=t} alpha_r (chunk-local).  Putting that back into u_t
 * gives the unit-lower-triangular system
 *     (I + A) U = diag(beta) V - diag(beta*gamma) K S0^T,
 *     A_ts = beta_t (gamma_t/gamma_s) (k_t . k_s)   for s < t, else 0,
 * so with Tinv = (I + A)^{-1} (forward substitution):
 *     W  = Tinv diag(beta*gamma) K,   Ut = Tinv diag(beta) V,   U = Ut - W S0^T
 *     O  = diag(gamma) Q S0^T + [ (Q K^T) o (gamma_t/gamma_s) ]_{s<=t} U
 *     S_n = gamma_n S0 + U^T Ktil,   Ktil_s = (gamma_n/gamma_s) k_s.
 * Ratios gamma_t/gamma_s (s <= t) are formed as products of the alphas in
 * (s, t], so an alpha of exactly 0 stays exact and nothing overflows.
 * ---------------------------------------------------------------------- */

/* decay[t][s] = prod_{r=s+1..t} alpha_r for s <= t (1 on the diagonal), 0 above. */
static void chunk_decays(const double *alpha, int64_t n, double *decay) {
    for (int64_t t = 0; t < n; ++t) {
        for (int64_t s = 0; s < n; ++s) {
            if (s > t) { decay[t * n + s] = 0.0; continue; }
            double p = 1.0;
            for (int64_t r = s + 1; r <= t; ++r) p *= alpha[r];
            decay[t * n + s] = p;
        }
    }
}

/* One chunk: consumes entry state S (dv x dk), writes o (n x dv, may be NULL)
 * and replaces S by the exit state.  Token rows are gathered into dense
 * n x d matrices by the caller. */
static void chunk_step(double *S, const double *Q, const double *K, const double *V,
                       const double *alpha, const double *beta, int64_t n, int64_t dk,
                       int64_t dv, double *o, double *work) {
    double *decay = work;                  /* n*n   */
    double *gamma = decay + n * n;         /* n     */
    double *A = gamma + n;                 /* n*n   */
    double *Tinv = A + n * n;              /* n*n   */
    double *Wm = Tinv + n * n;             /* n*dk  */
    double *Ut = Wm + n * dk;              /* n*dv  */
    double *U = Ut + n * dv;               /* n*dv  */
    double *Snew = U + n * dv;             /* dv*dk */

    chunk_decays(alpha, n, decay);
    for (int64_t t = 0; t < n; ++t) gamma[t] = decay[t * n + 0] * alpha[0];

    /* A_ts = beta_t (gamma_t/gamma_s) (k_t . k_s), strictly lower */
    for (int64_t t = 0; t < n; ++t)
        for (int64_t s = 0; s < n; ++s) {
            double a = 0.0;
            if (s < t) {
                double kk = 0.0;
                for (int64_t c = 0; c < dk; ++c) kk += K[t * dk + c] * K[s * dk + c];
                a = beta[t] * decay[t * n + s] * kk;
            }
            A[t * n + s] = a;
        }
    /* Tinv = (I + A)^{-1}: solve (I + A) X = I column by column, top to bottom */
    for (int64_t j = 0; j < n; ++j)
        for (int64_t t = 0; t < n; ++t) {
            double x = (t == j) ? 1.0 : 0.0;
            for (int64_t s = 0; s < t; ++s) x -= A[t * n + s] * Tinv[s * n + j];
            Tinv[t * n + j] = x;
        }
    /* W = Tinv diag(beta*gamma) K ;  Ut = Tinv diag(beta) V */
    for (int64_t t = 0; t < n; ++t) {
        for (int64_t c = 0; c < dk; ++c) {
            double acc = 0.0;
            for (int64_t s = 0; s < n; ++s) acc += Tinv[t * n + s] * beta[s] * gamma[s] * K[s * dk + c];
            Wm[t * dk + c] = acc;
        }
        for (int64_t r = 0; r < dv; ++r) {
            double acc = 0.0;
            for (int64_t s = 0; s < n; ++s) acc += Tinv[t * n + s] * beta[s] * V[s * dv + r];
            Ut[t * dv + r] = acc;
        }
    }
    /* U = Ut - W S0^T */
    for (int64_t t = 0; t < n; ++t)
        for (int64_t r = 0; r < dv; ++r) {
            double acc = 0.0;
            for (int64_t c = 0; c < dk; ++c) acc += Wm[t * dk + c] * S[r * dk + c];
            U[t * dv + r] = Ut[t * dv + r] - acc;
        }
    /* O = diag(gamma) Q S0^T + [(Q K^T) o decay]_{s<=t} U */
    if (o) {
        for (int64_t t = 0; t < n; ++t)
            for (int64_t r = 0; r < dv; ++r) {
                double inter = 0.0;
                for (int64_t c = 0; c < dk; ++c) inter += Q[t * dk + c] * S[r * dk + c];
                double intra = 0.0;
                for (int64_t s = 0; s <= t; ++s) {
                    double qk = 0.0;
                    for (int64_t c = 0; c < dk; ++c) qk += Q[t * dk + c] * K[s * dk + c];
                    intra += qk * decay[t * n + s] * U[s * dv + r];
                }
                o[t * dv + r] = gamma[t] * inter + intra;
            }
    }
    /* S_n = gamma_n S0 + U^T Ktil */
    for (int64_t r = 0; r < dv; ++r)
        for (int64_t c = 0; c < dk; ++c) {
            double acc = 0.0;
            for (int64_t s = 0; s < n; ++s) acc += U[s * dv + r] * decay[(n - 1) * n + s] * K[s * dk + c];
            Snew[r * dk + c] = gamma[n - 1] * S[r * dk + c] + acc;
        }
    memcpy(S, Snew, sizeof(double) * dv * dk);
}

static size_t chunk_work_doubles(int64_t C, int64_t dk, int64_t dv) {
    return (size_t)(3 * C * C + C + C * dk + 2 * C * dv + dv * dk);
}

/* Gather n token rows of one (b, h) into dense double matrices. */
static void gather_chunk(const float *q, const float *k, const float *v, const float *log_alpha,
                         const float *beta, int64_t b, int64_t h, int64_t t0, int64_t n,
                         int64_t T, int64_t H, int64_t dk, int64_t dv, double *Q, double *K,
                         double *V, double *al, double *be) {
    for (int64_t i = 0; i < n; ++i) {
        const int64_t t = t0 + i;
        for (int64_t c = 0; c < dk; ++c) {
            if (Q) Q[i * dk + c] = (double)q[IDX_TOK(b, t, h, c, T, H, dk)];
            K[i * dk + c] = (double)k[IDX_TOK(b, t, h, c, T, H, dk)];
        }
        for (int64_t r = 0; r < dv; ++r) V[i * dv + r] = (double)v[IDX_TOK(b, t, h, r, T, H, dv)];
        al[i] = exp((double)log_alpha[IDX_GATE(b, t, h, T, H)]);
        be[i] = (double)beta[IDX_GATE(b, t, h, T, H)];
    }
}

int gdn_oracle_forward_chunked(const float *q, const float *k, const float *v,
                               const float *log_alpha, const float *beta, const double *S0,
                               double *out, double *S_final, int64_t B, int64_t T, int64_t H,
                               int64_t dk, int64_t dv, int64_t C, int nthreads) {
    if (B < 0 || T < 0 || H < 0 || dk < 1 || dv < 1 || C < 1) return 1;
    set_threads(nthreads);
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        const int64_t b = bh / H, h = bh % H;
        double *S = (double *)malloc(sizeof(double) * dv * dk);
        double *Q = (double *)malloc(sizeof(double) * C * dk);
        double *K = (double *)malloc(sizeof(double) * C * dk);
        double *V = (double *)malloc(sizeof(double) * C * dv);
        double *al = (double *)malloc(sizeof(double) * C);
        double *be = (double *)malloc(sizeof(double) * C);
        double *o = (double *)malloc(sizeof(double) * C * dv);
        double *work = (double *)malloc(sizeof(double) * chunk_work_doubles(C, dk, dv));
        if (!S || !Q || !K || !V || !al || !be || !o || !work) {
#pragma omp atomic write
            failed = 1;
        } else {
            if (S0) memcpy(S, S0 + IDX_STATE(b, h, H, dv, dk), sizeof(double) * dv * dk);
            else memset(S, 0, sizeof(double) * dv * dk);
            for (int64_t t0 = 0; t0 < T; t0 += C) {
                const int64_t n = (T - t0 < C) ? (T - t0) : C;
                gather_chunk(q, k, v, log_alpha, beta, b, h, t0, n, T, H, dk, dv, Q, K, V, al, be);
                chunk_step(S, Q, K, V, al, be, n, dk, dv, o, work);
                if (out)
                    for (int64_t i = 0; i < n; ++i)
                        memcpy(out + IDX_TOK(b, t0 + i, h, 0, T, H, dv), o + i * dv, sizeof(double) * dv);
            }
            if (S_final) memcpy(S_final + IDX_STATE(b, h, H, dv, dk), S, sizeof(double) * dv * dk);
        }
        free(S); free(Q); free(K); free(V); free(al); free(be); free(o); free(work);
    }
    return failed ? 2 : 0;
}

/* ------------------------------------------------------------------------
 * Segment transfer.  Each chunk maps its entry state affinely:
 *     S_n = S0 (gamma_n I - W^T Ktil) + Ut^T Ktil = S0 Mc + Bc,
 * so a run of chunks maps S_start -> S_start Mseg + Bseg with
 *     Mseg <- Mseg Mc,  Bseg <- Bseg Mc + Bc   (chunk by chunk).
 * Mseg is dk x dk, Bseg is dv x dk.  Single (b, h): inputs are [T, d].
 * ---------------------------------------------------------------------- */
int gdn_oracle_segment_transfer(const float *k, const float *v, const float *log_alpha,
                                const float *beta, double *Mseg, double *Bseg, int64_t T,
                                int64_t dk, int64_t dv, int64_t C) {
    if (T < 0 || dk < 1 || dv < 1 || C < 1) return 1;
    double *K = (double *)malloc(sizeof(double) * C * dk);
    double *V = (double *)malloc(sizeof(double) * C * dv);
    double *al = (double *)malloc(sizeof(double) * C);
    double *be = (double *)malloc(sizeof(double) * C);
    /* the d_k transfer rows run through chunk_step as a state with d_k rows */
    double *work = (double *)malloc(sizeof(double) * chunk_work_doubles(C, dk, dv > dk ? dv : dk));
    double *Mc = (double *)malloc(sizeof(double) * dk * dk);
    double *Bc = (double *)malloc(sizeof(double) * dv * dk);
    double *tmpM = (double *)malloc(sizeof(double) * dk * dk);
    double *tmpB = (double *)malloc(sizeof(double) * dv * dk);
    int rc = 0;
    if (!K || !V || !al || !be || !work || !Mc || !Bc || !tmpM || !tmpB) { rc = 2; goto done; }
    for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < dk; ++j) Mseg[i * dk + j] = (i == j) ? 1.0 : 0.0;
    memset(Bseg, 0, sizeof(double) * dv * dk);
    for (int64_t t0 = 0; t0 < T; t0 += C) {
        const int64_t n = (T - t0 < C) ? (T - t0) : C;
        gather_chunk(NULL, k, v, log_alpha, beta, 0, 0, t0, n, T, 1, dk, dv, NULL, K, V, al, be);
        /* Bc = chunk applied to the zero state; Mc row i = chunk applied to e_i^T
         * with v = 0 (rows of the state evolve independently). */
        memset(Bc, 0, sizeof(double) * dv * dk);
        chunk_step(Bc, NULL, K, V, al, be, n, dk, dv, NULL, work);
        double *Vz = (double *)calloc((size_t)(n * dk), sizeof(double));
        if (!Vz) { rc = 2; goto done; }
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dk; ++j) Mc[i * dk + j] = (i == j) ? 1.0 : 0.0;
        chunk_step(Mc, NULL, K, Vz, al, be, n, dk, dk, NULL, work);
        free(Vz);
        /* compose */
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dk; ++j) {
                double acc = 0.0;
                for (int64_t l = 0; l < dk; ++l) acc += Mseg[i * dk + l] * Mc[l * dk + j];
                tmpM[i * dk + j] = acc;
            }
        for (int64_t r = 0; r < dv; ++r)
            for (int64_t j = 0; j < dk; ++j) {
                double acc = Bc[r * dk + j];
                for (int64_t l = 0; l < dk; ++l) acc += Bseg[r * dk + l] * Mc[l * dk + j];
                tmpB[r * dk + j] = acc;
            }
        memcpy(Mseg, tmpM, sizeof(double) * dk * dk);
        memcpy(Bseg, tmpB, sizeof(double) * dv * dk);
    }
done:
    free(K); free(V); free(al); free(be); free(work); free(Mc); free(Bc); free(tmpM); free(tmpB);
    return rc;
}

/* ------------------------------------------------------------------------
 * Brute force for tiny T, single (b, h), inputs [T, d]: with the explicit
 * d_k x d_k factors F_t = alpha_t (I - beta_t k_t k_t^T),
 *     S_t = S0 F_1 ... F_t + sum_{s<=t} beta_s v_s k_s^T F_{s+1} ... F_t,
 * every product formed from scratch for every t (no reuse between t).
 * ---------------------------------------------------------------------- */
int gdn_oracle_dense_product(const float *q, const float *k, const float *v,
                             const float *log_alpha, const float *beta, const double *S0,
                             double *out, double *S_final, int64_t T, int64_t dk, int64_t dv) {
    if (T < 0 || T > 16 || dk < 1 || dv < 1 || dk > 64 || dv > 64) return 1;
    double *F = (double *)malloc(sizeof(double) * (T > 0 ? T : 1) * dk * dk);
    double *P = (double *)malloc(sizeof(double) * dk * dk);
    double *tmp = (double *)malloc(sizeof(double) * dk * dk);
    double *St = (double *)malloc(sizeof(double) * dv * dk);
    if (!F || !P || !tmp || !St) { free(F); free(P); free(tmp); free(St); return 2; }
    for (int64_t t = 0; t < T; ++t) {
        const double a = exp((double)log_alpha[t]), bt = (double)beta[t];
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dk; ++j)
                F[t * dk * dk + i * dk + j] =
                    a * (((i == j) ? 1.0 : 0.0) - bt * (double)k[t * dk + i] * (double)k[t * dk + j]);
    }
    for (int64_t t = 0; t < T; ++t) {
        memset(St, 0, sizeof(double) * dv * dk);
        /* term j = -1 is S0 F_0..F_t ; term j >= 0 is beta_j v_j k_j^T F_{j+1}..F_t */
        for (int64_t j = -1; j <= t; ++j) {
            for (int64_t i = 0; i < dk; ++i)
                for (int64_t l = 0; l < dk; ++l) P[i * dk + l] = (i == l) ? 1.0 : 0.0;
            for (int64_t m = j + 1; m <= t; ++m) {
                for (int64_t i = 0; i < dk; ++i)
                    for (int64_t l = 0; l < dk; ++l) {
                        double acc = 0.0;
                        for (int64_t x = 0; x < dk; ++x) acc += P[i * dk + x] * F[m * dk * dk + x * dk + l];
                        tmp[i * dk + l] = acc;
                    }
                memcpy(P, tmp, sizeof(double) * dk * dk);
            }
            for (int64_t r = 0; r < dv; ++r)
                for (int64_t l = 0; l < dk; ++l) {
                    double acc = 0.0;
                    if (j < 0) {
                        if (S0)
                            for (int64_t x = 0; x < dk; ++x) acc += S0[r * dk + x] * P[x * dk + l];
                    } else {
                        const double bv = (double)beta[j] * (double)v[j * dv + r];
                        for (int64_t x = 0; x < dk; ++x) acc += bv * (double)k[j * dk + x] * P[x * dk + l];
                    }
                    St[r * dk + l] += acc;
                }
        }
        if (out)
            for (int64_t r = 0; r < dv; ++r) {
                double acc = 0.0;
                for (int64_t c = 0; c < dk; ++c) acc += St[r * dk + c] * (double)q[t * dk + c];
                out[t * dv + r] = acc;
            }
    }
    if (S_final) {
        if (T == 0) {
            if (S0) memcpy(S_final, S0, sizeof(double) * dv * dk);
            else memset(S_final, 0, sizeof(double) * dv * dk);
        } else {
            memcpy(S_final, St, sizeof(double) * dv * dk);
        }
    }
    free(F); free(P); free(tmp); free(St);
    return 0;
}

/* ------------------------------------------------------------------------
 * The input stage.  The memory of Sec. 3.3 reads unit-norm queries and keys
 * (App. A.2 takes ||q_t|| = ||k_t|| = 1), a decay alpha_t in (0, 1) and a write
 * strength beta_t in (0, 1).  From raw projections q, k and gate logits
 * x_alpha, x_beta this stage forms, in double,
 *     q_t / sqrt(|q_t|^2 + eps),  k_t / sqrt(|k_t|^2 + eps)   (eps = 1e-12)
 *     log alpha_t = -softplus(x_alpha) = -log(1 + exp(x_alpha))
 *     beta_t      = sigmoid(x_beta)    = 1 / (1 + exp(-x_beta))
 * The eps only keeps a zero vector at zero.  The *_raw functions run this
 * stage and then the same recurrence as gdn_oracle_forward / _decode_step,
 * on the double results (nothing is rounded back to float).
 */
#define GDN_ORACLE_NORM_EPS 1e-12

static void unit_row(const float *x, double *y, int64_t d) {
    double ss = 0.0;
    for (int64_t i = 0; i < d; ++i) ss += (double)x[i] * (double)x[i];
    const double inv = 1.0 / sqrt(ss + GDN_ORACLE_NORM_EPS);
    for (int64_t i = 0; i < d; ++i) y[i] = (double)x[i] * inv;
}

static double neg_softplus(double x) { return -log1p(exp(x)); }
static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* Input stage alone over `rows` (token, head) rows of d elements. */
int gdn_oracle_input_stage(const float *q, const float *k, const float *x_alpha, const float *x_beta,
                           double *qn, double *kn, double *log_alpha, double *beta, int64_t rows,
                           int64_t d) {
    if (rows < 0 || d < 1) return 1;
    for (int64_t r = 0; r < rows; ++r) {
        unit_row(q + r * d, qn + r * d, d);
        unit_row(k + r * d, kn + r * d, d);
        log_alpha[r] = neg_softplus((double)x_alpha[r]);
        beta[r] = sigmoid((double)x_beta[r]);
    }
    return 0;
}

/* One token of the Sec. 3.3 recurrence with double q, k and gates (the
 * counterpart of recurrence_step above for the input stage's outputs). */
static void recurrence_step_d(double *S, const double *q, const double *k, const float *v, double a,
                              double bt, double *o, double *x, int64_t dk, int64_t dv) {
    for (int64_t r = 0; r < dv; ++r) {
        double acc = 0.0;
        for (int64_t c = 0; c < dk; ++c) acc += S[r * dk + c] * k[c];
        x[r] = acc;
    }
    for (int64_t r = 0; r < dv; ++r)
        for (int64_t c = 0; c < dk; ++c) {
            const double sk = S[r * dk + c] - bt * x[r] * k[c];
            S[r * dk + c] = a * sk + bt * (double)v[r] * k[c];
        }
    for (int64_t r = 0; r < dv; ++r) {
        double acc = 0.0;
        for (int64_t c = 0; c < dk; ++c) acc += S[r * dk + c] * q[c];
        o[r] = acc;
    }
}

/* gdn_oracle_forward with the input stage first: q, k raw, x_alpha, x_beta the
 * gate logits (layouts as gdn_oracle_forward). */
int gdn_oracle_forward_raw(const float *q, const float *k, const float *v, const float *x_alpha,
                           const float *x_beta, const double *S0, double *out, double *S_final,
                           int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv, int nthreads) {
    if (B < 0 || T < 0 || H < 0 || dk < 1 || dv < 1) return 1;
    set_threads(nthreads);
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        const int64_t b = bh / H, h = bh % H;
        double *S = (double *)malloc(sizeof(double) * dv * dk);
        double *x = (double *)malloc(sizeof(double) * dv);
        double *o = (double *)malloc(sizeof(double) * dv);
        double *qk = (double *)malloc(sizeof(double) * 2 * dk);
        if (!S || !x || !o || !qk) {
            free(S); free(x); free(o); free(qk);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        if (S0) memcpy(S, S0 + IDX_STATE(b, h, H, dv, dk), sizeof(double) * dv * dk);
        else memset(S, 0, sizeof(double) * dv * dk);
        for (int64_t t = 0; t < T; ++t) {
            const int64_t gi = IDX_GATE(b, t, h, T, H);
            unit_row(q + IDX_TOK(b, t, h, 0, T, H, dk), qk, dk);
            unit_row(k + IDX_TOK(b, t, h, 0, T, H, dk), qk + dk, dk);
            recurrence_step_d(S, qk, qk + dk, v + IDX_TOK(b, t, h, 0, T, H, dv),
                              exp(neg_softplus((double)x_alpha[gi])), sigmoid((double)x_beta[gi]), o, x, dk,
                              dv);
            if (out) memcpy(out + IDX_TOK(b, t, h, 0, T, H, dv), o, sizeof(double) * dv);
        }
        if (S_final) memcpy(S_final + IDX_STATE(b, h, H, dv, dk), S, sizeof(double) * dv * dk);
        free(S); free(x); free(o); free(qk);
    }
    return failed ? 2 : 0;
}

/* gdn_oracle_decode_step with the input stage first. */
int gdn_oracle_decode_step_raw(const float *q, const float *k, const float *v, const float *x_alpha,
                               const float *x_beta, double *S, double *out, int64_t B, int64_t H,
                               int64_t dk, int64_t dv, int nthreads) {
    if (B < 0 || H < 0 || dk < 1 || dv < 1) return 1;
    set_threads(nthreads);
    int failed = 0;
#pragma omp parallel for schedule(static)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        double *x = (double *)malloc(sizeof(double) * dv);
        double *qk = (double *)malloc(sizeof(double) * 2 * dk);
        if (!x || !qk) {
            free(x); free(qk);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        unit_row(q + bh * dk, qk, dk);
        unit_row(k + bh * dk, qk + dk, dk);
        recurrence_step_d(S + bh * dv * dk, qk, qk + dk, v + bh * dv, exp(neg_softplus((double)x_alpha[bh])),
                          sigmoid((double)x_beta[bh]), out + bh * dv, x, dk, dv);
        free(x); free(qk);
    }
    return failed ? 2 : 0;
}

/* ------------------------------------------------------------------------
 * Backward (reverse mode) of the Sec. 3.3 recurrence, token by token.
 *
 * Given dL/do_t (d_out) and dL/dS_T (dS_final, NULL = 0) for the loss L of
 * the forward outputs, the adjoint G_t = dL/dS_t runs backwards:
 *     G_T = dS_final;   for t = T .. 1:
 *       G_t   += do_t q_t^T                       (o_t = S_t q_t)
 *       dq_t   = S_t^T do_t
 *       with x = S_{t-1} k_t and Gk = G_t k_t, from
 *       S_t = alpha_t S_{t-1} - alpha_t beta_t x k_t^T + beta_t v_t k_t^T:
 *       dv_t         = beta_t Gk
 *       dbeta_t      = (v_t - alpha_t x) . Gk
 *       dlog_alpha_t = alpha_t (<G_t, S_{t-1}> - beta_t x . Gk)
 *       dk_t         = -alpha_t beta_t (S_{t-1}^T Gk + G_t^T x) + beta_t G_t^T v_t
 *       G_{t-1}      = alpha_t G_t (I - beta_t k_t k_t^T)
 *     dS0 = G_0.
 * The forward states S_0 .. S_T are recomputed and kept (T + 1 states per
 * (b, h)), so this is for test sizes only.  All outputs are double.
 */
int gdn_oracle_backward(const float *q, const float *k, const float *v, const float *log_alpha,
                        const float *beta, const double *S0, const double *d_out,
                        const double *dS_final, double *dq, double *dk_out, double *dv_out,
                        double *dlog_alpha, double *dbeta, double *dS0, int64_t B, int64_t T,
                        int64_t H, int64_t dk, int64_t dv, int nthreads) {
    if (B < 0 || T < 0 || H < 0 || dk < 1 || dv < 1) return 1;
    set_threads(nthreads);
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        const int64_t b = bh / H, h = bh % H;
        const int64_t ns = dv * dk;
        double *St = (double *)malloc(sizeof(double) * ns * (T + 1));
        double *G = (double *)malloc(sizeof(double) * ns);
        double *x = (double *)malloc(sizeof(double) * dv);
        double *Gk = (double *)malloc(sizeof(double) * dv);
        double *o = (double *)malloc(sizeof(double) * dv);
        if (!St || !G || !x || !Gk || !o) {
            free(St); free(G); free(x); free(Gk); free(o);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        /* forward, keeping every state */
        if (S0) memcpy(St, S0 + IDX_STATE(b, h, H, dv, dk), sizeof(double) * ns);
        else memset(St, 0, sizeof(double) * ns);
        for (int64_t t = 0; t < T; ++t) {
            memcpy(St + (t + 1) * ns, St + t * ns, sizeof(double) * ns);
            recurrence_step(St + (t + 1) * ns, q + IDX_TOK(b, t, h, 0, T, H, dk), k + IDX_TOK(b, t, h, 0, T, H, dk),
                            v + IDX_TOK(b, t, h, 0, T, H, dv), log_alpha[IDX_GATE(b, t, h, T, H)],
                            beta[IDX_GATE(b, t, h, T, H)], o, x, dk, dv);
        }
        /* reverse sweep */
        if (dS_final) memcpy(G, dS_final + IDX_STATE(b, h, H, dv, dk), sizeof(double) * ns);
        else memset(G, 0, sizeof(double) * ns);
        for (int64_t t = T - 1; t >= 0; --t) {
            const float *qt = q + IDX_TOK(b, t, h, 0, T, H, dk), *kt = k + IDX_TOK(b, t, h, 0, T, H, dk);
            const float *vt = v + IDX_TOK(b, t, h, 0, T, H, dv);
            const double *dot = d_out + IDX_TOK(b, t, h, 0, T, H, dv);
            const double *Sn = St + (t + 1) * ns, *Sp = St + t * ns;   /* S_t and S_{t-1} */
            const int64_t gi = IDX_GATE(b, t, h, T, H);
            const double a = exp((double)log_alpha[gi]), bt = (double)beta[gi];
            for (int64_t r = 0; r < dv; ++r)
                for (int64_t c = 0; c < dk; ++c) G[r * dk + c] += dot[r] * (double)qt[c];
            double *dqt = dq + IDX_TOK(b, t, h, 0, T, H, dk);
            for (int64_t c = 0; c < dk; ++c) {
                double acc = 0.0;
                for (int64_t r = 0; r < dv; ++r) acc += Sn[r * dk + c] * dot[r];
                dqt[c] = acc;
            }
            double gs = 0.0, xgk = 0.0, vgk = 0.0;
            for (int64_t r = 0; r < dv; ++r) {
                double ax = 0.0, ag = 0.0;
                for (int64_t c = 0; c < dk; ++c) {
                    ax += Sp[r * dk + c] * (double)kt[c];
                    ag += G[r * dk + c] * (double)kt[c];
                    gs += G[r * dk + c] * Sp[r * dk + c];
                }
                x[r] = ax;
                Gk[r] = ag;
                xgk += ax * ag;
                vgk += (double)vt[r] * ag;
            }
            double *dvt = dv_out + IDX_TOK(b, t, h, 0, T, H, dv);
            for (int64_t r = 0; r < dv; ++r) dvt[r] = bt * Gk[r];
            dbeta[gi] = vgk - a * xgk;
            dlog_alpha[gi] = a * (gs - bt * xgk);
            double *dkt = dk_out + IDX_TOK(b, t, h, 0, T, H, dk);
            for (int64_t c = 0; c < dk; ++c) {
                double sgk = 0.0, gx = 0.0, gv = 0.0;
                for (int64_t r = 0; r < dv; ++r) {
                    sgk += Sp[r * dk + c] * Gk[r];
                    gx += G[r * dk + c] * x[r];
                    gv += G[r * dk + c] * (double)vt[r];
                }
                dkt[c] = -a * bt * (sgk + gx) + bt * gv;
            }
            for (int64_t r = 0; r < dv; ++r)
                for (int64_t c = 0; c < dk; ++c)
                    G[r * dk + c] = a * (G[r * dk + c] - bt * Gk[r] * (double)kt[c]);
        }
        if (dS0) memcpy(dS0 + IDX_STATE(b, h, H, dv, dk), G, sizeof(double) * ns);
        free(St); free(G); free(x); free(Gk); free(o);
    }
    return failed ? 2 : 0;
}

/* ------------------------------------------------------------------------
 * Grouped heads.  H_q query heads read the memories of H_kv = H_q / G
 * key-value heads: the memory of key-value head hk is written by its k, v
 * and gates (layouts [B, T, H_kv, .]) by the Sec. 3.3 recurrence, and query
 * head h = hk * G + g (g < G) reads it: o_t^(h) = S_t^(hk) q_t^(h).
 * q, out are [B, T, H_q, .]; S0, S_final are [B, H_kv, dv, dk].  (Reading:
 * the pages give the attention layers 8 query and 2 key-value heads but say
 * nothing of how the memory's heads map; this is the grouped-query mapping.)
 */
int gdn_oracle_forward_grouped(const float *q, const float *k, const float *v, const float *log_alpha,
                               const float *beta, const double *S0, double *out, double *S_final,
                               int64_t B, int64_t T, int64_t Hq, int64_t Hkv, int64_t dk, int64_t dv,
                               int nthreads) {
    if (B < 0 || T < 0 || Hq < 0 || Hkv < 1 || dk < 1 || dv < 1 || Hq % Hkv) return 1;
    const int64_t G = Hq / Hkv;
    set_threads(nthreads);
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < B * Hkv; ++bh) {
        const int64_t b = bh / Hkv, hk = bh % Hkv;
        double *S = (double *)malloc(sizeof(double) * dv * dk);
        double *x = (double *)malloc(sizeof(double) * dv);
        double *o = (double *)malloc(sizeof(double) * dv);
        if (!S || !x || !o) {
            free(S); free(x); free(o);
#pragma omp atomic write
            failed = 1;
            continue;
        }
        if (S0) memcpy(S, S0 + IDX_STATE(b, hk, Hkv, dv, dk), sizeof(double) * dv * dk);
        else memset(S, 0, sizeof(double) * dv * dk);
        for (int64_t t = 0; t < T; ++t) {
            /* the memory's step (its output for the first query head of the group is discarded
               and recomputed below with the others) */
            recurrence_step(S, q + IDX_TOK(b, t, hk * G, 0, T, Hq, dk), k + IDX_TOK(b, t, hk, 0, T, Hkv, dk),
                            v + IDX_TOK(b, t, hk, 0, T, Hkv, dv), log_alpha[IDX_GATE(b, t, hk, T, Hkv)],
                            beta[IDX_GATE(b, t, hk, T, Hkv)], o, x, dk, dv);
            for (int64_t g = 0; g < G; ++g) {
                const float *qh = q + IDX_TOK(b, t, hk * G + g, 0, T, Hq, dk);
                double *oh = out + IDX_TOK(b, t, hk * G + g, 0, T, Hq, dv);
                for (int64_t r = 0; r < dv; ++r) {
                    double acc = 0.0;
                    for (int64_t c = 0; c < dk; ++c) acc += S[r * dk + c] * (double)qh[c];
                    oh[r] = acc;
                }
            }
        }
        if (S_final) memcpy(S_final + IDX_STATE(b, hk, Hkv, dv, dk), S, sizeof(double) * dv * dk);
        free(S); free(x); free(o);
    }
    return failed ? 2 : 0;
}

/* ------------------------------------------------------------------------
 * The reverse mode in chunkwise form (test-only alternative form, float64).
 * For a chunk of n <= C tokens with entry state S (from the forward),
 * chunk-local g_t = sum_{r<=t} log alpha_r, gamma_t = e^{g_t}, dl_s =
 * e^{g_last - g_s}, A_ts = beta_t e^{g_t - g_s} (k_t . k_s) (s < t),
 * T = (I + A)^{-1}, R_t = beta_t (v_t - gamma_t S k_t), U = T R,
 * P_ts = e^{g_t - g_s} (q_t . k_s) (s <= t), O = diag(gamma) Q S^T + P U and
 * S' = gamma_last S + U^T diag(dl) K.  Given dO and dS' the adjoint of each
 * line, in reverse order:
 *   dU  = P^T dO + diag(dl) K dS'^T;   dR = T^T dU;   dV = diag(beta) dR
 *   dP_ts = dO_t . U_s (s <= t);       dA_ts = -dR_t . U_s (s < t)
 *   dQ  = diag(gamma) dO S + (dP o E) K,   E_ts = e^{g_t - g_s}
 *   dK  = (dP o E)^T Q + F K + F^T K - diag(beta gamma) dR S + diag(dl) U dS',
 *         F_ts = dA_ts beta_t E_ts
 *   dbeta_t = dR_t . (v_t - gamma_t S k_t) + sum_s dA_ts E_ts (k_t . k_s)
 *   dg: from gamma_t in O and R, from E in P and A, from dl and gamma_last;
 *       dlog_alpha_r = sum_{t >= r} dg_t + dg_last
 *   dS  = gamma_last dS' + dO^T diag(gamma) Q - dR^T diag(beta gamma) K
 * The chunk states come from the token recurrence.  Layouts as
 * gdn_oracle_backward.
 */
int gdn_oracle_backward_chunked(const float *q, const float *k, const float *v, const float *log_alpha,
                                const float *beta, const double *S0, const double *d_out,
                                const double *dS_final, double *dq, double *dk_out, double *dv_out,
                                double *dlog_alpha, double *dbeta, double *dS0, int64_t B, int64_t T,
                                int64_t H, int64_t dk, int64_t dv, int64_t C) {
    if (B < 0 || T < 0 || H < 0 || dk < 1 || dv < 1 || C < 1) return 1;
    const int64_t nc = (T + C - 1) / C, ns = dv * dk;
    for (int64_t bh = 0; bh < B * H; ++bh) {
        const int64_t b = bh / H, h = bh % H;
        double *Sc = (double *)malloc(sizeof(double) * ns * (nc + 1));
        double *S = (double *)malloc(sizeof(double) * ns);
        double *dS = (double *)malloc(sizeof(double) * ns), *dSn = (double *)malloc(sizeof(double) * ns);
        double *tmpx = (double *)malloc(sizeof(double) * dv), *tmpo = (double *)malloc(sizeof(double) * dv);
        double *g = (double *)malloc(sizeof(double) * C * 8);
        double *Am = (double *)malloc(sizeof(double) * C * C * 6);
        double *Mv = (double *)malloc(sizeof(double) * C * dv * 6);
        double *Mk = (double *)malloc(sizeof(double) * C * dk * 2);
        if (!Sc || !S || !dS || !dSn || !tmpx || !tmpo || !g || !Am || !Mv || !Mk) {
            free(Sc); free(S); free(dS); free(dSn); free(tmpx); free(tmpo); free(g); free(Am); free(Mv); free(Mk);
            return 2;
        }
        double *gam = g + C, *dl = g + 2 * C, *bet = g + 3 * C, *dg = g + 4 * C, *db = g + 5 * C;
        double *A = Am, *Tm = Am + C * C, *P = Am + 2 * C * C, *E = Am + 3 * C * C, *D = Am + 4 * C * C,
               *F = Am + 5 * C * C;
        double *X = Mv, *R = Mv + C * dv, *U = Mv + 2 * C * dv, *dO = Mv + 3 * C * dv, *dU = Mv + 4 * C * dv,
               *dR = Mv + 5 * C * dv;
        double *Q = Mk, *K = Mk + C * dk;
        /* chunk-start states by the token recurrence */
        if (S0) memcpy(S, S0 + IDX_STATE(b, h, H, dv, dk), sizeof(double) * ns);
        else memset(S, 0, sizeof(double) * ns);
        for (int64_t c = 0; c < nc; ++c) {
            memcpy(Sc + c * ns, S, sizeof(double) * ns);
            for (int64_t t = c * C; t < T && t < (c + 1) * C; ++t)
                recurrence_step(S, q + IDX_TOK(b, t, h, 0, T, H, dk), k + IDX_TOK(b, t, h, 0, T, H, dk),
                                v + IDX_TOK(b, t, h, 0, T, H, dv), log_alpha[IDX_GATE(b, t, h, T, H)],
                                beta[IDX_GATE(b, t, h, T, H)], tmpo, tmpx, dk, dv);
        }
        if (dS_final) memcpy(dS, dS_final + IDX_STATE(b, h, H, dv, dk), sizeof(double) * ns);
        else memset(dS, 0, sizeof(double) * ns);
        for (int64_t c = nc - 1; c >= 0; --c) {
            const int64_t t0 = c * C, n = (T - t0 < C) ? T - t0 : C;
            const double *Se = Sc + c * ns;
            double acc = 0.0;
            for (int64_t t = 0; t < n; ++t) {
                const int64_t gi = IDX_GATE(b, t0 + t, h, T, H);
                acc += (double)log_alpha[gi];
                g[t] = acc;
                gam[t] = exp(acc);
                bet[t] = (double)beta[gi];
                dg[t] = 0.0;
                db[t] = 0.0;
                for (int64_t i = 0; i < dk; ++i) {
                    Q[t * dk + i] = (double)q[IDX_TOK(b, t0 + t, h, i, T, H, dk)];
                    K[t * dk + i] = (double)k[IDX_TOK(b, t0 + t, h, i, T, H, dk)];
                }
                for (int64_t j = 0; j < dv; ++j) dO[t * dv + j] = d_out[IDX_TOK(b, t0 + t, h, j, T, H, dv)];
            }
            const double gl = g[n - 1], gaml = gam[n - 1];
            for (int64_t t = 0; t < n; ++t) dl[t] = exp(gl - g[t]);
            for (int64_t t = 0; t < n; ++t)
                for (int64_t s2 = 0; s2 < n; ++s2) {
                    double kk = 0.0, qk = 0.0;
                    for (int64_t i = 0; i < dk; ++i) {
                        kk += K[t * dk + i] * K[s2 * dk + i];
                        qk += Q[t * dk + i] * K[s2 * dk + i];
                    }
                    E[t * C + s2] = (s2 <= t) ? exp(g[t] - g[s2]) : 0.0;
                    A[t * C + s2] = (s2 < t) ? bet[t] * E[t * C + s2] * kk : 0.0;
                    P[t * C + s2] = (s2 <= t) ? E[t * C + s2] * qk : 0.0;
                }
            /* T = (I + A)^{-1} by forward substitution, column by column */
            for (int64_t j = 0; j < n; ++j)
                for (int64_t t = 0; t < n; ++t) {
                    double x = (t == j) ? 1.0 : 0.0;
                    for (int64_t s2 = 0; s2 < t; ++s2) x -= A[t * C + s2] * Tm[s2 * C + j];
                    Tm[t * C + j] = x;
                }
            /* X = gamma_t S k_t, R = beta (v - X), U = T R */
            for (int64_t t = 0; t < n; ++t)
                for (int64_t j = 0; j < dv; ++j) {
                    double a = 0.0;
                    for (int64_t i = 0; i < dk; ++i) a += Se[j * dk + i] * K[t * dk + i];
                    X[t * dv + j] = gam[t] * a;
                    R[t * dv + j] = bet[t] * ((double)v[IDX_TOK(b, t0 + t, h, j, T, H, dv)] - X[t * dv + j]);
                }
            for (int64_t t = 0; t < n; ++t)
                for (int64_t j = 0; j < dv; ++j) {
                    double a = 0.0;
                    for (int64_t s2 = 0; s2 <= t; ++s2) a += Tm[t * C + s2] * R[s2 * dv + j];
                    U[t * dv + j] = a;
                }
            /* dU = P^T dO + diag(dl) K dS^T, with d g from dl */
            double dgl = 0.0;
            for (int64_t s2 = 0; s2 < n; ++s2) {
                double w = 0.0;
                for (int64_t j = 0; j < dv; ++j) {
                    double a = 0.0, kd = 0.0;
                    for (int64_t t = s2; t < n; ++t) a += P[t * C + s2] * dO[t * dv + j];
                    for (int64_t i = 0; i < dk; ++i) kd += K[s2 * dk + i] * dS[j * dk + i];
                    dU[s2 * dv + j] = a + dl[s2] * kd;
                    w += U[s2 * dv + j] * dl[s2] * kd;
                }
                dg[s2] -= w;
                dgl += w;
            }
            /* d g from the outputs' gamma_t Q S^T term and from gamma_last S in S' */
            for (int64_t t = 0; t < n; ++t)
                for (int64_t j = 0; j < dv; ++j) {
                    double a = 0.0;
                    for (int64_t i = 0; i < dk; ++i) a += Se[j * dk + i] * Q[t * dk + i];
                    dg[t] += gam[t] * a * dO[t * dv + j];
                }
            for (int64_t e = 0; e < ns; ++e) dgl += gaml * dS[e] * Se[e];
            /* dR = T^T dU */
            for (int64_t s2 = 0; s2 < n; ++s2)
                for (int64_t j = 0; j < dv; ++j) {
                    double a = 0.0;
                    for (int64_t t = s2; t < n; ++t) a += Tm[t * C + s2] * dU[t * dv + j];
                    dR[s2 * dv + j] = a;
                }
            /* dV, dbeta and d g from R */
            for (int64_t t = 0; t < n; ++t) {
                double rb = 0.0, rg = 0.0;
                for (int64_t j = 0; j < dv; ++j) {
                    dv_out[IDX_TOK(b, t0 + t, h, j, T, H, dv)] = bet[t] * dR[t * dv + j];
                    rb += dR[t * dv + j] * ((double)v[IDX_TOK(b, t0 + t, h, j, T, H, dv)] - X[t * dv + j]);
                    rg += dR[t * dv + j] * X[t * dv + j];
                }
                db[t] += rb;
                dg[t] -= bet[t] * rg;
            }
            /* dP o E (= D), F from dA; dbeta and d g from P and A */
            for (int64_t t = 0; t < n; ++t)
                for (int64_t s2 = 0; s2 < n; ++s2) {
                    double dp = 0.0, da = 0.0;
                    for (int64_t j = 0; j < dv; ++j) {
                        dp += dO[t * dv + j] * U[s2 * dv + j];
                        da -= dR[t * dv + j] * U[s2 * dv + j];
                    }
                    D[t * C + s2] = (s2 <= t) ? dp * E[t * C + s2] : 0.0;
                    F[t * C + s2] = (s2 < t) ? da * bet[t] * E[t * C + s2] : 0.0;
                    if (s2 <= t) {
                        dg[t] += dp * P[t * C + s2];
                        dg[s2] -= dp * P[t * C + s2];
                    }
                    if (s2 < t) {
                        double kk = 0.0;
                        for (int64_t i = 0; i < dk; ++i) kk += K[t * dk + i] * K[s2 * dk + i];
                        db[t] += da * E[t * C + s2] * kk;
                        dg[t] += da * A[t * C + s2];
                        dg[s2] -= da * A[t * C + s2];
                    }
                }
            /* dQ, dK */
            for (int64_t t = 0; t < n; ++t)
                for (int64_t i = 0; i < dk; ++i) {
                    double aq = 0.0, ak = 0.0;
                    for (int64_t j = 0; j < dv; ++j) {
                        aq += gam[t] * dO[t * dv + j] * Se[j * dk + i];
                        ak += -bet[t] * gam[t] * dR[t * dv + j] * Se[j * dk + i] + dl[t] * U[t * dv + j] * dS[j * dk + i];
                    }
                    for (int64_t s2 = 0; s2 < n; ++s2) {
                        aq += D[t * C + s2] * K[s2 * dk + i];
                        ak += D[s2 * C + t] * Q[s2 * dk + i] + F[t * C + s2] * K[s2 * dk + i] + F[s2 * C + t] * K[s2 * dk + i];
                    }
                    dq[IDX_TOK(b, t0 + t, h, i, T, H, dk)] = aq;
                    dk_out[IDX_TOK(b, t0 + t, h, i, T, H, dk)] = ak;
                }
            /* d log alpha and dbeta */
            for (int64_t r = 0; r < n; ++r) {
                double sum = dgl;
                for (int64_t t = r; t < n; ++t) sum += dg[t];
                dlog_alpha[IDX_GATE(b, t0 + r, h, T, H)] = sum;
                dbeta[IDX_GATE(b, t0 + r, h, T, H)] = db[r];
            }
            /* dS for the previous chunk */
            for (int64_t j = 0; j < dv; ++j)
                for (int64_t i = 0; i < dk; ++i) {
                    double a = gaml * dS[j * dk + i];
                    for (int64_t t = 0; t < n; ++t)
                        a += gam[t] * dO[t * dv + j] * Q[t * dk + i] - bet[t] * gam[t] * dR[t * dv + j] * K[t * dk + i];
                    dSn[j * dk + i] = a;
                }
            memcpy(dS, dSn, sizeof(double) * ns);
        }
        if (dS0) memcpy(dS0 + IDX_STATE(b, h, H, dv, dk), dS, sizeof(double) * ns);
        free(Sc); free(S); free(dS); free(dSn); free(tmpx); free(tmpo); free(g); free(Am); free(Mv); free(Mk);
    }
    return 0;
}
