// bwd_simt.cu -- reverse mode of the chunkwise gated-delta forward, float32 on
// the CUDA cores, any supported (dk, dv, chunk).
//
// The forward is the Sec. 3.3 recurrence of "ATMA: Long-Context Language
// Modeling via Polar Attention and Gated-Delta Compression Memory" in its
// chunkwise form.  Inside a chunk with entry state S (chunk-local log-decay
// cumsum g_t, gamma_t = e^{g_t}, dl_s = e^{g_C - g_s}):
//     (I + A) U = R,   R_t = beta_t (v_t - gamma_t S k_t),
//     A_ts = beta_t e^{g_t - g_s} (k_t . k_s)            (s < t)
//     O    = diag(gamma) Q S^T + P U,  P_ts = e^{g_t - g_s} (q_t . k_s)   (s <= t)
//     S'   = gamma_C S + U^T diag(dl) K.
// Given dO and dS' this kernel walks the chunks backwards and applies, per
// chunk, the adjoint of each line in reverse order:
//     dU  = P^T dO + diag(dl) K dS'^T
//     dR  = (I + A)^{-T} dU                       (back substitution)
//     dV  = diag(beta) dR
//     dP  = dO U^T (s <= t),  dA = -dR U^T (s < t)
//     dQ  = diag(gamma) dO S + (dP o E) K,        E_ts = e^{g_t - g_s}
//     dK  = (dP o E)^T Q + F K + F^T K - diag(beta gamma) dR S + diag(dl) U dS',
//           F_ts = dA_ts beta_t E_ts
//     dbeta_t = dR_t . (v_t - gamma_t S k_t) + sum_s dA_ts E_ts (k_t . k_s)
//     dS  = gamma_C dS' + dO^T diag(gamma) Q - dR^T diag(beta gamma) K
// and the log-decays collect dg_t from every e^{g} they enter (outputs,
// R, P, A, dl and gamma_C); d log alpha_r = sum_{t >= r} dg_t + dg_C, the
// adjoint of the chunk-local cumsum.
//
// The states entering the chunks come from a forward recompute that writes
// them as checkpoints: the two-kernel tensor-core forward (its chain kernel
// stores the float32 state it holds in tensor memory at every chunk start)
// where that forward applies, else the CUDA-core forward with outputs off.  One CTA owns one (b, h) and a slab of
// `rows` value dimensions.  dU, dR, dV and the slab of dS depend only on the
// slab's value dimensions; dQ, dK, dbeta and dlog_alpha are sums over value
// dimensions, so each slab adds its share with float32 atomics.
#include <stdlib.h>
#include <string.h>

#include <atomic>

#include "common.cuh"
#include "gdn.h"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kThreads = 512;

struct BwdDims {
    int dk, dv, C, rows, nslab, nchunks;
    int ldk, ldr, ldc;
    size_t smem_floats() const {
        return 2 * (size_t)rows * ldk + 2 * (size_t)C * ldk + 5 * (size_t)C * ldr + 3 * (size_t)C * ldc +
               6 * (size_t)C + 4;
    }
};

// acc[a][b] += sum_c X[(i0+a)*ldx + c] * Y[(jb+G*b)*ldy + c],  c in [0, K).  The Y rows of a thread
// are G apart, so that neighbouring threads (consecutive jb, one i0) read neighbouring rows: the eight
// 16-byte loads of a quarter warp then fall in eight different bank groups (rows 4 apart would share
// two, with a row pitch of an odd number of 16-byte units).
__device__ __forceinline__ void tile_nt(const float *X, int ldx, const float *Y, int ldy, int i0, int jb, int G,
                                        int K, float acc[4][4]) {
    for (int c = 0; c < K; c += 4) {
        float4 x[4], y[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) x[a] = *reinterpret_cast<const float4 *>(X + (i0 + a) * ldx + c);
#pragma unroll
        for (int b = 0; b < 4; ++b) y[b] = *reinterpret_cast<const float4 *>(Y + (jb + G * b) * ldy + c);
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] += dot4(x[a], y[b]);
    }
}

// acc[a][b] += x[a] * y[b]
__device__ __forceinline__ void outer4(float acc[4][4], const float x[4], const float4 y) {
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        acc[a][0] = fmaf(x[a], y.x, acc[a][0]);
        acc[a][1] = fmaf(x[a], y.y, acc[a][1]);
        acc[a][2] = fmaf(x[a], y.z, acc[a][2]);
        acc[a][3] = fmaf(x[a], y.w, acc[a][3]);
    }
}

__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }

template <typename Tin>
__device__ __forceinline__ void store4(Tin *p, float a, float b, float c, float d);
template <>
__device__ __forceinline__ void store4<float>(float *p, float a, float b, float c, float d) {
    *reinterpret_cast<float4 *>(p) = make_float4(a, b, c, d);
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16 *p, float a, float b, float c, float d) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&lo);
    u.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(p) = u;
}

template <typename Tin>
__global__ void __launch_bounds__(kThreads)
bwd_simt_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                const float *__restrict__ log_alpha, const float *__restrict__ beta,
                const float *__restrict__ ckpt, const Tin *__restrict__ d_out, const float *__restrict__ dS_final,
                float *__restrict__ dq_acc, float *__restrict__ dk_acc, Tin *__restrict__ dv_out,
                float *__restrict__ dla_out, float *__restrict__ dbeta_out, float *__restrict__ dS0, int64_t T,
                int64_t H, BwdDims d) {
    extern __shared__ __align__(16) float sm[];
    const int dk = d.dk, dv = d.dv, C = d.C, rows = d.rows;
    const int LDK = d.ldk, LDR = d.ldr, LDC = d.ldc;
    float *Ss = sm;                 // rows x LDK  state slab entering the chunk
    float *dSs = Ss + rows * LDK;   // rows x LDK  dS slab (of the state leaving the chunk)
    float *Qs = dSs + rows * LDK;   // C x LDK
    float *Ks = Qs + C * LDK;       // C x LDK
    float *Vs = Ks + C * LDK;       // C x LDR  v slab
    float *Xs = Vs + C * LDR;       // C x LDR  gamma_t (S k_t) slab
    float *dOs = Xs + C * LDR;      // C x LDR
    float *Us = dOs + C * LDR;      // C x LDR
    float *dRs = Us + C * LDR;      // C x LDR  diag(dl) K dS^T, then dU, then dR
    float *MA = dRs + C * LDR;      // C x LDC  e^{g_t-g_s} (k_t . k_s) (s < t), then F
    float *MP = MA + C * LDC;       // C x LDC  P
    float *MD = MP + C * LDC;       // C x LDC  T = (I + A)^{-1}, then dP o E
    float *g = MD + C * LDC;        // C
    float *bet = g + C;             // C
    float *gam = bet + C;           // C
    float *dl = gam + C;            // C
    float *dg = dl + C;             // C  d g_t (this slab's share)
    float *db = dg + C;             // C  d beta_t (this slab's share)
    float *dgC = db + C;            // 1  d g_C

    const int tid = threadIdx.x;
    const int64_t bh = blockIdx.x / d.nslab;
    const int slab = blockIdx.x % d.nslab;
    const int64_t b = bh / H, h = bh % H;
    const int r0 = slab * rows;
    const int64_t tsk = H * dk, tsv = H * dv;  // token strides
    const int64_t base_k = (b * T * H + h) * dk, base_v = (b * T * H + h) * dv, base_g = b * T * H + h;

    // dS slab <- dS_final (or zero)
    for (int i = tid; i < rows * (dk / 4); i += kThreads) {
        const int j = i / (dk / 4), c4 = i % (dk / 4);
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        if (dS_final) s = ld4(dS_final + (bh * dv + r0 + j) * (int64_t)dk + 4 * c4);
        *reinterpret_cast<float4 *>(dSs + j * LDK + 4 * c4) = s;
    }

    for (int c = d.nchunks - 1; c >= 0; --c) {
        const int64_t t0 = (int64_t)c * C;
        const int n = (int)((T - t0 < C) ? (T - t0) : C);
        __syncthreads();  // the previous (later) chunk is done with every buffer
        // ---- load the chunk (zero-padded tail) and the state entering it ----
        for (int i = tid; i < C * (dk / 4); i += kThreads) {
            const int t = i / (dk / 4), c4 = i % (dk / 4);
            float4 qa = make_float4(0.f, 0.f, 0.f, 0.f), ka = qa;
            if (t < n) {
                qa = load4(q + base_k + (t0 + t) * tsk + 4 * c4);
                ka = load4(k + base_k + (t0 + t) * tsk + 4 * c4);
            }
            *reinterpret_cast<float4 *>(Qs + t * LDK + 4 * c4) = qa;
            *reinterpret_cast<float4 *>(Ks + t * LDK + 4 * c4) = ka;
        }
        for (int i = tid; i < C * (rows / 4); i += kThreads) {
            const int t = i / (rows / 4), c4 = i % (rows / 4);
            float4 va = make_float4(0.f, 0.f, 0.f, 0.f), oa = va;
            if (t < n) {
                va = load4(v + base_v + (t0 + t) * tsv + r0 + 4 * c4);
                oa = load4(d_out + base_v + (t0 + t) * tsv + r0 + 4 * c4);
            }
            *reinterpret_cast<float4 *>(Vs + t * LDR + 4 * c4) = va;
            *reinterpret_cast<float4 *>(dOs + t * LDR + 4 * c4) = oa;
        }
        {
            const float *src = ckpt + ((bh * d.nchunks + c) * dv + r0) * (int64_t)dk;
            for (int i = tid; i < rows * (dk / 4); i += kThreads) {
                const int j = i / (dk / 4), c4 = i % (dk / 4);
                *reinterpret_cast<float4 *>(Ss + j * LDK + 4 * c4) = ld4(src + (int64_t)j * dk + 4 * c4);
            }
        }
        if (tid < 32) {  // chunk-local inclusive cumsum of the clamped log_alpha (C <= 64)
            float x0 = 0.f, x1 = 0.f;
            const int e0 = 2 * tid, e1 = 2 * tid + 1;
            if (e0 < n) x0 = fmaxf(log_alpha[base_g + (t0 + e0) * H], kLogAlphaFloor);
            if (e1 < n) x1 = fmaxf(log_alpha[base_g + (t0 + e1) * H], kLogAlphaFloor);
            float s = x0 + x1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, s, off);
                if (tid >= off) s += y;
            }
            if (e0 < C) g[e0] = s - x1;
            if (e1 < C) g[e1] = s;
        }
        for (int t = tid; t < C; t += kThreads) {
            bet[t] = (t < n) ? beta[base_g + (t0 + t) * H] : 0.f;
            dg[t] = 0.f;
            db[t] = 0.f;
        }
        if (tid == 0) *dgC = 0.f;
        __syncthreads();
        for (int t = tid; t < C; t += kThreads) {
            gam[t] = expf(g[t]);
            dl[t] = expf(g[C - 1] - g[t]);
        }
        __syncthreads();

        // ---- pass 1: Xs = diag(gamma) K S^T;  MA = E o K K^T (s < t);  MP = P;  dRs = diag(dl) K dS^T ----
        {
            const int nx = (C / 4) * (rows / 4), nc = (C / 4) * (C / 4);
            for (int w = tid; w < 2 * nx + 2 * nc; w += kThreads) {
                float acc[4][4] = {};
                if (w < 2 * nx) {
                    const int ww = w % nx, G = rows / 4;
                    const int i0 = (ww / G) * 4, jb = ww % G;
                    const bool isx = w < nx;
                    tile_nt(Ks, LDK, isx ? Ss : dSs, LDK, i0, jb, G, dk, acc);
                    float *dst = isx ? Xs : dRs;
                    const float *f = isx ? gam : dl;
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int bb = 0; bb < 4; ++bb) dst[(i0 + a) * LDR + jb + G * bb] = f[i0 + a] * acc[a][bb];
                } else {
                    const int ww = (w - 2 * nx) % nc, G = C / 4;
                    const bool isa = (w - 2 * nx) < nc;
                    const int i0 = (ww / G) * 4, jb = ww % G;
                    if (jb <= i0 + 3) tile_nt(isa ? Ks : Qs, LDK, Ks, LDK, i0, jb, G, dk, acc);
                    float *dst = isa ? MA : MP;
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int bb = 0; bb < 4; ++bb) {
                            const int t = i0 + a, s = jb + G * bb;
                            const bool keep = isa ? (s < t) : (s <= t);
                            const float x = keep ? expf(g[t] - g[s]) * acc[a][bb] : 0.f;
                            dst[t * LDC + s] = x;
                        }
                }
            }
        }
        __syncthreads();

        // ---- pass 2: T = (I + A)^{-1} into MD, A_ts = beta_t MA_ts (unit lower triangular), blocked:
        //      16 x 16 diagonal blocks by substitution in registers (a thread per block column), then
        //      T_10 = -T_11 (A_10 T_00) for the 16 -> 32 and 32 -> 64 merges, with Us as scratch ----
        {
            for (int i = tid; i < C * C; i += kThreads) MD[(i / C) * LDC + (i % C)] = 0.f;
            __syncthreads();
            if (tid < C) {
                const int o = (tid / 16) * 16, col = tid % 16;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float acc = (r == col) ? 1.f : 0.f;
                    const float br = bet[o + r];
#pragma unroll
                    for (int s2 = 0; s2 < r; ++s2) acc = fmaf(-br * MA[(o + r) * LDC + o + s2], x[s2], acc);
                    x[r] = acc;
                }
#pragma unroll
                for (int r = 0; r < 16; ++r) MD[(o + r) * LDC + o + col] = x[r];
            }
            __syncthreads();
            float *Y = Us;  // [32][32] scratch, row stride 32
            for (int h = 16; h < C; h *= 2) {
                // each 2h block: Y = A_10 T_00 (h x h), then T_10 = -T_11 Y
                const int nb = C / (2 * h), per = h * h;
                for (int i = tid; i < nb * per; i += kThreads) {
                    const int blk = i / per, r = (i % per) / h, cc = i % h, o = blk * 2 * h;
                    float acc = 0.f;
                    const float br = bet[o + h + r];
                    for (int kk = cc; kk < h; ++kk)  // T_00 is lower triangular: rows kk >= cc
                        acc = fmaf(br * MA[(o + h + r) * LDC + o + kk], MD[(o + kk) * LDC + o + cc], acc);
                    Y[(blk * h + r) * 32 + cc] = acc;
                }
                __syncthreads();
                for (int i = tid; i < nb * per; i += kThreads) {
                    const int blk = i / per, r = (i % per) / h, cc = i % h, o = blk * 2 * h;
                    float acc = 0.f;
                    for (int kk = 0; kk <= r; ++kk)  // T_11 is lower triangular: columns kk <= r
                        acc = fmaf(MD[(o + h + r) * LDC + o + h + kk], Y[(blk * h + kk) * 32 + cc], acc);
                    MD[(o + h + r) * LDC + o + cc] = -acc;
                }
                __syncthreads();
            }
        }

        // ---- pass 2b: U = T R, R_s = beta_s (v_s - X_s), R formed on the fly; one row and four
        //      columns per thread, so that every thread has work ----
        {
            const int nu = C * (rows / 4);
            for (int w = tid; w < nu; w += kThreads) {
                const int t = w / (rows / 4), j0 = (w % (rows / 4)) * 4;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int s2 = 0; s2 <= t; ++s2) {
                    const float m = MD[t * LDC + s2] * bet[s2];
                    const float4 v4 = ld4(Vs + s2 * LDR + j0), x4 = ld4(Xs + s2 * LDR + j0);
                    acc.x = fmaf(m, v4.x - x4.x, acc.x);
                    acc.y = fmaf(m, v4.y - x4.y, acc.y);
                    acc.z = fmaf(m, v4.z - x4.z, acc.z);
                    acc.w = fmaf(m, v4.w - x4.w, acc.w);
                }
                *reinterpret_cast<float4 *>(Us + t * LDR + j0) = acc;
            }
        }
        __syncthreads();

        // ---- pass 3: dU = P^T dO + diag(dl) K dS^T (with d g from dl: w_s = U_s . dl_s (K dS^T)_s);
        //      d g_t from the outputs' gamma_t Q S^T term;  d g_C from gamma_C <dS, S> ----
        {
            const int nu = (C / 4) * (rows / 4), ny = nu, ns = rows * (dk / 4);
            float dgc_part = 0.f;  // this thread's share of d g_C, summed over its warp at the end
            for (int w = tid; w < nu + ny + ns; w += kThreads) {
                if (w < nu) {
                    const int s0 = (w / (rows / 4)) * 4, j0 = (w % (rows / 4)) * 4;
                    float acc[4][4] = {};
                    for (int t = s0; t < C; ++t) {
                        const float4 p4 = ld4(MP + t * LDC + s0);
                        const float pv[4] = {p4.x, p4.y, p4.z, p4.w};
                        outer4(acc, pv, ld4(dOs + t * LDR + j0));
                    }
                    float wsum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        float *dr = dRs + (s0 + a) * LDR + j0;
                        const float *u = Us + (s0 + a) * LDR + j0;
#pragma unroll
                        for (int bb = 0; bb < 4; ++bb) {
                            wsum[a] = fmaf(u[bb], dr[bb], wsum[a]);
                            dr[bb] += acc[a][bb];
                        }
                    }
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        atomicAdd(&dg[s0 + a], -wsum[a]);
                        dgc_part += wsum[a];
                    }
                } else if (w < nu + ny) {
                    const int ww = w - nu, G = rows / 4;
                    const int i0 = (ww / G) * 4, jb = ww % G;
                    float acc[4][4] = {};
                    tile_nt(Qs, LDK, Ss, LDK, i0, jb, G, dk, acc);
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        float x = 0.f;
#pragma unroll
                        for (int bb = 0; bb < 4; ++bb) x = fmaf(acc[a][bb], dOs[(i0 + a) * LDR + jb + G * bb], x);
                        atomicAdd(&dg[i0 + a], gam[i0 + a] * x);
                    }
                } else {
                    const int ww = w - nu - ny;
                    const int j = ww / (dk / 4), c4 = ww % (dk / 4);
                    const float4 a4 = ld4(dSs + j * LDK + 4 * c4), s4 = ld4(Ss + j * LDK + 4 * c4);
                    dgc_part = fmaf(gam[C - 1], dot4(a4, s4), dgc_part);
                }
            }
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) dgc_part += __shfl_xor_sync(0xffffffffu, dgc_part, off);
            if ((tid & 31) == 0) atomicAdd(dgC, dgc_part);
        }
        __syncthreads();

        // ---- pass 4: dR = T^T dU (in place: every tile is read before any is written) ----
        {
            const int nr = (C / 4) * (rows / 4);
            float acc[4][4] = {};
            int s0l = -1, j0 = 0;
            if (tid < nr) {  // nr <= kThreads: one tile per thread
                s0l = (tid / (rows / 4)) * 4;
                j0 = (tid % (rows / 4)) * 4;
                for (int t = s0l; t < C; ++t) {
                    const float4 m4 = ld4(MD + t * LDC + s0l);
                    const float x[4] = {m4.x, m4.y, m4.z, m4.w};
                    outer4(acc, x, ld4(dRs + t * LDR + j0));
                }
            }
            __syncthreads();
            if (s0l >= 0) {
#pragma unroll
                for (int a = 0; a < 4; ++a)
                    *reinterpret_cast<float4 *>(dRs + (s0l + a) * LDR + j0) =
                        make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
            }
        }
        __syncthreads();

        // ---- pass 5: dV = diag(beta) dR (stored);  dbeta, d g from R;  MD = dP o E (d g from P);
        //      MA <- F = dA beta_t E (dbeta, d g from A) ----
        {
            const int nv = (C / 4) * (rows / 4), nc = (C / 4) * (C / 4);
            for (int w = tid; w < nv + 2 * nc; w += kThreads) {
                if (w < nv) {
                    const int t0l = (w / (rows / 4)) * 4, j0 = (w % (rows / 4)) * 4;
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        const int t = t0l + a;
                        const float4 r4 = ld4(dRs + t * LDR + j0);
                        const float4 v4 = ld4(Vs + t * LDR + j0), x4 = ld4(Xs + t * LDR + j0);
                        const float4 w4 = make_float4(v4.x - x4.x, v4.y - x4.y, v4.z - x4.z, v4.w - x4.w);
                        atomicAdd(&db[t], dot4(r4, w4));
                        atomicAdd(&dg[t], -bet[t] * dot4(r4, x4));
                        if (t < n)
                            store4<Tin>(dv_out + base_v + (t0 + t) * tsv + r0 + j0, bet[t] * r4.x, bet[t] * r4.y,
                                        bet[t] * r4.z, bet[t] * r4.w);
                    }
                } else {
                    const int ww = (w - nv) % nc, G = C / 4;
                    const bool isp = (w - nv) < nc;
                    const int i0 = (ww / G) * 4, jb = ww % G;
                    // dP = dO U^T, or -dA = dR U^T
                    float acc[4][4] = {};
                    if (jb <= i0 + 3) tile_nt(isp ? dOs : dRs, LDR, Us, LDR, i0, jb, G, rows, acc);
                    float rs[4] = {0.f, 0.f, 0.f, 0.f}, cs[4] = {0.f, 0.f, 0.f, 0.f}, bs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int bb = 0; bb < 4; ++bb) {
                            const int t = i0 + a, s = jb + G * bb;
                            if (isp) {
                                float dd = 0.f;
                                if (s <= t) {
                                    const float e = expf(g[t] - g[s]);
                                    const float gp = acc[a][bb] * MP[t * LDC + s];  // dP_ts P_ts
                                    rs[a] += gp;
                                    cs[bb] += gp;
                                    dd = acc[a][bb] * e;
                                }
                                MD[t * LDC + s] = dd;
                            } else {
                                float f = 0.f;
                                if (s < t) {
                                    const float e = expf(g[t] - g[s]);
                                    const float ea = -acc[a][bb];  // dA_ts
                                    const float kk = MA[t * LDC + s];  // E_ts (k_t . k_s)
                                    bs[a] += ea * kk;
                                    const float ga = ea * bet[t] * kk;  // dA_ts A_ts
                                    rs[a] += ga;
                                    cs[bb] += ga;
                                    f = ea * bet[t] * e;
                                }
                                MA[t * LDC + s] = f;
                            }
                        }
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        if (rs[a] != 0.f) atomicAdd(&dg[i0 + a], rs[a]);
                        if (cs[a] != 0.f) atomicAdd(&dg[jb + G * a], -cs[a]);
                        if (!isp && bs[a] != 0.f) atomicAdd(&db[i0 + a], bs[a]);
                    }
                }
            }
        }
        __syncthreads();

        // ---- pass 6: dQ, dK (this slab's share, float32 atomics);  dbeta, dlog_alpha ----
        {
            const int nq = (C / 4) * (dk / 4);
            for (int w = tid; w < 2 * nq; w += kThreads) {
                const int ww = w % nq;
                const int i0 = (ww / (dk / 4)) * 4, c0 = (ww % (dk / 4)) * 4;
                float acc[4][4] = {};
                if (w < nq) {
                    // dQ = diag(gamma) dO S + (dP o E) K; the row operands are read four columns at a time
                    for (int j = 0; j < rows; j += 4) {
                        float xo[4][4];
#pragma unroll
                        for (int a = 0; a < 4; ++a) {
                            const float4 o4 = ld4(dOs + (i0 + a) * LDR + j);
                            const float ga = gam[i0 + a];
                            xo[0][a] = o4.x * ga; xo[1][a] = o4.y * ga; xo[2][a] = o4.z * ga; xo[3][a] = o4.w * ga;
                        }
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) outer4(acc, xo[jj], ld4(Ss + (j + jj) * LDK + c0));
                    }
                    for (int s = 0; s <= i0; s += 4) {  // columns s .. s + 3; D is zero above the diagonal
                        float xd[4][4];
#pragma unroll
                        for (int a = 0; a < 4; ++a) {
                            const float4 d4 = ld4(MD + (i0 + a) * LDC + s);
                            xd[0][a] = d4.x; xd[1][a] = d4.y; xd[2][a] = d4.z; xd[3][a] = d4.w;
                        }
#pragma unroll
                        for (int ss = 0; ss < 4; ++ss) outer4(acc, xd[ss], ld4(Ks + (s + ss) * LDK + c0));
                    }
                } else {
                    // dK = (dP o E)^T Q + F^T K + F K - diag(beta gamma) dR S + diag(dl) U dS
                    for (int t = i0; t < C; ++t) {
                        const float4 d4 = ld4(MD + t * LDC + i0), f4 = ld4(MA + t * LDC + i0);
                        const float xd[4] = {d4.x, d4.y, d4.z, d4.w}, xf[4] = {f4.x, f4.y, f4.z, f4.w};
                        outer4(acc, xd, ld4(Qs + t * LDK + c0));
                        outer4(acc, xf, ld4(Ks + t * LDK + c0));
                    }
                    for (int s = 0; s <= i0; s += 4) {  // F K; F is zero on and above the diagonal
                        float xf[4][4];
#pragma unroll
                        for (int a = 0; a < 4; ++a) {
                            const float4 f4 = ld4(MA + (i0 + a) * LDC + s);
                            xf[0][a] = f4.x; xf[1][a] = f4.y; xf[2][a] = f4.z; xf[3][a] = f4.w;
                        }
#pragma unroll
                        for (int ss = 0; ss < 4; ++ss) outer4(acc, xf[ss], ld4(Ks + (s + ss) * LDK + c0));
                    }
                    float fr[4], fu[4];
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        fr[a] = -bet[i0 + a] * gam[i0 + a];
                        fu[a] = dl[i0 + a];
                    }
                    for (int j = 0; j < rows; j += 4) {
                        float xr[4][4], xu[4][4];
#pragma unroll
                        for (int a = 0; a < 4; ++a) {
                            const float4 r4 = ld4(dRs + (i0 + a) * LDR + j), u4 = ld4(Us + (i0 + a) * LDR + j);
                            xr[0][a] = r4.x * fr[a]; xr[1][a] = r4.y * fr[a]; xr[2][a] = r4.z * fr[a];
                            xr[3][a] = r4.w * fr[a];
                            xu[0][a] = u4.x * fu[a]; xu[1][a] = u4.y * fu[a]; xu[2][a] = u4.z * fu[a];
                            xu[3][a] = u4.w * fu[a];
                        }
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) {
                            outer4(acc, xr[jj], ld4(Ss + (j + jj) * LDK + c0));
                            outer4(acc, xu[jj], ld4(dSs + (j + jj) * LDK + c0));
                        }
                    }
                }
                float *dst = (w < nq) ? dq_acc : dk_acc;
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const int t = i0 + a;
                    if (t < n) {
                        float *p = dst + base_k + (t0 + t) * tsk + c0;
#pragma unroll
                        for (int bb = 0; bb < 4; ++bb) atomicAdd(p + bb, acc[a][bb]);
                    }
                }
            }
            // d log_alpha_r = sum_{t >= r} dg_t + dg_C (zero where the forward clamped log_alpha)
            for (int r = tid; r < n; r += kThreads) {
                float s = *dgC;
                for (int t = r; t < C; ++t) s += dg[t];
                const float la = log_alpha[base_g + (t0 + r) * H];
                atomicAdd(&dla_out[base_g + (t0 + r) * H], la >= kLogAlphaFloor ? s : 0.f);
                atomicAdd(&dbeta_out[base_g + (t0 + r) * H], db[r]);
            }
        }
        __syncthreads();

        // ---- pass 7: dS <- gamma_C dS + dO^T diag(gamma) Q - dR^T diag(beta gamma) K ----
        {
            const float gC = gam[C - 1];
            const int ns = (rows / 4) * (dk / 4);
            for (int w = tid; w < ns; w += kThreads) {
                const int j0 = (w / (dk / 4)) * 4, c0 = (w % (dk / 4)) * 4;
                float acc[4][4] = {};
                for (int t = 0; t < C; ++t) {
                    const float4 o4 = ld4(dOs + t * LDR + j0), r4 = ld4(dRs + t * LDR + j0);
                    const float fo = gam[t], fr = -bet[t] * gam[t];
                    const float xo[4] = {o4.x * fo, o4.y * fo, o4.z * fo, o4.w * fo};
                    const float xr[4] = {r4.x * fr, r4.y * fr, r4.z * fr, r4.w * fr};
                    outer4(acc, xo, ld4(Qs + t * LDK + c0));
                    outer4(acc, xr, ld4(Ks + t * LDK + c0));
                }
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    float4 *sp = reinterpret_cast<float4 *>(dSs + (j0 + a) * LDK + c0);
                    float4 s = *sp;
                    s.x = fmaf(gC, s.x, acc[a][0]);
                    s.y = fmaf(gC, s.y, acc[a][1]);
                    s.z = fmaf(gC, s.z, acc[a][2]);
                    s.w = fmaf(gC, s.w, acc[a][3]);
                    *sp = s;
                }
            }
        }
    }
    __syncthreads();
    if (dS0) {
        for (int i = tid; i < rows * (dk / 4); i += kThreads) {
            const int j = i / (dk / 4), c4 = i % (dk / 4);
            *reinterpret_cast<float4 *>(dS0 + (bh * dv + r0 + j) * (int64_t)dk + 4 * c4) =
                ld4(dSs + j * LDK + 4 * c4);
        }
    }
}

// float32 accumulators -> dtype outputs
__global__ void cast_bf16_kernel(const float *__restrict__ src, __nv_bfloat16 *__restrict__ dst, int64_t n4) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        const float4 x = ld4(src + 4 * i);
        store4<__nv_bfloat16>(dst + 4 * i, x.x, x.y, x.z, x.w);
    }
}

BwdDims plan(const BwdProblem &p, int sm_count) {
    BwdDims d;
    d.dk = (int)p.f.dk;
    d.dv = (int)p.f.dv;
    d.C = (int)p.f.chunk;
    d.nchunks = (int)((p.f.T + p.f.chunk - 1) / p.f.chunk);
    d.ldk = d.dk + 4;
    d.ldc = d.C + 4;
    const int64_t heads = p.f.B * p.f.H;
    int nslab = 1;
    auto fits = [&](int ns) {
        BwdDims t = d;
        t.rows = d.dv / ns;
        t.ldr = t.rows + 4;
        return t.smem_floats() * sizeof(float) <= 227 * 1024;
    };
    while ((!fits(nslab) || heads * nslab < sm_count) && d.dv / (nslab * 2) >= 16) nslab *= 2;
    d.nslab = nslab;
    d.rows = d.dv / nslab;
    d.ldr = d.rows + 4;
    return d;
}

// The tensor-core recompute serves the shapes of the two-kernel forward unless
// GDN_BWD_RECOMPUTE=simt.
bool tc_recompute(const FwdProblem &f) {
    const char *e = getenv("GDN_BWD_RECOMPUTE");
    return fwd_split_supported(f) && !(e && strcmp(e, "simt") == 0);
}

// workspace: checkpoints | (bf16) float32 dq, dk accumulators | (tensor-core recompute) its
// per-chunk workspace and an output buffer
struct BwdLayout {
    size_t ckpt, acc, fwd_ws, fwd_out, total;
    int nseg;
};

BwdLayout layout(const BwdProblem &p, int sm_count) {
    const FwdProblem &f = p.f;
    BwdLayout l;
    const int64_t nchunks = (f.T + f.chunk - 1) / f.chunk, ntok = f.B * f.T * f.H;
    auto round = [](size_t x) { return (x + 255) & ~size_t(255); };
    l.ckpt = round((size_t)(f.B * f.H) * nchunks * f.dv * f.dk * 4);
    l.acc = f.dtype != GDN_F32 ? round(2 * (size_t)ntok * f.dk * 4) : 0;
    l.nseg = 1;
    l.fwd_ws = l.fwd_out = 0;
    if (tc_recompute(f)) {
        l.nseg = fwd_tc_segments(f, sm_count, true);
        l.fwd_ws = round(fwd_split_workspace_bytes(f, l.nseg));
        l.fwd_out = round((size_t)ntok * f.dv * 2);
    }
    l.total = l.ckpt + l.acc + l.fwd_ws + l.fwd_out;
    return l;
}

template <typename Tin>
cudaError_t launch_t(const BwdProblem &p, int sm_count, void *workspace, cudaStream_t stream) {
    const FwdProblem &f = p.f;
    const BwdDims d = plan(p, sm_count);
    const BwdLayout l = layout(p, sm_count);
    const size_t smem = d.smem_floats() * sizeof(float);
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    const int64_t ntok = f.B * f.T * f.H;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *ckpt = reinterpret_cast<float *>(ws);
    const bool f32 = f.dtype == GDN_F32;
    float *dq_acc = f32 ? static_cast<float *>(p.dq) : reinterpret_cast<float *>(ws + l.ckpt);
    float *dk_acc = f32 ? static_cast<float *>(p.dk) : dq_acc + ntok * f.dk;
    cudaError_t e;
    // forward recompute: the state entering every chunk
    FwdProblem fc = f;
    fc.out = nullptr;
    fc.S_final = nullptr;
    fc.ckpt = ckpt;
    fc.raw_inputs = 0;
    if (l.fwd_ws) {
        fc.out = ws + l.ckpt + l.acc + l.fwd_ws;
        if ((e = launch_fwd_split(fc, l.nseg, sm_count, ws + l.ckpt + l.acc, stream)) != cudaSuccess) return e;
    } else if ((e = launch_fwd_simt(fc, sm_count, stream)) != cudaSuccess) {
        return e;
    }
    if ((e = cudaMemsetAsync(dq_acc, 0, (size_t)ntok * f.dk * 4, stream)) != cudaSuccess ||
        (e = cudaMemsetAsync(dk_acc, 0, (size_t)ntok * f.dk * 4, stream)) != cudaSuccess ||
        (e = cudaMemsetAsync(p.dlog_alpha, 0, (size_t)ntok * 4, stream)) != cudaSuccess ||
        (e = cudaMemsetAsync(p.dbeta, 0, (size_t)ntok * 4, stream)) != cudaSuccess)
        return e;
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        if ((e = cudaFuncSetAttribute(bwd_simt_kernel<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      227 * 1024)) != cudaSuccess)
            return e;
        configured.fetch_or(bit);
    }
    {
        TimedLaunch tl_(GDN_KERNEL_BACKWARD, stream);
        bwd_simt_kernel<Tin><<<(unsigned)(f.B * f.H * d.nslab), kThreads, smem, stream>>>(
            static_cast<const Tin *>(f.q), static_cast<const Tin *>(f.k), static_cast<const Tin *>(f.v), f.log_alpha,
            f.beta, ckpt, static_cast<const Tin *>(p.d_out), p.dS_final, dq_acc, dk_acc, static_cast<Tin *>(p.dv),
            p.dlog_alpha, p.dbeta, p.dS0, f.T, f.H, d);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (!f32) {
        const int64_t n4 = ntok * f.dk / 4;
        const unsigned grid = (unsigned)(n4 / 256 + 1 < (int64_t)sm_count * 8 ? n4 / 256 + 1 : (int64_t)sm_count * 8);
        {
            TimedLaunch tl_(GDN_KERNEL_BACKWARD, stream);
            cast_bf16_kernel<<<grid, 256, 0, stream>>>(dq_acc, static_cast<__nv_bfloat16 *>(p.dq), n4);
        }
        {
            TimedLaunch tl_(GDN_KERNEL_BACKWARD, stream);
            cast_bf16_kernel<<<grid, 256, 0, stream>>>(dk_acc, static_cast<__nv_bfloat16 *>(p.dk), n4);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

size_t bwd_simt_workspace_bytes(const BwdProblem &p, int sm_count) { return layout(p, sm_count).total; }

cudaError_t launch_bwd_simt(const BwdProblem &p, int sm_count, void *workspace, cudaStream_t stream) {
    if (p.f.B * p.f.H == 0 || p.f.T == 0) return cudaSuccess;
    if (p.f.dtype == GDN_F32) return launch_t<float>(p, sm_count, workspace, stream);
    return launch_t<__nv_bfloat16>(p, sm_count, workspace, stream);
}

}  // namespace gdn
