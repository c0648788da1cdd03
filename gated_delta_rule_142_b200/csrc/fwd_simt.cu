// fwd_simt.cu -- chunkwise gated-delta forward in float32 on the CUDA cores.
//
// This is the float32-exact path (dtype GDN_F32) and the path for every
// (dk, dv, chunk) that the tensor-core kernel does not cover.  It computes the
// Sec. 3.3 recurrence of "ATMA: Long-Context Language Modeling via Polar
// Attention and Gated-Delta Compression Memory" chunk by chunk.  Inside a
// chunk of C tokens with entry state S (chunk-local log-decay cumsum g_t,
// gamma_t = e^{g_t}), writing S_t = alpha_t S_{t-1} + u_t k_t^T with
// u_t = beta_t (v_t - alpha_t S_{t-1} k_t) gives
//     (I + A) U = diag(beta) X,   X = V - diag(gamma) K S^T,
//     A_ts = beta_t e^{g_t - g_s} (k_t . k_s) for s < t,
//     O    = diag(gamma) Q S^T + [ (Q K^T) o e^{g_t - g_s} ]_{s<=t} U,
//     S'   = gamma_C S + U^T diag(e^{g_C - g_s}) K,
// the chunkwise (UT-transform) form used by the works the paper cites for
// this memory ("Gated delta networks"; "Parallelizing linear transformers
// with the delta rule over sequence length").  Here the unit-lower-triangular
// system is solved for U directly by forward substitution, in float32.
//
// One CTA owns one (b, h) and a slab of `rows` state rows (value dims); it
// walks the chunks in order with its state slab resident in shared memory.
// Rows of the state evolve independently given the chunk's keys, so slabs of
// one head run in parallel (each recomputes the slab-independent A and P).
// Tail chunks are zero-padded with log_alpha = 0, beta = 0, which leaves the
// recurrence unchanged.
//
// Grouped heads (group > 1): q and out have H heads, k, v and the gates H / group;
// query head h reads the memory of key-value head h / group, which each of the
// group's CTAs recomputes (S0 / S_final are per query head here; the caller
// expands and picks them).
//
// For the backward pass the same kernel recomputes the forward with outputs
// off (out == nullptr) and writes the state at the start of every chunk to a
// checkpoint array [B*H][chunks][dv][dk].
#include <atomic>

#include "common.cuh"
#include "gdn.h"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kThreads = 256;

struct SimtDims {
    int dk, dv, C, rows, nslab;
    int ldk, ldr, ldc;
    size_t smem_floats() const {
        return (size_t)rows * ldk + 2 * (size_t)C * ldk + 2 * (size_t)C * ldr + (size_t)C * ldc + 4 * (size_t)C;
    }
};

// acc[a][b] += sum_c X[(i0+a)*ldx + c] * Y[(j0+b)*ldy + c],  c in [0, K)
__device__ __forceinline__ void tile_nt(const float *X, int ldx, const float *Y, int ldy, int i0, int j0,
                                        int K, float acc[4][4]) {
    for (int c = 0; c < K; c += 4) {
        float4 x[4], y[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) x[a] = *reinterpret_cast<const float4 *>(X + (i0 + a) * ldx + c);
#pragma unroll
        for (int b = 0; b < 4; ++b) y[b] = *reinterpret_cast<const float4 *>(Y + (j0 + b) * ldy + c);
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] += dot4(x[a], y[b]);
    }
}

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
fwd_simt_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                const float *__restrict__ log_alpha, const float *__restrict__ beta,
                const float *__restrict__ S0, Tin *__restrict__ out, float *__restrict__ S_final,
                float *__restrict__ ckpt, int64_t T, int64_t H, int group, SimtDims d) {
    extern __shared__ __align__(16) float sm[];
    const int dk = d.dk, dv = d.dv, C = d.C, rows = d.rows;
    const int LDK = d.ldk, LDR = d.ldr, LDC = d.ldc;
    float *Ss = sm;                  // rows x LDK  state slab
    float *Qs = Ss + rows * LDK;     // C x LDK
    float *Ks = Qs + C * LDK;        // C x LDK
    float *Xs = Ks + C * LDK;        // C x LDR     V slab, then X, then Q S^T
    float *Us = Xs + C * LDR;        // C x LDR
    float *Ps = Us + C * LDR;        // C x LDC     A, then masked decayed Q K^T
    float *g = Ps + C * LDC;         // C
    float *bet = g + C;              // C
    float *gam = bet + C;            // C  e^{g_t}
    float *dl = gam + C;             // C  e^{g_last - g_s}

    const int tid = threadIdx.x;
    const int64_t bh = blockIdx.x / d.nslab;
    const int slab = blockIdx.x % d.nslab;
    const int64_t b = bh / H, h = bh % H;
    const int r0 = slab * rows;
    const int64_t Hkv = H / group, hk = h / group;  // key-value heads; this query head's
    const int64_t tok_stride_q = H * dk, tok_stride_k = Hkv * dk, tok_stride_v = Hkv * dv, tok_stride_o = H * dv;
    const Tin *qb = q + (b * T * H + h) * dk;
    const Tin *kb = k + (b * T * Hkv + hk) * dk;
    const Tin *vb = v + (b * T * Hkv + hk) * dv + r0;
    Tin *ob = out + (b * T * H + h) * dv + r0;
    const float *lab = log_alpha + b * T * Hkv + hk;
    const float *beb = beta + b * T * Hkv + hk;

    // state slab <- S0 (or zero)
    for (int i = tid; i < rows * (dk / 4); i += kThreads) {
        const int j = i / (dk / 4), c4 = i % (dk / 4);
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        if (S0) s = *reinterpret_cast<const float4 *>(S0 + (bh * dv + r0 + j) * (int64_t)dk + 4 * c4);
        *reinterpret_cast<float4 *>(Ss + j * LDK + 4 * c4) = s;
    }

    const int tpc = kThreads / rows;  // threads per column in the substitution
    const bool want_out = out != nullptr;
    const int64_t nchunks = (T + C - 1) / C;
    for (int64_t t0 = 0; t0 < T; t0 += C) {
        const int n = (int)((T - t0 < C) ? (T - t0) : C);
        __syncthreads();  // previous chunk fully consumed
        if (ckpt) {  // the state entering this chunk
            float *dst = ckpt + ((bh * nchunks + t0 / C) * dv + r0) * (int64_t)dk;
            for (int i = tid; i < rows * (dk / 4); i += kThreads) {
                const int j = i / (dk / 4), c4 = i % (dk / 4);
                *reinterpret_cast<float4 *>(dst + (int64_t)j * dk + 4 * c4) =
                    *reinterpret_cast<const float4 *>(Ss + j * LDK + 4 * c4);
            }
        }
        // ---- load chunk (zero-padded tail) ----
        for (int i = tid; i < C * (dk / 4); i += kThreads) {
            const int t = i / (dk / 4), c4 = i % (dk / 4);
            float4 qa = make_float4(0.f, 0.f, 0.f, 0.f), ka = qa;
            if (t < n) {
                qa = load4(qb + (t0 + t) * tok_stride_q + 4 * c4);
                ka = load4(kb + (t0 + t) * tok_stride_k + 4 * c4);
            }
            *reinterpret_cast<float4 *>(Qs + t * LDK + 4 * c4) = qa;
            *reinterpret_cast<float4 *>(Ks + t * LDK + 4 * c4) = ka;
        }
        for (int i = tid; i < C * (rows / 4); i += kThreads) {
            const int t = i / (rows / 4), c4 = i % (rows / 4);
            float4 va = make_float4(0.f, 0.f, 0.f, 0.f);
            if (t < n) va = load4(vb + (t0 + t) * tok_stride_v + 4 * c4);
            *reinterpret_cast<float4 *>(Xs + t * LDR + 4 * c4) = va;
        }
        if (tid < 32) {  // chunk-local inclusive cumsum of clamped log_alpha (C <= 64)
            float x0 = 0.f, x1 = 0.f;
            const int e0 = 2 * tid, e1 = 2 * tid + 1;
            if (e0 < n) x0 = fmaxf(lab[(t0 + e0) * Hkv], kLogAlphaFloor);
            if (e1 < n) x1 = fmaxf(lab[(t0 + e1) * Hkv], kLogAlphaFloor);
            float s = x0 + x1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, s, off);
                if (tid >= off) s += y;
            }
            if (e0 < C) g[e0] = s - x1;
            if (e1 < C) g[e1] = s;
        }
        for (int t = tid; t < C; t += kThreads) bet[t] = (t < n) ? beb[(t0 + t) * Hkv] : 0.f;
        __syncthreads();
        for (int t = tid; t < C; t += kThreads) {
            gam[t] = expf(g[t]);
            dl[t] = expf(g[C - 1] - g[t]);
        }
        __syncthreads();

        // ---- X = V - diag(gamma) K S^T ;  A = strict_lower(beta_t e^{g_t-g_s} K K^T) ----
        {
            const int nx = (C / 4) * (rows / 4), na = (C / 4) * (C / 4);
            for (int w = tid; w < nx + na; w += kThreads) {
                float acc[4][4] = {};
                if (w < nx) {
                    const int i0 = (w / (rows / 4)) * 4, j0 = (w % (rows / 4)) * 4;
                    tile_nt(Ks, LDK, Ss, LDK, i0, j0, dk, acc);
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int bb = 0; bb < 4; ++bb) Xs[(i0 + a) * LDR + j0 + bb] -= gam[i0 + a] * acc[a][bb];
                } else {
                    const int ww = w - nx;
                    const int i0 = (ww / (C / 4)) * 4, j0 = (ww % (C / 4)) * 4;
                    if (j0 <= i0 + 3) tile_nt(Ks, LDK, Ks, LDK, i0, j0, dk, acc);
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int bb = 0; bb < 4; ++bb) {
                            const int t = i0 + a, s = j0 + bb;
                            Ps[t * LDC + s] = (s < t) ? bet[t] * expf(g[t] - g[s]) * acc[a][bb] : 0.f;
                        }
                }
            }
        }
        __syncthreads();

        // ---- U: forward substitution  U_t = beta_t X_t - sum_{s<t} A_ts U_s ----
        {
            const int j = tid / tpc, part = tid % tpc;
            for (int t = 0; t < C; ++t) {
                float acc = 0.f;
                for (int s = part; s < t; s += tpc) acc += Ps[t * LDC + s] * Us[s * LDR + j];
                for (int off = tpc / 2; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
                if (part == 0) Us[t * LDR + j] = bet[t] * Xs[t * LDR + j] - acc;
                __syncthreads();
            }
        }

        // ---- P = mask_{s<=t}(Q K^T o e^{g_t-g_s}) ;  Xs <- diag(gamma) Q S^T ----
        if (want_out) {
            const int nx = (C / 4) * (rows / 4), na = (C / 4) * (C / 4);
            for (int w = tid; w < nx + na; w += kThreads) {
                float acc[4][4] = {};
                if (w < nx) {
                    const int i0 = (w / (rows / 4)) * 4, j0 = (w % (rows / 4)) * 4;
                    tile_nt(Qs, LDK, Ss, LDK, i0, j0, dk, acc);
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int bb = 0; bb < 4; ++bb) Xs[(i0 + a) * LDR + j0 + bb] = gam[i0 + a] * acc[a][bb];
                } else {
                    const int ww = w - nx;
                    const int i0 = (ww / (C / 4)) * 4, j0 = (ww % (C / 4)) * 4;
                    if (j0 <= i0 + 3) tile_nt(Qs, LDK, Ks, LDK, i0, j0, dk, acc);
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int bb = 0; bb < 4; ++bb) {
                            const int t = i0 + a, s = j0 + bb;
                            Ps[t * LDC + s] = (s <= t) ? expf(g[t] - g[s]) * acc[a][bb] : 0.f;
                        }
                }
            }
        }
        __syncthreads();

        // ---- O = Xs + P U  (to global) ;  S <- gamma_last S + U^T diag(dl) K ----
        {
            const int no = want_out ? (C / 4) * (rows / 4) : 0, ns = (rows / 4) * (dk / 4);
            const float gl = gam[C - 1];
            for (int w = tid; w < no + ns; w += kThreads) {
                float acc[4][4] = {};
                if (w < no) {
                    const int i0 = (w / (rows / 4)) * 4, j0 = (w % (rows / 4)) * 4;
                    for (int s = 0; s <= i0 + 3; ++s) {
                        const float4 u = *reinterpret_cast<const float4 *>(Us + s * LDR + j0);
#pragma unroll
                        for (int a = 0; a < 4; ++a) {
                            const float p = Ps[(i0 + a) * LDC + s];
                            acc[a][0] += p * u.x;
                            acc[a][1] += p * u.y;
                            acc[a][2] += p * u.z;
                            acc[a][3] += p * u.w;
                        }
                    }
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        const int t = i0 + a;
                        if (t < n) {
                            const float *x = Xs + t * LDR + j0;
                            store4<Tin>(ob + (t0 + t) * tok_stride_o + j0, x[0] + acc[a][0], x[1] + acc[a][1],
                                        x[2] + acc[a][2], x[3] + acc[a][3]);
                        }
                    }
                } else {
                    const int ww = w - no;
                    const int j0 = (ww / (dk / 4)) * 4, c0 = (ww % (dk / 4)) * 4;
                    for (int s = 0; s < C; ++s) {
                        const float4 u = *reinterpret_cast<const float4 *>(Us + s * LDR + j0);
                        float4 kk = *reinterpret_cast<const float4 *>(Ks + s * LDK + c0);
                        const float f = dl[s];
                        kk.x *= f; kk.y *= f; kk.z *= f; kk.w *= f;
                        const float uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                        for (int a = 0; a < 4; ++a) {
                            acc[a][0] += uu[a] * kk.x;
                            acc[a][1] += uu[a] * kk.y;
                            acc[a][2] += uu[a] * kk.z;
                            acc[a][3] += uu[a] * kk.w;
                        }
                    }
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        float4 *sp = reinterpret_cast<float4 *>(Ss + (j0 + a) * LDK + c0);
                        float4 s = *sp;
                        s.x = fmaf(gl, s.x, acc[a][0]);
                        s.y = fmaf(gl, s.y, acc[a][1]);
                        s.z = fmaf(gl, s.z, acc[a][2]);
                        s.w = fmaf(gl, s.w, acc[a][3]);
                        *sp = s;
                    }
                }
            }
        }
    }
    __syncthreads();
    if (S_final) {
        for (int i = tid; i < rows * (dk / 4); i += kThreads) {
            const int j = i / (dk / 4), c4 = i % (dk / 4);
            *reinterpret_cast<float4 *>(S_final + (bh * dv + r0 + j) * (int64_t)dk + 4 * c4) =
                *reinterpret_cast<const float4 *>(Ss + j * LDK + 4 * c4);
        }
    }
}

template <typename Tin>
cudaError_t launch_t(const FwdProblem &p, int sm_count, cudaStream_t stream) {
    SimtDims d;
    d.dk = (int)p.dk;
    d.dv = (int)p.dv;
    d.C = (int)p.chunk;
    int nslab = 1;
    const int64_t heads = p.B * p.H;
    while (heads * nslab < sm_count && p.dv / (nslab * 2) >= 16 && nslab < 8) nslab *= 2;
    d.nslab = nslab;
    d.rows = d.dv / nslab;
    d.ldk = d.dk + 4;
    d.ldr = d.rows + 4;
    d.ldc = d.C + 4;
    const size_t smem = d.smem_floats() * sizeof(float);
    static std::atomic<uint64_t> configured{0};  // one bit per device: smem opt-in done
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(fwd_simt_kernel<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             227 * 1024);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit);
    }
    const int64_t grid = heads * nslab;
    {
        TimedLaunch tl_(GDN_KERNEL_SIMT, stream);
        fwd_simt_kernel<Tin><<<(unsigned)grid, kThreads, smem, stream>>>(
            static_cast<const Tin *>(p.q), static_cast<const Tin *>(p.k), static_cast<const Tin *>(p.v), p.log_alpha,
            p.beta, p.S0, static_cast<Tin *>(p.out), p.S_final, p.ckpt, p.T, p.H, p.group, d);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_simt(const FwdProblem &p, int sm_count, cudaStream_t stream) {
    if (p.dtype == 0) return launch_t<float>(p, sm_count, stream);
    return launch_t<__nv_bfloat16>(p, sm_count, stream);
}

}  // namespace gdn
