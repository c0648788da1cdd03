// fwd_tc.cu -- chunkwise gated-delta forward on the 5th-generation tensor
// cores (tcgen05) for bf16 q/k/v with dk = dv = 128 and chunk C = 64.
//
// Operation: "ATMA: Long-Context Language Modeling via Polar Attention and
// Gated-Delta Compression Memory", Sec. 3.3 (gated-delta memory equation),
// computed in the chunkwise UT-transform form of the works that paper cites
// for the memory ("Gated delta networks"; "Parallelizing linear transformers
// with the delta rule over sequence length").  Per chunk of 64 tokens with
// entry state S (dv x dk, float32), chunk-local log-decay cumsum g_t and
// gamma_t = e^{g_t}:
//     G   = [Q; K] K^T                                        (tcgen05, M=128)
//     A   = strict_lower(beta_t e^{g_t-g_s} (K K^T)_ts)
//     P   = lower(e^{g_t-g_s} (Q K^T)_ts)        (diagonal included)
//     T   = (I + A)^{-1}                          (blocked substitution, fp32)
//     Ut^T = V^T (T diag(beta))^T,  W^T = K^T (T diag(beta gamma))^T   (tcgen05)
//     D   = S [W; diag(gamma) Q]^T                (tcgen05, A = bf16 S in TMEM)
//     U^T = Ut^T - D[:, :64]
//     O^T = D[:, 64:] + U^T P^T                   (tcgen05, A = bf16 U^T in TMEM)
//     S  <- gamma_C S + U^T Ktil,  Ktil_s = e^{g_C-g_s} k_s     (tcgen05, into S)
// S stays in tensor memory in float32 for the whole sequence; the bf16 copy
// used as an MMA operand is rewritten from it every chunk.
//
// Data movement: Q, K, V chunk tiles (64 tokens x 128, bf16) arrive by TMA
// (4-D tensor maps over [B, T, H, d], 128-byte swizzle, zero fill past T)
// into a double buffer; the next chunk's tiles load while this one computes.
// Shared-memory operand tiles use the canonical 128-byte-swizzled layouts
// (K-major: 8-row x 128-byte atoms; MN-major: 64-element x 8-row atoms).
//
// One CTA of 128 threads per (b, h); thread j owns TMEM lane j (state row j).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>

#include "gdn_internal.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kThreadsTc = 128;

// Shared memory map (bytes, from a 1024-aligned base).
constexpr uint32_t OFF_QK = 0;            // 2 x 32 KB: per 64-column block j: [Q 8 KB | K 8 KB]
constexpr uint32_t QK_BYTES = 32768;
constexpr uint32_t OFF_V = 65536;         // 2 x 16 KB: per 64-column block j: V 8 KB
constexpr uint32_t V_BYTES = 16384;
constexpr uint32_t OFF_P = 98304;         // 8 KB   P      [t][s] K-major
constexpr uint32_t OFF_TB = 106496;       // 8 KB   T diag(beta)       [t][s] K-major
constexpr uint32_t OFF_TBG = 114688;      // 8 KB   T diag(beta gamma) [t][s] K-major
constexpr uint32_t OFF_W = 122880;        // 16 KB  W stored MN-major: row i (key dim), 64 t per row
constexpr int LDM = 68;                   // row stride (floats) of the fp32 64x64 tiles: conflict-free rows
constexpr uint32_t OFF_AM = 139264;       // 17 KB  A  fp32 [64][LDM]
constexpr uint32_t OFF_TM = 156672;       // 17 KB  T  fp32 [64][LDM]
constexpr uint32_t OFF_Y = 174080;        // 3 KB   block-substitution scratch
constexpr uint32_t OFF_GATES = 177152;    // 1.5 KB g, beta, gamma, decay-to-end, e^{g-c}, e^{c-g}
constexpr uint32_t OFF_BARS = 178688;     // mbarriers: full[2], mma
constexpr uint32_t OFF_MISC = 178752;     // tmem base slot, scan scratch
constexpr uint32_t SMEM_TC = 178816 + 1024;
constexpr uint32_t OFF_OST = OFF_P;       // output staging [64][136] bf16 (reuses P/T/W tiles)
constexpr int LDO = 136;
constexpr uint32_t kTxBytes = 3 * 2 * 8192;  // Q, K, V: two 8 KB boxes each

// TMEM column map (512 columns allocated).
constexpr uint32_t TM_S = 0;      // 128 cols  S float32 (row j in lane j)
constexpr uint32_t TM_D1 = 128;   // 128 cols  [S W^T | O^T]
constexpr uint32_t TM_G = 256;    // 64 cols   [Q;K] K^T, later W^T
constexpr uint32_t TM_UT = 320;   // 64 cols   Ut^T
constexpr uint32_t TM_SB = 384;   // 64 cols   bf16 S (A operand, 2 per column)
constexpr uint32_t TM_UB = 448;   // 32 cols   bf16 U^T (A operand)

constexpr uint32_t IDESC_G = instr_desc_bf16(128, 64, 0, 0);    // [Q;K] . K^T
constexpr uint32_t IDESC_MN64 = instr_desc_bf16(128, 64, 1, 0); // V^T / K^T (MN-major A) . T^T
constexpr uint32_t IDESC_W = instr_desc_bf16(128, 64, 0, 1);    // S . W^T  (W stored MN-major)
constexpr uint32_t IDESC_Q = instr_desc_bf16(128, 64, 0, 0);    // S . Qg^T, U^T . P^T
constexpr uint32_t IDESC_S = instr_desc_bf16(128, 128, 0, 1);   // U^T . Ktil (MN-major B)

__device__ int g_tc_timeout;  // set when a bounded mbarrier wait gives up

#ifdef GDN_TC_DEBUG
// Debug builds only: intermediate values of chunk 0 of CTA 0, for diagnosing
// the tensor-core stages (layout: G 128x64, A 64x64, T 64x64, Ut^T 128x64,
// W^T 128x64, D 128x128, O^T 128x64, S 128x128, all float32 row-major).
__device__ float *g_dbg;
#define DBG_ON (g_dbg != nullptr && blockIdx.x == 0 && c == 0)
// per-phase clock stamps of CTA 0, chunks 0..7 (int64 at float offset 73728, 16 per chunk)
#define DBG_CLK(i)                                                                     \
    if (g_dbg != nullptr && blockIdx.x == 0 && tid == 0 && c < 8)                      \
        reinterpret_cast<long long *>(g_dbg + 73728)[c * 16 + (i)] = clock64();
__device__ __forceinline__ void dbg_tmem_rows(uint32_t taddr, int ncols, float *dst) {
    for (int q = 0; q < ncols; q += 32) {
        uint32_t r[32];
        tmem_ld32(taddr + q, r);
        tmem_wait_ld();
        for (int i = 0; i < 32; ++i) dst[q + i] = __uint_as_float(r[i]);
    }
}
#else
#define DBG_CLK(i)
#endif

struct TcArgs {
    const float *log_alpha, *beta, *S0;
    __nv_bfloat16 *out;
    float *S_final;
    int64_t T, H;
};

// Byte offset of 16-byte chunk `c` of row `r` in a 128-byte-swizzled tile
// whose rows are 128 bytes (8-row, 1024-byte atoms).
__device__ __forceinline__ uint32_t sw128(uint32_t r, uint32_t c) {
    return (r >> 3) * 1024u + (r & 7u) * 128u + ((c ^ (r & 7u)) << 4);
}

__device__ __forceinline__ void scale_row_bf16(uint8_t *row, float f) {
    uint4 *p = reinterpret_cast<uint4 *>(row);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4 u = p[c];
        uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&w[i]);
            float2 x = __bfloat1622float2(v);
            w[i] = pack_bf16x2(x.x * f, x.y * f);
        }
        p[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

__global__ void __launch_bounds__(kThreadsTc, 1)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, TcArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *Am = reinterpret_cast<float *>(sm + OFF_AM);
    float *Tm = reinterpret_cast<float *>(sm + OFF_TM);
    float *Y = reinterpret_cast<float *>(sm + OFF_Y);
    float *g = reinterpret_cast<float *>(sm + OFF_GATES);
    float *bet = g + 64;
    float *gam = g + 128;
    float *dl = g + 192;
    float *ea = g + 256;  // e^{g_t - c}
    float *eb = g + 320;  // e^{c - g_s}
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + OFF_BARS);
    uint64_t *mma_bar = full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    float *scan_tmp = reinterpret_cast<float *>(sm + OFF_MISC + 16);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t T = p.T, H = p.H;
    const int64_t bh = blockIdx.x;
    const int b = (int)(bh / H), h = (int)(bh % H);
    const int64_t nchunks = (T + kC - 1) / kC;
    const uint32_t sbase = smem_u32(sm);

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(mma_bar, 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;
    const uint32_t lb = (uint32_t)(warp * 32) << 16;  // this warp's TMEM lane base

    auto issue_loads = [&](int64_t c, int buf) {
        const int t0 = (int)(c * kC);
        mbar_arrive_expect_tx(&full[buf], kTxBytes);
        uint8_t *qk = sm + OFF_QK + buf * QK_BYTES;
        uint8_t *vv = sm + OFF_V + buf * V_BYTES;
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
            tma_load_4d(qk + blk * 16384, &tm_q, &full[buf], blk * 64, h, t0, b);
            tma_load_4d(qk + blk * 16384 + 8192, &tm_k, &full[buf], blk * 64, h, t0, b);
            tma_load_4d(vv + blk * 8192, &tm_v, &full[buf], blk * 64, h, t0, b);
        }
    };
    if (tid == 0 && nchunks > 0) issue_loads(0, 0);

    // S0 -> TMEM (row j = tid)
    {
        const float *src = p.S0 ? p.S0 + (bh * kD + tid) * (int64_t)kD : nullptr;
#pragma unroll
        for (int piece = 0; piece < 4; ++piece) {
            uint32_t r[32];
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                float4 v = src ? *reinterpret_cast<const float4 *>(src + piece * 32 + i) : make_float4(0, 0, 0, 0);
                r[i] = __float_as_uint(v.x);
                r[i + 1] = __float_as_uint(v.y);
                r[i + 2] = __float_as_uint(v.z);
                r[i + 3] = __float_as_uint(v.w);
            }
            tmem_st32(tm + lb + TM_S + piece * 32, r);
        }
        tmem_wait_st();
    }

    uint32_t full_phase[2] = {0u, 0u};
    uint32_t mma_phase = 0u;
    bool ok = true;

    for (int64_t c = 0; c < nchunks && ok; ++c) {
        const int buf = (int)(c & 1);
        const int64_t t0 = c * kC;
        const int n = (int)((T - t0 < kC) ? (T - t0) : kC);
        const uint32_t qk = sbase + OFF_QK + buf * QK_BYTES;
        const uint32_t vv = sbase + OFF_V + buf * V_BYTES;
        uint8_t *qk_ptr = sm + OFF_QK + buf * QK_BYTES;

        if (tid == 0 && c + 1 < nchunks) issue_loads(c + 1, buf ^ 1);
        DBG_CLK(0)

        // ---- wait for this chunk's tiles; G = [Q;K] K^T ----
        DBG_CLK(1)
        bool w = mbar_wait(&full[buf], full_phase[buf]);
        full_phase[buf] ^= 1u;
        if (!__syncthreads_and(w)) { ok = false; break; }
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t a = qk + (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_ss(tm + TM_G, smem_desc_sw128(a, 16, 1024), smem_desc_sw128(a + 8192, 16, 1024), IDESC_G,
                       kk > 0);
            }
            mma_commit(mma_bar);
        }

        DBG_CLK(2)
        // ---- gates: g = cumsum(max(log_alpha, floor)), beta; zero past T ----
        if (tid < 64) {
            const int64_t gi = ((int64_t)b * T + t0 + tid) * H + h;
            const float x = (tid < n) ? fmaxf(p.log_alpha[gi], kLogAlphaFloor) : 0.f;
            bet[tid] = (tid < n) ? p.beta[gi] : 0.f;
            float s = x;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, s, off);
                if (lane >= off) s += y;
            }
            if (tid == 31) scan_tmp[0] = s;
            g[tid] = s;
        }
        __syncthreads();
        if (tid >= 32 && tid < 64) g[tid] += scan_tmp[0];
        __syncthreads();
        // e^{g_t - g_s} = e^{g_t - c} e^{c - g_s} with c = g_31, exact to a few ulp while every
        // |g_t - c| < 80; a chunk with a wider decay span uses expf(g_t - g_s) per element.
        bool narrow = true;
        if (tid < 64) {
            const float gt = g[tid], cm = g[31];
            gam[tid] = expf(gt);
            dl[tid] = expf(g[63] - gt);
            ea[tid] = expf(gt - cm);
            eb[tid] = expf(cm - gt);
            narrow = fabsf(gt - cm) < 80.f;
        }
        DBG_CLK(3)
        w = mbar_wait(mma_bar, mma_phase);
        mma_phase ^= 1u;
        narrow = __syncthreads_and(narrow);
        if (!__syncthreads_and(w)) { ok = false; break; }
        tc_fence_after();

        DBG_CLK(4)
#ifdef GDN_TC_DEBUG
        if (DBG_ON) dbg_tmem_rows(tm + lb + TM_G, 64, g_dbg + tid * 64);
#endif
        // ---- epilogue of G: P (bf16 tile) from the Q rows, A (fp32) from the K rows; Q <- gamma Q ----
        {
            const int t = tid & 63;
            const float gt = g[t], at = ea[t];
            if (tid < 64) {
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r[32];
                    tmem_ld32(tm + lb + TM_G + half * 32, r);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        const int s = half * 32 + i;
                        const float d0 = narrow ? at * eb[s] : expf(gt - g[s]);
                        const float d1 = narrow ? at * eb[s + 1] : expf(gt - g[s + 1]);
                        const float v0 = (s <= t) ? __uint_as_float(r[i]) * d0 : 0.f;
                        const float v1 = (s + 1 <= t) ? __uint_as_float(r[i + 1]) * d1 : 0.f;
                        pk[i >> 1] = pack_bf16x2(v0, v1);
                    }
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
                        *reinterpret_cast<uint4 *>(sm + OFF_P + sw128(t, half * 4 + cc)) =
                            make_uint4(pk[cc * 4], pk[cc * 4 + 1], pk[cc * 4 + 2], pk[cc * 4 + 3]);
                }
                const float gm = gam[t];
                scale_row_bf16(qk_ptr + t * 128, gm);
                scale_row_bf16(qk_ptr + 16384 + t * 128, gm);
            } else {
                const float bt = bet[t];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r[32];
                    tmem_ld32(tm + lb + TM_G + half * 32, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        float v[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int s = half * 32 + i + e;
                            const float dd = narrow ? at * eb[s] : expf(gt - g[s]);
                            v[e] = (s < t) ? bt * dd * __uint_as_float(r[i + e]) : 0.f;
                        }
                        *reinterpret_cast<float4 *>(Am + t * LDM + half * 32 + i) = make_float4(v[0], v[1], v[2], v[3]);
                    }
                }
            }
        }
        __syncthreads();

        DBG_CLK(5)
        // ---- T = (I + A)^{-1}: 16x16 diagonal blocks by substitution (one warp each, a column per lane) ----
        if (lane < 16) {
            const int o = warp * 16;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = (r == lane) ? 1.f : 0.f;
#pragma unroll
                for (int s = 0; s < r; ++s) acc -= Am[(o + r) * LDM + o + s] * x[s];
                x[r] = acc;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) Tm[(o + r) * LDM + o + lane] = x[r];
        }
        __syncthreads();
        DBG_CLK(6)
        // block rows I = 1..3:  T_IJ = -T_II sum_{K=J}^{I-1} A_IK T_KJ ; one thread per (J, row, 4 columns)
        for (int I = 1; I < 4; ++I) {
            for (int e = tid; e < I * 64; e += kThreadsTc) {
                const int J = e >> 6, r = (e >> 2) & 15, c4 = (e & 3) * 4;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int K = J; K < I; ++K) {
                    const float *arow = Am + (16 * I + r) * LDM + 16 * K;
                    const float *tcol = Tm + (16 * K) * LDM + 16 * J + c4;
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        const float a = arow[m];
                        const float4 tv = *reinterpret_cast<const float4 *>(tcol + m * LDM);
                        acc.x = fmaf(a, tv.x, acc.x);
                        acc.y = fmaf(a, tv.y, acc.y);
                        acc.z = fmaf(a, tv.z, acc.z);
                        acc.w = fmaf(a, tv.w, acc.w);
                    }
                }
                *reinterpret_cast<float4 *>(Y + J * 256 + r * 16 + c4) = acc;
            }
            __syncthreads();
            for (int e = tid; e < I * 64; e += kThreadsTc) {
                const int J = e >> 6, r = (e >> 2) & 15, c4 = (e & 3) * 4;
                const float *trow = Tm + (16 * I + r) * LDM + 16 * I;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float a = trow[m];
                    const float4 y = *reinterpret_cast<const float4 *>(Y + J * 256 + m * 16 + c4);
                    acc.x = fmaf(a, y.x, acc.x);
                    acc.y = fmaf(a, y.y, acc.y);
                    acc.z = fmaf(a, y.z, acc.z);
                    acc.w = fmaf(a, y.w, acc.w);
                }
                *reinterpret_cast<float4 *>(Tm + (16 * I + r) * LDM + 16 * J + c4) =
                    make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
            }
            __syncthreads();
        }
        DBG_CLK(7)
#ifdef GDN_TC_DEBUG
        if (DBG_ON)
            for (int e = tid; e < 4096; e += kThreadsTc) {
                g_dbg[8192 + e] = Am[(e >> 6) * LDM + (e & 63)];
                g_dbg[12288 + e] = ((e & 63) <= (e >> 6)) ? Tm[(e >> 6) * LDM + (e & 63)] : 0.f;
            }
#endif
        // T diag(beta) (threads 0..63) and T diag(beta gamma) (threads 64..127), bf16, lower triangle
        {
            const int t = tid & 63;
            const bool with_gamma = tid >= 64;
            uint8_t *dst = sm + (with_gamma ? OFF_TBG : OFF_TB);
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                uint32_t pk[4];
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                    const int s = cc * 8 + i;
                    float v0 = (s <= t) ? Tm[t * LDM + s] * bet[s] : 0.f;
                    float v1 = (s + 1 <= t) ? Tm[t * LDM + s + 1] * bet[s + 1] : 0.f;
                    if (with_gamma) {
                        v0 *= gam[s];
                        v1 *= gam[s + 1];
                    }
                    pk[i >> 1] = pack_bf16x2(v0, v1);
                }
                *reinterpret_cast<uint4 *>(dst + sw128(t, cc)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        DBG_CLK(8)
        // ---- Ut^T = V^T (T beta)^T ;  W^T = K^T (T beta gamma)^T ----
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t bdesc = smem_desc_sw128(sbase + OFF_TB + kk * 32, 16, 1024);
                mma_ss(tm + TM_UT, smem_desc_sw128(vv + kk * 2048, 8192, 1024), bdesc, IDESC_MN64, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t bdesc = smem_desc_sw128(sbase + OFF_TBG + kk * 32, 16, 1024);
                mma_ss(tm + TM_G, smem_desc_sw128(qk + 8192 + kk * 2048, 16384, 1024), bdesc, IDESC_MN64, kk > 0);
            }
            mma_commit(mma_bar);
        }

        DBG_CLK(9)
        // ---- meanwhile: S -> bf16 operand copy; S <- gamma_C S (float32, in TMEM) ----
        {
            const float gC = gam[63];
#pragma unroll
            for (int piece = 0; piece < 4; ++piece) {
                uint32_t r[32];
                tmem_ld32(tm + lb + TM_S + piece * 32, r);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) pk[i >> 1] = pack_bf16x2(__uint_as_float(r[i]), __uint_as_float(r[i + 1]));
                tmem_st16(tm + lb + TM_SB + piece * 16, pk);
#pragma unroll
                for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * gC);
                tmem_st32(tm + lb + TM_S + piece * 32, r);
            }
            tmem_wait_st();
        }
        DBG_CLK(10)
        w = mbar_wait(mma_bar, mma_phase);
        mma_phase ^= 1u;
        if (!__syncthreads_and(w)) { ok = false; break; }
        tc_fence_after();

#ifdef GDN_TC_DEBUG
        if (DBG_ON) {
            dbg_tmem_rows(tm + lb + TM_UT, 64, g_dbg + 16384 + tid * 64);
            dbg_tmem_rows(tm + lb + TM_G, 64, g_dbg + 24576 + tid * 64);
        }
#endif
        // ---- W (bf16, MN-major rows i) from W^T in TMEM;  K <- Ktil = e^{g_C - g_s} K ----
        {
            const int i = tid;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t r[32];
                tmem_ld32(tm + lb + TM_G + half * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(r[cc * 8 + 0]), __uint_as_float(r[cc * 8 + 1]));
                    v.y = pack_bf16x2(__uint_as_float(r[cc * 8 + 2]), __uint_as_float(r[cc * 8 + 3]));
                    v.z = pack_bf16x2(__uint_as_float(r[cc * 8 + 4]), __uint_as_float(r[cc * 8 + 5]));
                    v.w = pack_bf16x2(__uint_as_float(r[cc * 8 + 6]), __uint_as_float(r[cc * 8 + 7]));
                    *reinterpret_cast<uint4 *>(sm + OFF_W + sw128(i, half * 4 + cc)) = v;
                }
            }
            const int s = tid & 63, blk = tid >> 6;
            scale_row_bf16(qk_ptr + blk * 16384 + 8192 + s * 128, dl[s]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        DBG_CLK(11)
        // ---- D = S [W; gamma Q]^T  (A = bf16 S from TMEM) ----
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_ts(tm + TM_D1, tm + TM_SB + kk * 8, smem_desc_sw128(sbase + OFF_W + kk * 2048, 8192, 1024),
                       IDESC_W, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_ts(tm + TM_D1 + 64, tm + TM_SB + kk * 8,
                       smem_desc_sw128(qk + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024), IDESC_Q, kk > 0);
            mma_commit(mma_bar);
        }
        w = mbar_wait(mma_bar, mma_phase);
        mma_phase ^= 1u;
        if (!__syncthreads_and(w)) { ok = false; break; }
        tc_fence_after();

#ifdef GDN_TC_DEBUG
        if (DBG_ON) dbg_tmem_rows(tm + lb + TM_D1, 128, g_dbg + 32768 + tid * 128);
#endif
        DBG_CLK(12)
        // ---- U^T = Ut^T - S W^T  -> bf16 A operand in TMEM ----
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            uint32_t d[32], u[32];
            tmem_ld32(tm + lb + TM_D1 + half * 32, d);
            tmem_ld32(tm + lb + TM_UT + half * 32, u);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2)
                pk[i >> 1] = pack_bf16x2(__uint_as_float(u[i]) - __uint_as_float(d[i]),
                                         __uint_as_float(u[i + 1]) - __uint_as_float(d[i + 1]));
            tmem_st16(tm + lb + TM_UB + half * 16, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();

        DBG_CLK(13)
        // ---- O^T += U^T P^T ;  S += U^T Ktil ----
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_ts(tm + TM_D1 + 64, tm + TM_UB + kk * 8, smem_desc_sw128(sbase + OFF_P + kk * 32, 16, 1024),
                       IDESC_Q, 1);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_ts(tm + TM_S, tm + TM_UB + kk * 8, smem_desc_sw128(qk + 8192 + kk * 2048, 16384, 1024), IDESC_S,
                       1);
            mma_commit(mma_bar);
        }
        w = mbar_wait(mma_bar, mma_phase);
        mma_phase ^= 1u;
        if (!__syncthreads_and(w)) { ok = false; break; }
        tc_fence_after();

#ifdef GDN_TC_DEBUG
        if (DBG_ON) {
            dbg_tmem_rows(tm + lb + TM_D1 + 64, 64, g_dbg + 49152 + tid * 64);
            dbg_tmem_rows(tm + lb + TM_S, 128, g_dbg + 57344 + tid * 128);
        }
#endif
        DBG_CLK(14)
        // ---- outputs: thread j holds o[t][j]; stage [t][j] in shared memory, then coalesced rows ----
        {
            __nv_bfloat16 *ost = reinterpret_cast<__nv_bfloat16 *>(sm + OFF_OST);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t r[32];
                tmem_ld32(tm + lb + TM_D1 + 64 + half * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) ost[(half * 32 + i) * LDO + tid] = __float2bfloat16_rn(__uint_as_float(r[i]));
            }
            __syncthreads();
            __nv_bfloat16 *ob = p.out + (((int64_t)b * T + t0) * H + h) * kD;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int q = tid + k * kThreadsTc;  // 16-byte piece: row q / 16, column (q % 16) * 8
                const int t = q >> 4, c8 = (q & 15) * 8;
                if (t < n)
                    *reinterpret_cast<uint4 *>(ob + (int64_t)t * H * kD + c8) =
                        *reinterpret_cast<const uint4 *>(ost + t * LDO + c8);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        DBG_CLK(15)
    }

    if (!ok && tid == 0) atomicExch(&g_tc_timeout, 1);
    if (ok && p.S_final) {
        float *dst = p.S_final + (bh * kD + tid) * (int64_t)kD;
#pragma unroll
        for (int piece = 0; piece < 4; ++piece) {
            uint32_t r[32];
            tmem_ld32(tm + lb + TM_S + piece * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4 *>(dst + piece * 32 + i) =
                    make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]), __uint_as_float(r[i + 2]),
                                __uint_as_float(r[i + 3]));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 512);
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static std::atomic<EncodeTiledFn> fn{nullptr};
    EncodeTiledFn f = fn.load();
    if (!f) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !ptr) {
            cudaGetLastError();
            return nullptr;
        }
        f = reinterpret_cast<EncodeTiledFn>(ptr);
        fn.store(f);
    }
    return f;
}

// [B, T, H, 128] bf16 viewed as a 4-D tensor (d, h, t, b); box = 64 columns x 1 head x 64 tokens.
bool make_map(CUtensorMap *m, const void *base, int64_t B, int64_t T, int64_t H) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)(H * kD * 2), (cuuint64_t)(T * H * kD * 2)};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)kC, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

#ifdef GDN_TC_DEBUG
extern "C" int gdn_debug_set_dump(float *ptr) {
    return cudaMemcpyToSymbol(g_dbg, &ptr, sizeof(ptr)) == cudaSuccess ? 0 : 1;
}
#endif

bool fwd_tc_supported(const FwdProblem &p) {
    return p.dtype == 1 && p.dk == kD && p.dv == kD && p.chunk == kC && p.T <= (int64_t)INT32_MAX &&
           p.B <= (int64_t)INT32_MAX && p.H <= (int64_t)INT32_MAX;
}

cudaError_t launch_fwd_tc(const FwdProblem &p, cudaStream_t stream) {
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, p.q, p.B, p.T, p.H) || !make_map(&mk, p.k, p.B, p.T, p.H) ||
        !make_map(&mv, p.v, p.B, p.T, p.H))
        return cudaErrorInvalidValue;
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_TC);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit);
    }
    TcArgs a;
    a.log_alpha = p.log_alpha;
    a.beta = p.beta;
    a.S0 = p.S0;
    a.out = static_cast<__nv_bfloat16 *>(p.out);
    a.S_final = p.S_final;
    a.T = p.T;
    a.H = p.H;
    fwd_tc_kernel<<<(unsigned)(p.B * p.H), kThreadsTc, SMEM_TC, stream>>>(mq, mk, mv, a);
    return cudaGetLastError();
}

}  // namespace gdn
