// fwd_tc.cu -- chunkwise gated-delta forward on the 5th-generation tensor
// cores (tcgen05) for bf16 q/k/v with dk = dv = 128 and chunk C = 64.
//
// Operation: "ATMA: Long-Context Language Modeling via Polar Attention and
// Gated-Delta Compression Memory", Sec. 3.3 (gated-delta memory equation),
// computed in the chunkwise UT-transform form of the works that paper cites
// for the memory ("Gated delta networks"; "Parallelizing linear transformers
// with the delta rule over sequence length").  Per chunk of 64 tokens with
// entry state S (dv x dk, float32), chunk-local log-decay cumsum g_t,
// gamma_t = e^{g_t} and dl_s = e^{g_C - g_s}:
//   prep (independent of S):
//     G    = [Q; K] K^T                                   (tcgen05, M = 128)
//     A    = strict_lower(beta_t e^{g_t-g_s} (K K^T)_ts),  P = lower(e^{g_t-g_s} (Q K^T)_ts)
//     T    = (I + A)^{-1}                                  (blocked substitution, fp32)
//     Ut^T = V^T (T diag(beta))^T,  W^T = K^T (T diag(beta gamma))^T   (tcgen05)
//     Qg   = diag(gamma) Q
//   chain (needs S; sequential over chunks):
//     U^T  = Ut^T - S W^T                      (tcgen05 accumulate, B negated; A = bf16 S in TMEM)
//     O^T  = S Qg^T + U^T P^T                  (tcgen05; A = bf16 S, then bf16 U^T in TMEM)
//     S   <- gamma_C S + (U^T diag(dl)) K      (tcgen05 accumulate into the float32 state)
// The state S stays in tensor memory in float32 for the whole sequence; its
// bf16 operand copy is rewritten from it every chunk.
//
// Warp roles (512 threads):
//   warp 0      control: TMA loads (double-buffered Q/K/V tiles) and every
//               tcgen05.mma, issued by one thread in dependency order
//   warps 4-11  prep for chunk c+1 (256 threads) while the chain runs chunk c
//   warps 12-15 chain: state conversion, U^T epilogue, outputs (thread j owns
//               TMEM lane j, i.e. state row j)
//   warps 1-3   idle
// Roles hand work to each other through mbarriers (tcgen05.commit for MMA
// completion, single-thread arrivals after a named barrier otherwise).  Every
// wait is bounded; a wait that gives up sets an abort flag that makes every
// other wait return at once, so the CTA always reaches its exit, frees its
// tensor memory and records the timeout.
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
constexpr int kThreadsTc = 512;
constexpr int kPrepWarp0 = 4, kNumPrep = 256;
constexpr int kChainWarp0 = 12, kNumChain = 128;
constexpr int kBarPrep = 1, kBarChain = 2;  // named barrier ids (0 is __syncthreads)

// Shared memory map (bytes, from a 1024-aligned base).
constexpr uint32_t OFF_QK = 0;           // 2 x 32 KB: per 64-column block j: [Q 8 KB | K 8 KB]
constexpr uint32_t QK_BYTES = 32768;
constexpr uint32_t OFF_V = 65536;        // 2 x 16 KB: per 64-column block j: V 8 KB
constexpr uint32_t V_BYTES = 16384;
constexpr uint32_t OFF_P = 98304;        // 2 x 8 KB  P [t][s] K-major (per chunk parity)
constexpr uint32_t OFF_TB = 114688;      // 8 KB   T diag(beta)       [t][s] K-major
constexpr uint32_t OFF_TBG = 122880;     // 8 KB   T diag(beta gamma) [t][s] K-major
constexpr uint32_t OFF_W = 131072;       // 16 KB  W stored MN-major: row i (key dim), 64 t per row
constexpr int LDM = 68;                  // row stride (floats) of the fp32 64x64 tiles
constexpr uint32_t OFF_AM = 147456;      // 17 KB  A  fp32 [64][LDM]
constexpr uint32_t OFF_TM = 164864;      // 17 KB  T  fp32 [64][LDM]
constexpr uint32_t OFF_Y = 182272;       // 3 KB   block-substitution scratch
constexpr uint32_t OFF_PG = 185344;      // prep gates: g, beta, gamma, e^{g-c}, e^{c-g} (64 each)
constexpr uint32_t OFF_CG = 186624;      // chain gates: dl (64), scratch
constexpr uint32_t OFF_BARS = 187136;    // mbarriers
constexpr uint32_t OFF_MISC = 187264;    // tmem slot, abort flag, scan scratch
constexpr uint32_t SMEM_TC = 187328 + 1024;
constexpr uint32_t kTxBytes = 3 * 2 * 8192;  // Q, K, V: two 8 KB boxes each

// TMEM column map (512 columns).
constexpr uint32_t TM_S = 0;     // 128  S float32 (row j in lane j)
constexpr uint32_t TM_SB = 128;  // 64   bf16 S (A operand, 2 per column)
constexpr uint32_t TM_O = 192;   // 64   O^T accumulator
constexpr uint32_t TM_UB = 256;  // 32   bf16 U^T (A operand)
constexpr uint32_t TM_UDB = 288; // 32   bf16 U^T diag(dl) (A operand)
constexpr uint32_t TM_DU = 320;  // 2 x 64  Ut^T, accumulated into U^T (per chunk parity)
constexpr uint32_t TM_G = 448;   // 64   [Q;K] K^T, later W^T

constexpr uint32_t IDESC_G = instr_desc_bf16(128, 64, 0, 0);                 // [Q;K] . K^T
constexpr uint32_t IDESC_MN64 = instr_desc_bf16(128, 64, 1, 0);              // V^T / K^T (MN-major A) . T^T
constexpr uint32_t IDESC_WNEG = instr_desc_bf16(128, 64, 0, 1) | (1u << 14); // S . (-W)^T, W MN-major
constexpr uint32_t IDESC_Q = instr_desc_bf16(128, 64, 0, 0);                 // S . Qg^T, U^T . P^T
constexpr uint32_t IDESC_S = instr_desc_bf16(128, 128, 0, 1);                // (U^T dl) . K (MN-major B)

enum Bar { B_FULL0 = 0, B_FULL1, B_GDONE, B_UWDONE, B_M1DONE, B_M2DONE, B_TBREADY, B_PREPREADY, B_SREADY, B_UREADY,
           B_OFREE, B_COUNT };

__device__ int g_tc_timeout;  // set when a bounded mbarrier wait gives up

#ifdef GDN_TC_DEBUG
// Debug builds only: per-phase clock stamps of CTA 0 for chunks 0..7, three
// rows of 16 int64 per chunk (control, prep, chain), at float offset 73728.
__device__ float *g_dbg;
#define DBG_CLK(row, i)                                                          \
    if (g_dbg != nullptr && blockIdx.x == 0 && c < 8)                            \
        reinterpret_cast<long long *>(g_dbg + 73728)[(c * 3 + (row)) * 16 + (i)] = clock64();
#else
#define DBG_CLK(row, i)
#endif

struct TcArgs {
    const float *log_alpha, *beta, *S0;
    __nv_bfloat16 *out;
    float *S_final;
    int64_t T, H;
};

__device__ __forceinline__ void named_bar(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Byte offset of 16-byte chunk `c` of row `r` in a 128-byte-swizzled tile
// whose rows are 128 bytes (8-row, 1024-byte atoms).
__device__ __forceinline__ uint32_t sw128(uint32_t r, uint32_t c) {
    return (r >> 3) * 1024u + (r & 7u) * 128u + ((c ^ (r & 7u)) << 4);
}

// Bounded wait on an mbarrier phase that gives up at once when another role
// has already aborted.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    for (uint32_t i = 0; i < (1u << 22); ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 63u && *abort_flag) return false;
    }
    *abort_flag = 1;
    return false;
}

// Barrier over one role's threads that also ANDs a predicate across them.
__device__ __forceinline__ bool bar_and(int id, int n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, %2, %3, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// A wait taken by every thread of a role: the outcome is the same for all of them,
// so a timeout makes the whole role leave its loop together.
__device__ __forceinline__ bool role_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int id, int n) {
    return bar_and(id, n, wait_bar(bar, parity, abort_flag));
}

__device__ __forceinline__ void arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void scale_bf16x8(uint4 &u, float f) {
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&w[i]);
        float2 x = __bfloat1622float2(v);
        w[i] = pack_bf16x2(x.x * f, x.y * f);
    }
    u = make_uint4(w[0], w[1], w[2], w[3]);
}

// 64-token inclusive cumsum by two full warps (t = 0..63 across them); `x` is
// this thread's value, `tmp` a shared slot, (bar_id, n) the role's barrier,
// which every thread of the role must reach once (callers with t >= 64 call
// named_bar themselves).
__device__ __forceinline__ float chunk_cumsum(float x, int t, float *tmp, int bar_id, int n) {
    float s = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, s, off);
        if ((t & 31) >= off) s += y;
    }
    if (t == 31) *tmp = s;
    named_bar(bar_id, n);
    if (t >= 32) s += *tmp;
    return s;
}

__global__ void __launch_bounds__(kThreadsTc, 1)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, TcArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BARS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + 4);
    float *prep_tmp = reinterpret_cast<float *>(sm + OFF_MISC + 8);
    int *prep_flags = reinterpret_cast<int *>(sm + OFF_MISC + 16);  // [2]
    float *chain_tmp = reinterpret_cast<float *>(sm + OFF_MISC + 24);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t T = p.T, H = p.H;
    const int64_t bh = blockIdx.x;
    const int b = (int)(bh / H), h = (int)(bh % H);
    const int N = (int)((T + kC - 1) / kC);
    const uint32_t sbase = smem_u32(sm);

    if (tid == 0) {
        for (int i = 0; i < B_COUNT; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
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
    const uint32_t lb = (uint32_t)((warp & 3) * 32) << 16;  // this warp's TMEM lane quadrant

    if (warp == 0) {
        // ============================== control ==============================
        if (lane == 0) {
            auto issue_loads = [&](int c) {
                const int buf = c & 1, t0 = c * kC;
                mbar_arrive_expect_tx(&bars[B_FULL0 + buf], kTxBytes);
                uint8_t *qk = sm + OFF_QK + buf * QK_BYTES;
                uint8_t *vv = sm + OFF_V + buf * V_BYTES;
#pragma unroll
                for (int blk = 0; blk < 2; ++blk) {
                    tma_load_4d(qk + blk * 16384, &tm_q, &bars[B_FULL0 + buf], blk * 64, h, t0, b);
                    tma_load_4d(qk + blk * 16384 + 8192, &tm_k, &bars[B_FULL0 + buf], blk * 64, h, t0, b);
                    tma_load_4d(vv + blk * 8192, &tm_v, &bars[B_FULL0 + buf], blk * 64, h, t0, b);
                }
            };
            auto mma_G = [&](int c) {
                const uint32_t qk = sbase + OFF_QK + (c & 1) * QK_BYTES;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t a = qk + (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_ss(tm + TM_G, smem_desc_sw128(a, 16, 1024), smem_desc_sw128(a + 8192, 16, 1024), IDESC_G,
                           kk > 0);
                }
                mma_commit(&bars[B_GDONE]);
            };
            auto mma_UW = [&](int c) {
                const int buf = c & 1;
                const uint32_t qk = sbase + OFF_QK + buf * QK_BYTES, vv = sbase + OFF_V + buf * V_BYTES;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss(tm + TM_DU + buf * 64, smem_desc_sw128(vv + kk * 2048, 8192, 1024),
                           smem_desc_sw128(sbase + OFF_TB + kk * 32, 16, 1024), IDESC_MN64, kk > 0);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss(tm + TM_G, smem_desc_sw128(qk + 8192 + kk * 2048, 16384, 1024),
                           smem_desc_sw128(sbase + OFF_TBG + kk * 32, 16, 1024), IDESC_MN64, kk > 0);
                mma_commit(&bars[B_UWDONE]);
            };
            bool ok = true;
            issue_loads(0);
            if (N > 1) issue_loads(1);
            ok = wait_bar(&bars[B_FULL0], 0, abort_flag);
            if (ok) mma_G(0);
            if (ok) ok = wait_bar(&bars[B_TBREADY], 0, abort_flag);
            if (ok) mma_UW(0);
            for (int c = 0; c < N && ok; ++c) {
                const int buf = c & 1;
                const uint32_t par = c & 1;
                const uint32_t qk = sbase + OFF_QK + buf * QK_BYTES;
                DBG_CLK(0, 0)
                if (!(ok = wait_bar(&bars[B_PREPREADY], par, abort_flag))) break;
                DBG_CLK(0, 1)
                if (!(ok = wait_bar(&bars[B_SREADY], par, abort_flag))) break;
                DBG_CLK(0, 2)
                tc_fence_after();
                // U^T accumulates -S W^T onto Ut^T
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tm + TM_DU + buf * 64, tm + TM_SB + kk * 8,
                           smem_desc_sw128(sbase + OFF_W + kk * 2048, 8192, 1024), IDESC_WNEG, 1);
                DBG_CLK(0, 3)
                if (c > 0 && !(ok = wait_bar(&bars[B_OFREE], (c - 1) & 1, abort_flag))) break;
                DBG_CLK(0, 4)
                tc_fence_after();
                // O^T = S Qg^T
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tm + TM_O, tm + TM_SB + kk * 8,
                           smem_desc_sw128(qk + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024), IDESC_Q, kk > 0);
                mma_commit(&bars[B_M1DONE]);
                DBG_CLK(0, 5)
                if (c + 1 < N) {
                    if (!(ok = wait_bar(&bars[B_FULL0 + ((c + 1) & 1)], ((c + 1) >> 1) & 1, abort_flag))) break;
                    DBG_CLK(0, 6)
                    mma_G(c + 1);
                }
                DBG_CLK(0, 7)
                if (!(ok = wait_bar(&bars[B_UREADY], par, abort_flag))) break;
                DBG_CLK(0, 8)
                tc_fence_after();
                // O^T += U^T P^T ;  S += (U^T diag(dl)) K
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(tm + TM_O, tm + TM_UB + kk * 8,
                           smem_desc_sw128(sbase + OFF_P + buf * 8192 + kk * 32, 16, 1024), IDESC_Q, 1);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(tm + TM_S, tm + TM_UDB + kk * 8, smem_desc_sw128(qk + 8192 + kk * 2048, 16384, 1024),
                           IDESC_S, 1);
                mma_commit(&bars[B_M2DONE]);
                DBG_CLK(0, 9)
                if (c + 2 < N) {
                    if (!(ok = wait_bar(&bars[B_M2DONE], par, abort_flag))) break;
                    DBG_CLK(0, 10)
                    issue_loads(c + 2);
                }
                DBG_CLK(0, 11)
                if (c + 1 < N) {
                    if (!(ok = wait_bar(&bars[B_TBREADY], (c + 1) & 1, abort_flag))) break;
                    DBG_CLK(0, 12)
                    mma_UW(c + 1);
                }
                DBG_CLK(0, 13)
            }
            // drain: the last MMAs must be complete before tensor memory is released
            if (ok && N > 0) wait_bar(&bars[B_M2DONE], (N - 1) & 1, abort_flag);
        }
        __syncwarp();
    } else if (warp >= kPrepWarp0 && warp < kChainWarp0) {
        // ============================== prep ==============================
        const int pt = tid - kPrepWarp0 * 32;     // 0..255
        const int ch = (warp - kPrepWarp0) >> 2;  // column half of the TMEM epilogues
        float *g = reinterpret_cast<float *>(sm + OFF_PG);
        float *bet = g + 64, *gam = g + 128, *ea = g + 192, *eb = g + 256;
        float *Am = reinterpret_cast<float *>(sm + OFF_AM);
        float *Tm = reinterpret_cast<float *>(sm + OFF_TM);
        float *Y = reinterpret_cast<float *>(sm + OFF_Y);
        bool ok = true;
        // gates of the chunk being prepared, loaded one chunk ahead (threads pt < 64)
        float la_next = 0.f, be_next = 0.f;
        if (pt < 64 && pt < T) {
            const int64_t gi = ((int64_t)b * T + pt) * H + h;
            la_next = p.log_alpha[gi];
            be_next = p.beta[gi];
        }
        for (int c = 0; c < N && ok; ++c) {
            const int buf = c & 1;
            const uint32_t par = c & 1;
            const int t0 = c * kC;
            const int n = (T - t0 < kC) ? (int)(T - t0) : kC;
            uint8_t *qk_ptr = sm + OFF_QK + buf * QK_BYTES;
            DBG_CLK(1, 0)
            // ---- gates ----
            if (pt < 64) {
                const float x = (pt < n) ? fmaxf(la_next, kLogAlphaFloor) : 0.f;
                bet[pt] = (pt < n) ? be_next : 0.f;
                const float s = chunk_cumsum(x, pt, prep_tmp, kBarPrep, kNumPrep);
                g[pt] = s;
                const int64_t tn = (int64_t)t0 + kC + pt;
                if (tn < T) {
                    const int64_t gi = ((int64_t)b * T + tn) * H + h;
                    la_next = p.log_alpha[gi];
                    be_next = p.beta[gi];
                }
            } else {
                named_bar(kBarPrep, kNumPrep);  // the barrier inside chunk_cumsum
            }
            named_bar(kBarPrep, kNumPrep);
            if (pt < 64) {
                const float gt = g[pt], cm = g[31];
                gam[pt] = expf(gt);
                ea[pt] = expf(gt - cm);
                eb[pt] = expf(cm - gt);
                // e^{g_t - g_s} = e^{g_t - c} e^{c - g_s}, exact to a few ulp while every |g_t - c| < 80
                const bool nr = __all_sync(0xffffffffu, fabsf(gt - cm) < 80.f);
                if (lane == 0) prep_flags[pt >> 5] = nr ? 1 : 0;
            }
            named_bar(kBarPrep, kNumPrep);
            const bool narrow = prep_flags[0] && prep_flags[1];
            DBG_CLK(1, 1)
            if (!(ok = role_wait(&bars[B_GDONE], par, abort_flag, kBarPrep, kNumPrep))) break;
            tc_fence_after();
            DBG_CLK(1, 2)
            // ---- epilogue of G: rows 0..63 -> P (bf16), rows 64..127 -> A (fp32); columns split by half ----
            {
                const int m = (warp & 3) * 32 + lane;  // TMEM lane = row of [Q; K]
                const int t = m & 63;
                const float gt = g[t], at = ea[t];
                uint32_t r[32];
                tmem_ld32(tm + lb + TM_G + ch * 32, r);
                tmem_wait_ld();
                float d[32];
                DBG_CLK(1, 3)
                if (narrow) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) d[i] = at * eb[ch * 32 + i];
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) d[i] = expf(gt - g[ch * 32 + i]);
                }
                if (m < 64) {
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        const int s = ch * 32 + i;
                        const float v0 = (s <= t) ? __uint_as_float(r[i]) * d[i] : 0.f;
                        const float v1 = (s + 1 <= t) ? __uint_as_float(r[i + 1]) * d[i + 1] : 0.f;
                        pk[i >> 1] = pack_bf16x2(v0, v1);
                    }
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
                        *reinterpret_cast<uint4 *>(sm + OFF_P + buf * 8192 + sw128(t, ch * 4 + cc)) =
                            make_uint4(pk[cc * 4], pk[cc * 4 + 1], pk[cc * 4 + 2], pk[cc * 4 + 3]);
                } else {
                    const float bt = bet[t];
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        float v[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int s = ch * 32 + i + e;
                            v[e] = (s < t) ? bt * d[i + e] * __uint_as_float(r[i + e]) : 0.f;
                        }
                        *reinterpret_cast<float4 *>(Am + t * LDM + ch * 32 + i) = make_float4(v[0], v[1], v[2], v[3]);
                    }
                }
                DBG_CLK(1, 4)
                // Qg = diag(gamma) Q in place (MMA-G has consumed Q): a quarter row-block per thread
                {
                    const int qt = pt & 63, blk = (pt >> 6) & 1, qh = pt >> 7;
                    uint4 *row = reinterpret_cast<uint4 *>(qk_ptr + blk * 16384 + qt * 128 + qh * 64);
                    const float gm = gam[qt];
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        uint4 u = row[cc];
                        scale_bf16x8(u, gm);
                        row[cc] = u;
                    }
                }
            }
            __syncwarp();
            named_bar(kBarPrep, kNumPrep);
            DBG_CLK(1, 5)
            // ---- T = (I + A)^{-1}: 16x16 diagonal blocks (warps 4..7, a column per lane) ----
            if (warp < kPrepWarp0 + 4 && lane < 16) {
                const int o = (warp - kPrepWarp0) * 16;
                float x[16];
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) {
                    float acc = (rr == lane) ? 1.f : 0.f;
#pragma unroll
                    for (int s = 0; s < rr; ++s) acc -= Am[(o + rr) * LDM + o + s] * x[s];
                    x[rr] = acc;
                }
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) Tm[(o + rr) * LDM + o + lane] = x[rr];
            }
            __syncwarp();
            named_bar(kBarPrep, kNumPrep);
            DBG_CLK(1, 6)
            // block rows I = 1..3:  T_IJ = -T_II sum_{K=J}^{I-1} A_IK T_KJ ; a thread per (J, row, 4 columns)
            for (int I = 1; I < 4; ++I) {
                if (pt < I * 64) {
                    const int J = pt >> 6, rr = (pt >> 2) & 15, c4 = (pt & 3) * 4;
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                    for (int K = J; K < I; ++K) {
                        const float *arow = Am + (16 * I + rr) * LDM + 16 * K;
                        const float *tcol = Tm + (16 * K) * LDM + 16 * J + c4;
#pragma unroll
                        for (int mm = 0; mm < 16; ++mm) {
                            const float a = arow[mm];
                            const float4 tv = *reinterpret_cast<const float4 *>(tcol + mm * LDM);
                            acc.x = fmaf(a, tv.x, acc.x);
                            acc.y = fmaf(a, tv.y, acc.y);
                            acc.z = fmaf(a, tv.z, acc.z);
                            acc.w = fmaf(a, tv.w, acc.w);
                        }
                    }
                    *reinterpret_cast<float4 *>(Y + J * 256 + rr * 16 + c4) = acc;
                }
                named_bar(kBarPrep, kNumPrep);
                if (pt < I * 64) {
                    const int J = pt >> 6, rr = (pt >> 2) & 15, c4 = (pt & 3) * 4;
                    const float *trow = Tm + (16 * I + rr) * LDM + 16 * I;
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int mm = 0; mm < 16; ++mm) {
                        const float a = trow[mm];
                        const float4 y = *reinterpret_cast<const float4 *>(Y + J * 256 + mm * 16 + c4);
                        acc.x = fmaf(a, y.x, acc.x);
                        acc.y = fmaf(a, y.y, acc.y);
                        acc.z = fmaf(a, y.z, acc.z);
                        acc.w = fmaf(a, y.w, acc.w);
                    }
                    *reinterpret_cast<float4 *>(Tm + (16 * I + rr) * LDM + 16 * J + c4) =
                        make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
                }
                named_bar(kBarPrep, kNumPrep);
                DBG_CLK(1, 6 + I)
            }
            // ---- T diag(beta) and T diag(beta gamma), bf16 K-major: a (tile, row, column half) per thread ----
            {
                const int t = pt & 63, with_gamma = (pt >> 6) & 1, hh = pt >> 7;
                uint8_t *dst = sm + (with_gamma ? OFF_TBG : OFF_TB);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t pk[4];
#pragma unroll
                    for (int i = 0; i < 8; i += 2) {
                        const int s = hh * 32 + cc * 8 + i;
                        float v0 = (s <= t) ? Tm[t * LDM + s] * bet[s] : 0.f;
                        float v1 = (s + 1 <= t) ? Tm[t * LDM + s + 1] * bet[s + 1] : 0.f;
                        if (with_gamma) {
                            v0 *= gam[s];
                            v1 *= gam[s + 1];
                        }
                        pk[i >> 1] = pack_bf16x2(v0, v1);
                    }
                    *reinterpret_cast<uint4 *>(dst + sw128(t, hh * 4 + cc)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
            fence_proxy_async_smem();
            named_bar(kBarPrep, kNumPrep);
            if (pt == 0) arrive(&bars[B_TBREADY]);
            DBG_CLK(1, 10)
            // ---- W (bf16, MN-major rows i) from W^T in TMEM (MMA-1 of the previous chunk is done with W) ----
            if (!(ok = role_wait(&bars[B_UWDONE], par, abort_flag, kBarPrep, kNumPrep))) break;
            if (c > 0 && !(ok = role_wait(&bars[B_M1DONE], (c - 1) & 1, abort_flag, kBarPrep, kNumPrep))) break;
            tc_fence_after();
            DBG_CLK(1, 11)
            {
                const int i = (warp & 3) * 32 + lane;
                uint32_t r[32];
                tmem_ld32(tm + lb + TM_G + ch * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(r[cc * 8 + 0]), __uint_as_float(r[cc * 8 + 1]));
                    v.y = pack_bf16x2(__uint_as_float(r[cc * 8 + 2]), __uint_as_float(r[cc * 8 + 3]));
                    v.z = pack_bf16x2(__uint_as_float(r[cc * 8 + 4]), __uint_as_float(r[cc * 8 + 5]));
                    v.w = pack_bf16x2(__uint_as_float(r[cc * 8 + 6]), __uint_as_float(r[cc * 8 + 7]));
                    *reinterpret_cast<uint4 *>(sm + OFF_W + sw128(i, ch * 4 + cc)) = v;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(kBarPrep, kNumPrep);
            if (pt == 0) arrive(&bars[B_PREPREADY]);
            DBG_CLK(1, 12)
        }
    } else if (warp >= kChainWarp0) {
        // ============================== chain ==============================
        const int j = tid - kChainWarp0 * 32;  // TMEM lane / state row, 0..127
        float *dl = reinterpret_cast<float *>(sm + OFF_CG);
        float *gcs = dl + 64;  // [0] = gamma_C of the chunk
        bool ok = true;
        // S0 -> TMEM
        {
            const float *src = p.S0 ? p.S0 + (bh * kD + j) * (int64_t)kD : nullptr;
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
        float la_next = 0.f;
        if (j < 64 && j < T) la_next = p.log_alpha[((int64_t)b * T + j) * H + h];
        auto write_out = [&](int cprev) {
            const int64_t t0p = (int64_t)cprev * kC;
            const int np = (T - t0p < kC) ? (int)(T - t0p) : kC;
            __nv_bfloat16 *ob = p.out + (((int64_t)b * T + t0p) * H + h) * kD + j;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t r[32];
                tmem_ld32(tm + lb + TM_O + half * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int t = half * 32 + i;
                    if (t < np) ob[(int64_t)t * H * kD] = __float2bfloat16_rn(__uint_as_float(r[i]));
                }
            }
        };
        for (int c = 0; c < N && ok; ++c) {
            const int buf = c & 1;
            const uint32_t par = c & 1;
            const int t0 = c * kC;
            const int n = (T - t0 < kC) ? (int)(T - t0) : kC;
            DBG_CLK(2, 0)
            // ---- chain gates: dl_s = e^{g_C - g_s} and gamma_C ----
            {
                float s = 0.f;
                if (j < 64) {
                    const float x = (j < n) ? fmaxf(la_next, kLogAlphaFloor) : 0.f;
                    s = chunk_cumsum(x, j, chain_tmp, kBarChain, kNumChain);
                    const int64_t tn = (int64_t)t0 + kC + j;
                    if (tn < T) la_next = p.log_alpha[((int64_t)b * T + tn) * H + h];
                    dl[j] = s;
                } else {
                    named_bar(kBarChain, kNumChain);  // the barrier inside chunk_cumsum
                }
                named_bar(kBarChain, kNumChain);
                const float g63 = dl[63];
                named_bar(kBarChain, kNumChain);
                if (j < 64) dl[j] = expf(g63 - s);
                if (j == 0) gcs[0] = expf(g63);
                named_bar(kBarChain, kNumChain);
            }
            // ---- S -> bf16 operand copy; S <- gamma_C S ----
            {
                const float gC = gcs[0];
#pragma unroll
                for (int piece = 0; piece < 4; ++piece) {
                    uint32_t r[32];
                    tmem_ld32(tm + lb + TM_S + piece * 32, r);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 2)
                        pk[i >> 1] = pack_bf16x2(__uint_as_float(r[i]), __uint_as_float(r[i + 1]));
                    tmem_st16(tm + lb + TM_SB + piece * 16, pk);
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * gC);
                    tmem_st32(tm + lb + TM_S + piece * 32, r);
                }
                tmem_wait_st();
                tc_fence_before();
                named_bar(kBarChain, kNumChain);
                if (j == 0) arrive(&bars[B_SREADY]);
            }
            DBG_CLK(2, 1)
            // ---- outputs of the previous chunk (frees the O accumulator) ----
            if (c > 0) {
                write_out(c - 1);
                tc_fence_before();
                named_bar(kBarChain, kNumChain);
                if (j == 0) arrive(&bars[B_OFREE]);
            }
            DBG_CLK(2, 2)
            if (!(ok = role_wait(&bars[B_M1DONE], par, abort_flag, kBarChain, kNumChain))) break;
            tc_fence_after();
            DBG_CLK(2, 3)
            // ---- U^T (accumulated in TMEM) -> bf16 U^T and bf16 U^T diag(dl) ----
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t u[32];
                tmem_ld32(tm + lb + TM_DU + buf * 64 + half * 32, u);
                tmem_wait_ld();
                uint32_t pk[16], pd[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const float u0 = __uint_as_float(u[i]), u1 = __uint_as_float(u[i + 1]);
                    pk[i >> 1] = pack_bf16x2(u0, u1);
                    pd[i >> 1] = pack_bf16x2(u0 * dl[half * 32 + i], u1 * dl[half * 32 + i + 1]);
                }
                tmem_st16(tm + lb + TM_UB + half * 16, pk);
                tmem_st16(tm + lb + TM_UDB + half * 16, pd);
            }
            tmem_wait_st();
            tc_fence_before();
            named_bar(kBarChain, kNumChain);
            if (j == 0) arrive(&bars[B_UREADY]);
            DBG_CLK(2, 4)
            if (!(ok = role_wait(&bars[B_M2DONE], par, abort_flag, kBarChain, kNumChain))) break;
            tc_fence_after();
            DBG_CLK(2, 5)
        }
        if (ok && N > 0) write_out(N - 1);
        if (ok && p.S_final) {
            float *dst = p.S_final + (bh * kD + j) * (int64_t)kD;
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
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) atomicExch(&g_tc_timeout, 1);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, 512);
    }
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
    return p.dtype == 1 && p.dk == kD && p.dv == kD && p.chunk == kC && p.T <= (int64_t)INT32_MAX / 2 &&
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
