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
//     T    = (I + A)^{-1}   16x16 diagonal blocks by substitution, merged 16->32->64
//                           with warp-level TF32 MMAs (fp32 accumulation); the final writer
//                           of each entry also writes T diag(beta) and T diag(beta gamma) in bf16
//     Ut^T = V^T (T diag(beta))^T,  W^T = K^T (T diag(beta gamma))^T   (tcgen05)
//   chain (needs S; sequential over chunks):
//     U^T  = Ut^T - S W^T                      (tcgen05 accumulate, B negated; A = bf16 S in TMEM)
//     S   <- gamma_C S + (U^T diag(dl)) K      (tcgen05 accumulate into the float32 state)
//   outputs (off the chain), with e^{g_t - g_s} = e^{g_t - c} e^{c - g_s} (c = g_31) when the
//   chunk's decay span allows it (always exact; otherwise P' = P and f2 = 1):
//     O1^T = S Q^T,  O2^T = U^T P'^T,  P'_ts = e^{c - g_s} (Q K^T)_ts (s <= t)   (tcgen05)
//     o_t  = gamma_t O1_t + e^{g_t - c} O2_t, staged in shared memory, written by TMA
// The state S stays in tensor memory in float32 for the whole sequence; its
// bf16 operand copy is rewritten from it every chunk.
//
// Warp roles (640 threads).  One thread issuing tcgen05.mma sustains about
// one MMA per ~90 cycles, more than an M128xN64xK16 MMA takes to execute, so
// the MMAs are issued by three threads, one per independent stream:
//   warp 0      chain issuer: TMA loads, U^T and S updates (the critical path)
//   warp 1      output issuer: O1^T = S Q^T, O2^T = U^T P'^T
//   warp 2      prep issuer: G, Ut^T, W^T
//   warps 4-11  prep for chunk c+1 (256 threads) while the chain runs chunk c
//   warps 12-19 chain: state conversion, U^T epilogue, outputs (two warps per
//               TMEM lane quadrant; a thread owns state row j and a column half)
//   warp 3      idle
// Roles hand work to each other through mbarriers (tcgen05.commit for MMA
// completion, single-thread arrivals after a named barrier otherwise); every
// barrier completes once per chunk, and no role can run two completions ahead
// of a role that waits on it.  Every wait is bounded; a wait that gives up
// sets an abort flag that releases every other wait, and each role leaves its
// loop as a whole, so the CTA always frees its tensor memory and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <stdlib.h>

#include <atomic>

#include "gdn.h"
#include "gdn_internal.h"
#include "sm100.cuh"
#include "tc_util.cuh"

namespace gdn {
namespace {

using namespace sm100;
using namespace tcu;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kThreadsTc = 640;
constexpr int kPrepWarp0 = 4, kNumPrep = 256;
constexpr int kChainWarp0 = 12, kNumChain = 256;
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
constexpr uint32_t OFF_XS = 182272;      // 5 KB   merge scratch: 4 x [16][8] (16->32), then [32][LDX2] (32->64)
constexpr int LDX2 = 40;
constexpr uint32_t OFF_PG = 187392;      // prep gates per chunk parity: g, beta, gamma, e^{g-c}, e^{c-g} (2 x 5 x 64)
constexpr uint32_t OFF_CG = 189952;      // chain gates per chunk parity: dl[2][64], f1[2][64], f2[2][64], gamma_C[2]
constexpr uint32_t OFF_OST = 192512;     // 16 KB  output staging: two [64 t][64 d] bf16 boxes, 128-byte swizzle
constexpr uint32_t OFF_BARS = 208896;    // mbarriers
constexpr uint32_t OFF_MISC = 209024;    // tmem slot, abort flag, scan scratch
constexpr uint32_t SMEM_TC = 209088 + 1024;
constexpr uint32_t kTxBytes = 3 * 2 * 8192;  // Q, K, V: two 8 KB boxes each

// TMEM column map (512 columns).
constexpr uint32_t TM_S = 0;     // 128  S float32 (row j in lane j)
constexpr uint32_t TM_SB = 128;  // 64   bf16 S (A operand, 2 per column)
constexpr uint32_t TM_O = 192;   // 64   O1^T = S Q^T
constexpr uint32_t TM_UB = 256;  // 32   bf16 U^T (A operand)
constexpr uint32_t TM_UDB = 288; // 32   bf16 U^T diag(dl) (A operand)
constexpr uint32_t TM_DU = 320;  // 64   Ut^T, accumulated into U^T
constexpr uint32_t TM_G = 384;   // 64   [Q;K] K^T, later W^T
constexpr uint32_t TM_O2 = 448;  // 64   O2^T = U^T P'^T

constexpr uint32_t IDESC_G = instr_desc_bf16(128, 64, 0, 0);                 // [Q;K] . K^T
constexpr uint32_t IDESC_MN64 = instr_desc_bf16(128, 64, 1, 0);              // V^T / K^T (MN-major A) . T^T
constexpr uint32_t IDESC_WNEG = instr_desc_bf16(128, 64, 0, 1) | (1u << 14); // S . (-W)^T, W MN-major
constexpr uint32_t IDESC_Q = instr_desc_bf16(128, 64, 0, 0);                 // S . Qg^T, U^T . P^T
constexpr uint32_t IDESC_S = instr_desc_bf16(128, 128, 0, 1);                // (U^T dl) . K (MN-major B)

enum Bar {
    B_FULL0 = 0, B_FULL1,                                 // TMA tiles landed (per buffer)
    B_GDONE, B_WDONE, B_UTDONE,                           // prep MMAs complete
    B_M1ADONE, B_M2BDONE,                                 // chain MMAs complete
    B_M1BDONE, B_M2ADONE,                                 // output MMAs complete
    B_TBREADY, B_PREPREADY, B_SREADY, B_UREADY, B_OFREE,  // role hand-offs
    B_COUNT
};

static_assert(B_COUNT * 8 <= OFF_MISC - OFF_BARS, "mbarriers overflow their shared-memory slot");

__device__ int g_tc_timeout;  // set when a bounded mbarrier wait gives up

#ifdef GDN_TC_DEBUG
// Debug builds only: per-phase clock stamps of CTA 0 for chunks 0..7, five
// rows of 16 int64 per chunk (chain issuer, output issuer, prep issuer, prep,
// chain), at float offset 73728.
__device__ float *g_dbg;
#define DBG_CLK(row, i)                                                          \
    if (g_dbg != nullptr && blockIdx.x == 0 && c < 8)                            \
        reinterpret_cast<long long *>(g_dbg + 73728)[(c * 5 + (row)) * 16 + (i)] = clock64();
#else
#define DBG_CLK(row, i)
#endif

// One launch covers every (b, h) and, for long sequences with few heads, every
// segment of the sequence.  mode 0: one CTA per (b, h, segment) computes the
// outputs of its chunk range from that segment's entry state (S0 for the first
// segment, else S_entry) and writes S_final from the last segment.  mode 1:
// two CTAs per (b, h, segment < nseg - 1) compute the segment's affine transfer
// S_end = S_start M + B: one runs the recurrence from the zero state (-> Bw), the
// other from the identity with v = 0 (-> Mw; rows of the state evolve
// independently, so each row of M is a state row with no write term).
struct TcArgs {
    const float *log_alpha, *beta, *S0;
    __nv_bfloat16 *out;
    float *S_final;
    int64_t T, H;
    int mode, nseg, seg_len;
    const float *S_entry;  // [B*H][nseg-1][dv][dk]: entry states of segments 1..nseg-1
    float *Bw, *Mw;        // [B*H][nseg-1][dv][dk] / [dk][dk]: segment transfers
};

// Writes entries (row, col) and (row, col + 1) (col even) of T diag(beta) and
// T diag(beta gamma) into their bf16 K-major 128-byte-swizzled tiles.
__device__ __forceinline__ void store_tb_pair(uint8_t *sm, int row, int col, float v0, float v1, const float *bet,
                                              const float *gam) {
    const uint32_t off = sw128(row, col >> 3) + (col & 7) * 2;
    const float b0 = bet[col], b1 = bet[col + 1];
    *reinterpret_cast<uint32_t *>(sm + OFF_TB + off) = pack_bf16x2(v0 * b0, v1 * b1);
    *reinterpret_cast<uint32_t *>(sm + OFF_TBG + off) = pack_bf16x2(v0 * b0 * gam[col], v1 * b1 * gam[col + 1]);
}

__global__ void __launch_bounds__(kThreadsTc, 1)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o, TcArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BARS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + 4);
    float *prep_tmp = reinterpret_cast<float *>(sm + OFF_MISC + 8);
    int *prep_flags = reinterpret_cast<int *>(sm + OFF_MISC + 16);  // [2 parities][2 warps]
    float *chain_tmp = reinterpret_cast<float *>(sm + OFF_MISC + 32);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t T = p.T, H = p.H;
    // work item: (b, h), segment, and kind (0 = outputs, 1 = transfer B, 2 = transfer M)
    int64_t bh;
    int seg, kind;
    if (p.mode == 0) {
        bh = blockIdx.x / p.nseg;
        seg = (int)(blockIdx.x % p.nseg);
        kind = 0;
    } else {
        const int64_t q = blockIdx.x >> 1;
        bh = q / (p.nseg - 1);
        seg = (int)(q % (p.nseg - 1));
        kind = 1 + (int)(blockIdx.x & 1);
    }
    const bool outputs = (kind == 0);
    const int b = (int)(bh / H), h = (int)(bh % H);
    const int Ntot = (int)((T + kC - 1) / kC);
    const int c0 = seg * p.seg_len;                                      // first chunk of this CTA
    const int N = (Ntot - c0 < p.seg_len) ? (Ntot - c0) : p.seg_len;     // chunks of this CTA
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
        // ====================== chain issuer (and TMA) ======================
        if (lane == 0) {
            auto issue_loads = [&](int c) {
                const int buf = c & 1, t0 = (c0 + c) * kC;
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
            bool ok = true;
            issue_loads(0);
            if (N > 1) issue_loads(1);
            for (int c = 0; c < N && ok; ++c) {
                const uint32_t par = c & 1;
                const uint32_t qk = sbase + OFF_QK + (c & 1) * QK_BYTES;
                DBG_CLK(0, 0)
                if (!(ok = wait_bar(&bars[B_PREPREADY], par, abort_flag))) break;
                if (!(ok = wait_bar(&bars[B_SREADY], par, abort_flag))) break;
                if (!(ok = wait_bar(&bars[B_UTDONE], par, abort_flag))) break;
                DBG_CLK(0, 1)
                tc_fence_after();
                // U^T = Ut^T - S W^T  (transfer-M runs have v = 0, so Ut^T = 0 and U^T starts fresh)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tm + TM_DU, tm + TM_SB + kk * 8, smem_desc_sw128(sbase + OFF_W + kk * 2048, 8192, 1024),
                           IDESC_WNEG, (kind != 2 || kk > 0) ? 1u : 0u);
                mma_commit(&bars[B_M1ADONE]);
                DBG_CLK(0, 2)
                if (!(ok = wait_bar(&bars[B_UREADY], par, abort_flag))) break;
                DBG_CLK(0, 3)
                tc_fence_after();
                // S += (U^T diag(dl)) K
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(tm + TM_S, tm + TM_UDB + kk * 8, smem_desc_sw128(qk + 8192 + kk * 2048, 16384, 1024),
                           IDESC_S, 1);
                mma_commit(&bars[B_M2BDONE]);
                DBG_CLK(0, 4)
                if (c + 2 < N) {
                    // buffer c & 1 is free once both final MMAs of chunk c are done with K and Q
                    if (!(ok = wait_bar(&bars[B_M2BDONE], par, abort_flag))) break;
                    if (!(ok = wait_bar(&bars[B_M2ADONE], par, abort_flag))) break;
                    issue_loads(c + 2);
                }
                DBG_CLK(0, 5)
            }
            if (ok && N > 0) wait_bar(&bars[B_M2BDONE], (N - 1) & 1, abort_flag);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ========================= output issuer =========================
        if (lane == 0) {
            bool ok = true;
            for (int c = 0; c < N && ok; ++c) {
                const uint32_t par = c & 1;
                const uint32_t qk = sbase + OFF_QK + (c & 1) * QK_BYTES;
                DBG_CLK(1, 0)
                if (!(ok = wait_bar(&bars[B_PREPREADY], par, abort_flag))) break;
                if (!(ok = wait_bar(&bars[B_SREADY], par, abort_flag))) break;
                if (c > 0 && !(ok = wait_bar(&bars[B_OFREE], (c - 1) & 1, abort_flag))) break;
                DBG_CLK(1, 1)
                tc_fence_after();
                // O1^T = S Q^T  (transfer runs issue no output MMAs; the commits below still arrive)
                if (outputs) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ts(tm + TM_O, tm + TM_SB + kk * 8,
                               smem_desc_sw128(qk + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024), IDESC_Q, kk > 0);
                }
                mma_commit(&bars[B_M1BDONE]);
                DBG_CLK(1, 2)
                if (!(ok = wait_bar(&bars[B_UREADY], par, abort_flag))) break;
                DBG_CLK(1, 3)
                tc_fence_after();
                // O2^T = U^T P'^T
                if (outputs) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(tm + TM_O2, tm + TM_UB + kk * 8,
                               smem_desc_sw128(sbase + OFF_P + (c & 1) * 8192 + kk * 32, 16, 1024), IDESC_Q, kk > 0);
                }
                mma_commit(&bars[B_M2ADONE]);
                DBG_CLK(1, 4)
            }
            if (ok && N > 0) wait_bar(&bars[B_M2ADONE], (N - 1) & 1, abort_flag);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ========================== prep issuer ==========================
        if (lane == 0) {
            bool ok = true;
            for (int c = 0; c < N && ok; ++c) {
                const int buf = c & 1;
                const uint32_t par = c & 1;
                const uint32_t qk = sbase + OFF_QK + buf * QK_BYTES, vv = sbase + OFF_V + buf * V_BYTES;
                DBG_CLK(2, 0)
                if (!(ok = wait_bar(&bars[B_FULL0 + buf], (c >> 1) & 1, abort_flag))) break;
                // the G region is free once the prep role has read W^T of the previous chunk
                if (c > 0 && !(ok = wait_bar(&bars[B_PREPREADY], (c - 1) & 1, abort_flag))) break;
                DBG_CLK(2, 1)
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t a = qk + (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_ss(tm + TM_G, smem_desc_sw128(a, 16, 1024), smem_desc_sw128(a + 8192, 16, 1024), IDESC_G,
                           kk > 0);
                }
                mma_commit(&bars[B_GDONE]);
                DBG_CLK(2, 2)
                if (!(ok = wait_bar(&bars[B_TBREADY], par, abort_flag))) break;
                DBG_CLK(2, 3)
                tc_fence_after();
                // W^T first: the prep role is waiting for it
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss(tm + TM_G, smem_desc_sw128(qk + 8192 + kk * 2048, 16384, 1024),
                           smem_desc_sw128(sbase + OFF_TBG + kk * 32, 16, 1024), IDESC_MN64, kk > 0);
                mma_commit(&bars[B_WDONE]);
                // the DU region is free once the chain has read U^T of the previous chunk
                if (c > 0 && !(ok = wait_bar(&bars[B_UREADY], (c - 1) & 1, abort_flag))) break;
                tc_fence_after();
                if (kind != 2) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss(tm + TM_DU, smem_desc_sw128(vv + kk * 2048, 8192, 1024),
                               smem_desc_sw128(sbase + OFF_TB + kk * 32, 16, 1024), IDESC_MN64, kk > 0);
                }
                mma_commit(&bars[B_UTDONE]);
                DBG_CLK(2, 4)
            }
            if (ok && N > 0) wait_bar(&bars[B_UTDONE], (N - 1) & 1, abort_flag);
        }
        __syncwarp();
    } else if (warp >= kPrepWarp0 && warp < kChainWarp0) {
        // ============================== prep ==============================
        const int pt = tid - kPrepWarp0 * 32;     // 0..255
        const int pw = warp - kPrepWarp0;         // 0..7
        const int ch = pw >> 2;                   // column half of the TMEM epilogues
        const int g8 = lane >> 2, t4 = lane & 3;  // MMA fragment coordinates
        float *Am = reinterpret_cast<float *>(sm + OFF_AM);
        float *Tm = reinterpret_cast<float *>(sm + OFF_TM);
        float *Xs = reinterpret_cast<float *>(sm + OFF_XS);
        bool ok = true;
        // the upper triangles of the bf16 T tiles are never written below: zero both tiles once
#pragma unroll
        for (int it = 0; it < 4; ++it)
            reinterpret_cast<uint4 *>(sm + OFF_TB)[pt + 256 * it] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
        // gates of the chunk being prepared, loaded one chunk ahead (threads pt < 64)
        float la_next = 0.f, be_next = 0.f;
        if (pt < 64 && (int64_t)c0 * kC + pt < T) {
            const int64_t gi = ((int64_t)b * T + (int64_t)c0 * kC + pt) * H + h;
            la_next = p.log_alpha[gi];
            be_next = p.beta[gi];
        }
        // gates of chunk cg into buffer cg & 1: g (chunk cumsum of log alpha), beta, gamma = e^g,
        // e^{g_t - c}, e^{c - g_t} with c = g_31, and the narrow-chunk flags
        auto prep_gates = [&](int cg) {
            float *gb = reinterpret_cast<float *>(sm + OFF_PG) + (cg & 1) * 320;
            const int64_t t0g = (int64_t)(c0 + cg) * kC;
            const int ng = (T - t0g < kC) ? (int)(T - t0g) : kC;
            if (pt < 64) {
                const float x = (pt < ng) ? fmaxf(la_next, kLogAlphaFloor) : 0.f;
                gb[64 + pt] = (pt < ng) ? be_next : 0.f;
                const float s = chunk_cumsum(x, pt, prep_tmp, kBarPrep, kNumPrep);
                gb[pt] = s;
                const int64_t tn = t0g + kC + pt;
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
                const float gt = gb[pt], cm = gb[31];
                gb[128 + pt] = expf(gt);
                gb[192 + pt] = expf(gt - cm);
                gb[256 + pt] = expf(cm - gt);
                // e^{g_t - g_s} = e^{g_t - c} e^{c - g_s}, exact to a few ulp; used while every
                // |g_t - c| < 60, so that neither factor nor the output partial sums overflow
                const bool nr = __all_sync(0xffffffffu, fabsf(gt - cm) < 60.f);
                if (lane == 0) prep_flags[(cg & 1) * 2 + (pt >> 5)] = nr ? 1 : 0;
            }
            named_bar(kBarPrep, kNumPrep);
        };
        prep_gates(0);
        for (int c = 0; c < N && ok; ++c) {
            const int buf = c & 1;
            const uint32_t par = c & 1;
            const float *g = reinterpret_cast<const float *>(sm + OFF_PG) + buf * 320;
            const float *bet = g + 64, *gam = g + 128, *ea = g + 192, *eb = g + 256;
            const bool narrow = prep_flags[buf * 2] && prep_flags[buf * 2 + 1];
            DBG_CLK(3, 0)
            DBG_CLK(3, 1)
            if (!(ok = role_wait(&bars[B_GDONE], par, abort_flag, kBarPrep, kNumPrep))) break;
            tc_fence_after();
            DBG_CLK(3, 2)
            // ---- epilogue of G: rows 0..63 -> P' (bf16), rows 64..127 -> A (fp32); columns split by half.
            //      P'_ts = e^{c - g_s} (q_t . k_s) when the chunk is narrow (the output applies e^{g_t - c}),
            //      else P_ts = e^{g_t - g_s} (q_t . k_s) ----
            {
                const int m = (warp & 3) * 32 + lane;  // TMEM lane = row of [Q; K]
                const int t = m & 63;
                const float gt = g[t], at = ea[t], bt = bet[t];
                const float sc = (m < 64) ? 1.f : at;
#pragma unroll 1
                for (int piece = 0; piece < 2; ++piece) {
                    const int s0 = ch * 32 + piece * 16;  // first column of this piece
                    uint32_t r[16];
                    tmem_ld16(tm + lb + TM_G + s0, r);
                    tmem_wait_ld();
                    // decay factor of column s: e^{c - g_s} (times e^{g_t - c} for A rows) in a narrow
                    // chunk, else e^{g_t - g_s}
                    float d[16];
                    if (narrow) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) d[i] = sc * eb[s0 + i];
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) d[i] = expf(gt - g[s0 + i]);
                    }
                    if (m < 64) {
                        uint32_t pk[8];
#pragma unroll
                        for (int i = 0; i < 16; i += 2) {
                            const float v0 = (s0 + i <= t) ? __uint_as_float(r[i]) * d[i] : 0.f;
                            const float v1 = (s0 + i + 1 <= t) ? __uint_as_float(r[i + 1]) * d[i + 1] : 0.f;
                            pk[i >> 1] = pack_bf16x2(v0, v1);
                        }
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc)
                            *reinterpret_cast<uint4 *>(sm + OFF_P + buf * 8192 + sw128(t, (s0 >> 3) + cc)) =
                                make_uint4(pk[cc * 4], pk[cc * 4 + 1], pk[cc * 4 + 2], pk[cc * 4 + 3]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; i += 4) {
                            float v[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                v[e] = (s0 + i + e < t) ? bt * d[i + e] * __uint_as_float(r[i + e]) : 0.f;
                            *reinterpret_cast<float4 *>(Am + t * LDM + s0 + i) = make_float4(v[0], v[1], v[2], v[3]);
                        }
                    }
                }
            }
            __syncwarp();
            named_bar(kBarPrep, kNumPrep);
            DBG_CLK(3, 3)
            // ---- T = (I + A)^{-1} ----
            // (1) 16x16 diagonal blocks by substitution: role warps 0..3, a column per lane; warps 0 and 2
            //     also zero the upper 16x16 block inside their 32x32 diagonal block
            if (pw < 4 && lane < 16) {
                const int o = pw * 16;
                float x[16];
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) {
                    float a0 = (rr == lane) ? 1.f : 0.f, a1 = 0.f;
#pragma unroll
                    for (int s = 0; s + 1 < rr; s += 2) {
                        a0 -= Am[(o + rr) * LDM + o + s] * x[s];
                        a1 -= Am[(o + rr) * LDM + o + s + 1] * x[s + 1];
                    }
                    if (rr & 1) a0 -= Am[(o + rr) * LDM + o + rr - 1] * x[rr - 1];
                    x[rr] = a0 + a1;
                }
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) Tm[(o + rr) * LDM + o + lane] = x[rr];
                if ((pw & 1) == 0) {
#pragma unroll
                    for (int rr = 0; rr < 16; ++rr) Tm[(o + rr) * LDM + o + 16 + lane] = 0.f;
                }
            }
            __syncwarp();
            named_bar(kBarPrep, kNumPrep);
            DBG_CLK(3, 4)
            // (2) 16 -> 32: T_10 = -T_11 (A_10 T_00) inside each 32x32 diagonal block; one warp per
            //     (block, 8-column tile); X goes through a per-warp scratch tile. Meanwhile role warps
            //     4..7 write the four 16x16 diagonal blocks as bf16 T diag(beta) and T diag(beta gamma),
            //     eight columns (one 16-byte swizzle unit) per thread
            if (pw >= 4) {
                const int idx = pt - 128, row = idx >> 1, col = (row & ~15) + (idx & 1) * 8;
                const float4 x0 = *reinterpret_cast<const float4 *>(Tm + row * LDM + col);
                const float4 x1 = *reinterpret_cast<const float4 *>(Tm + row * LDM + col + 4);
                const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                uint32_t wb[4], wg[4];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const float b0 = bet[col + e], b1 = bet[col + e + 1];
                    wb[e >> 1] = pack_bf16x2(xv[e] * b0, xv[e + 1] * b1);
                    wg[e >> 1] = pack_bf16x2(xv[e] * (b0 * gam[col + e]), xv[e + 1] * (b1 * gam[col + e + 1]));
                }
                const uint32_t off = sw128(row, col >> 3);
                *reinterpret_cast<uint4 *>(sm + OFF_TB + off) = make_uint4(wb[0], wb[1], wb[2], wb[3]);
                *reinterpret_cast<uint4 *>(sm + OFF_TBG + off) = make_uint4(wg[0], wg[1], wg[2], wg[3]);
            } else {
                const int q0 = (pw >> 1) * 32, n0 = (pw & 1) * 8;
                float *xs = Xs + pw * 128;  // [16][8]
                float dacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    uint32_t a[4], bb[2];
                    load_a(a, Am, LDM, q0 + 16, q0 + 8 * kk, g8, t4);
                    load_b(bb, Tm, LDM, q0 + 8 * kk, q0 + n0, g8, t4);
                    mma_tf32(dacc, a, bb);
                }
                store_d(xs, 8, 0, 0, dacc, g8, t4);
                __syncwarp();
                float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    uint32_t a[4], bb[2];
                    load_a(a, Tm, LDM, q0 + 16, q0 + 16 + 8 * kk, g8, t4);
                    load_b(bb, xs, 8, 8 * kk, 0, g8, t4);
                    mma_tf32(e, a, bb);
                }
                store_neg_d(Tm, LDM, q0 + 16, q0 + n0, e, g8, t4);
                store_tb_pair(sm, q0 + 16 + g8, q0 + n0 + 2 * t4, -e[0], -e[1], bet, gam);
                store_tb_pair(sm, q0 + 24 + g8, q0 + n0 + 2 * t4, -e[2], -e[3], bet, gam);
            }
            named_bar(kBarPrep, kNumPrep);
            DBG_CLK(3, 5)
            // (3) 32 -> 64: X = A[32:64, 0:32] T[0:32, 0:32], then T[32:64, 0:32] = -T[32:64, 32:64] X;
            //     one warp per (16-row, 8-column) tile; T is lower triangular, so zero k-steps are skipped
            {
                const int mi = pw >> 2, ni = pw & 3;
                float *x2 = Xs;  // [32][LDX2], reuses the 16->32 scratch (a barrier separates the two)
                float dacc[4] = {0.f, 0.f, 0.f, 0.f};
                for (int kk = ni; kk < 4; ++kk) {
                    uint32_t a[4], bb[2];
                    load_a(a, Am, LDM, 32 + 16 * mi, 8 * kk, g8, t4);
                    load_b(bb, Tm, LDM, 8 * kk, 8 * ni, g8, t4);
                    mma_tf32(dacc, a, bb);
                }
                store_d(x2, LDX2, 16 * mi, 8 * ni, dacc, g8, t4);
                named_bar(kBarPrep, kNumPrep);
                float e[4] = {0.f, 0.f, 0.f, 0.f};
                for (int kk = 0; kk <= 2 * mi + 1; ++kk) {
                    uint32_t a[4], bb[2];
                    load_a(a, Tm, LDM, 32 + 16 * mi, 32 + 8 * kk, g8, t4);
                    load_b(bb, x2, LDX2, 8 * kk, 8 * ni, g8, t4);
                    mma_tf32(e, a, bb);
                }
                store_tb_pair(sm, 32 + 16 * mi + g8, 8 * ni + 2 * t4, -e[0], -e[1], bet, gam);
                store_tb_pair(sm, 40 + 16 * mi + g8, 8 * ni + 2 * t4, -e[2], -e[3], bet, gam);
            }
            fence_proxy_async_smem();
            named_bar(kBarPrep, kNumPrep);
            if (pt == 0) arrive(&bars[B_TBREADY]);
            DBG_CLK(3, 6)
            // gates of the next chunk, while the W MMA of this one runs
            if (c + 1 < N) prep_gates(c + 1);
            DBG_CLK(3, 7)
            // ---- W (bf16, MN-major rows i) from W^T in TMEM (the MMAs of the previous chunk that read W
            //      and the bf16 state copy are done) ----
            if (!(ok = role_wait(&bars[B_WDONE], par, abort_flag, kBarPrep, kNumPrep))) break;
            if (c > 0 && !(ok = role_wait(&bars[B_M1ADONE], (c - 1) & 1, abort_flag, kBarPrep, kNumPrep))) break;
            if (c > 0 && !(ok = role_wait(&bars[B_M1BDONE], (c - 1) & 1, abort_flag, kBarPrep, kNumPrep))) break;
            tc_fence_after();
            DBG_CLK(3, 8)
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
            DBG_CLK(3, 9)
        }
    } else if (warp >= kChainWarp0) {
        // ============================== chain ==============================
        // two warps per TMEM lane quadrant: thread (j, ch) owns state row j and column half ch
        const int ct = tid - kChainWarp0 * 32;       // 0..255
        const int j = (warp & 3) * 32 + lane;        // TMEM lane / state row, 0..127
        const int ch = (warp - kChainWarp0) >> 2;    // column half
        float *dl = reinterpret_cast<float *>(sm + OFF_CG);  // [2][64] e^{g_C - g_s} per chunk parity
        float *f1 = dl + 128;                                // [2][64] gamma_t
        float *f2 = dl + 256;                                // [2][64] e^{g_t - c} (narrow chunk) or 1
        float *gcs = dl + 384;                               // [2]    gamma_C
        int *chain_flags = reinterpret_cast<int *>(dl + 388); // [2]
        bool ok = true;
        // entry state -> TMEM: S0 (or zero) for the first segment, the prefix-scanned entry state for
        // later segments, zero for transfer-B runs and the identity for transfer-M runs
        {
            const float *src = nullptr;
            if (kind == 0)
                src = (seg == 0) ? (p.S0 ? p.S0 + (bh * kD + j) * (int64_t)kD : nullptr)
                                 : p.S_entry + ((bh * (p.nseg - 1) + seg - 1) * kD + j) * (int64_t)kD;
#pragma unroll 1
            for (int piece = 0; piece < 2; ++piece) {
                const int col0 = ch * 64 + piece * 32;
                uint32_t r[32];
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    float4 v = src ? *reinterpret_cast<const float4 *>(src + col0 + i) : make_float4(0, 0, 0, 0);
                    r[i] = __float_as_uint(v.x);
                    r[i + 1] = __float_as_uint(v.y);
                    r[i + 2] = __float_as_uint(v.z);
                    r[i + 3] = __float_as_uint(v.w);
                }
                if (kind == 2) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint((col0 + i == j) ? 1.f : 0.f);
                }
                tmem_st32(tm + lb + TM_S + col0, r);
            }
            tmem_wait_st();
        }
        // chain gates of chunk cg into buffer cg & 1: dl_s = e^{g_C - g_s}, gamma_C and the output
        // factors; the narrow test repeats the prep role's computation on identical values, so
        // both roles take the same decision
        float la_next = 0.f;
        if (ct < 64 && (int64_t)c0 * kC + ct < T)
            la_next = p.log_alpha[((int64_t)b * T + (int64_t)c0 * kC + ct) * H + h];
        auto chain_gates = [&](int cg) {
            const int64_t t0g = (int64_t)(c0 + cg) * kC;
            const int ng = (T - t0g < kC) ? (int)(T - t0g) : kC;
            float *dlb = dl + (cg & 1) * 64;
            float s = 0.f;
            if (ct < 64) {
                const float x = (ct < ng) ? fmaxf(la_next, kLogAlphaFloor) : 0.f;
                s = chunk_cumsum(x, ct, chain_tmp, kBarChain, kNumChain);
                const int64_t tn = t0g + kC + ct;
                if (tn < T) la_next = p.log_alpha[((int64_t)b * T + tn) * H + h];
                dlb[ct] = s;
            } else {
                named_bar(kBarChain, kNumChain);  // the barrier inside chunk_cumsum
            }
            named_bar(kBarChain, kNumChain);
            const float g63 = dlb[63], cm = dlb[31];
            if (ct < 64) {
                const bool nr = __all_sync(0xffffffffu, fabsf(s - cm) < 60.f);
                if ((ct & 31) == 0) chain_flags[ct >> 5] = nr ? 1 : 0;
            }
            named_bar(kBarChain, kNumChain);
            const bool narrow = chain_flags[0] && chain_flags[1];
            if (ct < 64) {
                dlb[ct] = expf(g63 - s);
                f1[(cg & 1) * 64 + ct] = expf(s);
                f2[(cg & 1) * 64 + ct] = narrow ? expf(s - cm) : 1.f;
            }
            if (ct == 0) gcs[cg & 1] = expf(g63);
            named_bar(kBarChain, kNumChain);
        };
        // outputs of chunk cprev: o_t = f1_t O1_t + f2_t O2_t for this thread's column j and tokens
        // t in its half, staged as two 64x64 bf16 boxes in the TMA layout, written by two TMA stores
        auto write_out = [&](int cprev) {
            const float *f1c = f1 + (cprev & 1) * 64 + ch * 32, *f2c = f2 + (cprev & 1) * 64 + ch * 32;
            if (ct == 0) bulk_wait_read0();  // the previous chunk's stores have read the staging buffer
            named_bar(kBarChain, kNumChain);
            const int par = j & 1, colw = j - par;  // this lane writes column pair (colw, colw + 1)
            uint8_t *stage = sm + OFF_OST + (colw >> 6) * 8192;
            const uint32_t cbyte = (colw & 7) * 2, cchunk = (colw & 63) >> 3;
#pragma unroll 1
            for (int piece = 0; piece < 2; ++piece) {
                uint32_t r1[16], r2[16];
                tmem_ld16(tm + lb + TM_O + ch * 32 + piece * 16, r1);
                tmem_ld16(tm + lb + TM_O2 + ch * 32 + piece * 16, r2);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; i += 2) {
                    const int t = piece * 16 + i;
                    const float o0 = f1c[t] * __uint_as_float(r1[i]) + f2c[t] * __uint_as_float(r2[i]);
                    const float o1 = f1c[t + 1] * __uint_as_float(r1[i + 1]) + f2c[t + 1] * __uint_as_float(r2[i + 1]);
                    // even lanes keep row t and take the neighbour's column; odd lanes keep row t+1
                    const float send = par ? o0 : o1;
                    const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
                    const uint32_t word = par ? pack_bf16x2(recv, o1) : pack_bf16x2(o0, recv);
                    const int row = ch * 32 + t + par;
                    *reinterpret_cast<uint32_t *>(stage + sw128(row, cchunk) + cbyte) = word;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(kBarChain, kNumChain);
            if (ct == 0) {
                tma_store_4d(&tm_o, sm + OFF_OST, 0, h, (c0 + cprev) * kC, b);
                tma_store_4d(&tm_o, sm + OFF_OST + 8192, 64, h, (c0 + cprev) * kC, b);
                bulk_commit();
            }
        };
        chain_gates(0);
        for (int c = 0; c < N && ok; ++c) {
            const uint32_t par = c & 1;
            const float *dlc = dl + (c & 1) * 64 + ch * 32;
            DBG_CLK(4, 0)
            if (c > 0) {
                // the state update of the previous chunk is complete, and its output MMA is done
                // reading the bf16 state copy
                if (!(ok = role_wait(&bars[B_M2BDONE], (c - 1) & 1, abort_flag, kBarChain, kNumChain))) break;
                if (!(ok = role_wait(&bars[B_M1BDONE], (c - 1) & 1, abort_flag, kBarChain, kNumChain))) break;
                tc_fence_after();
            }
            DBG_CLK(4, 1)
            // ---- S -> bf16 operand copy; S <- gamma_C S (this thread: row j, 64 columns) ----
            {
                const float gC = gcs[c & 1];
#pragma unroll 1
                for (int piece = 0; piece < 2; ++piece) {
                    const int col0 = ch * 64 + piece * 32;
                    uint32_t r[32];
                    tmem_ld32(tm + lb + TM_S + col0, r);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 2)
                        pk[i >> 1] = pack_bf16x2(__uint_as_float(r[i]), __uint_as_float(r[i + 1]));
                    tmem_st16(tm + lb + TM_SB + col0 / 2, pk);
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * gC);
                    tmem_st32(tm + lb + TM_S + col0, r);
                }
                tmem_wait_st();
                tc_fence_before();
                named_bar(kBarChain, kNumChain);
                if (ct == 0) arrive(&bars[B_SREADY]);
            }
            DBG_CLK(4, 2)
            // ---- outputs of the previous chunk (frees the O accumulators) ----
            if (c > 0) {
                if (!(ok = role_wait(&bars[B_M2ADONE], (c - 1) & 1, abort_flag, kBarChain, kNumChain))) break;
                tc_fence_after();
                if (outputs) write_out(c - 1);  // ends with a chain barrier after the O reads
                if (ct == 0) arrive(&bars[B_OFREE]);
            }
            DBG_CLK(4, 3)
            if (!(ok = role_wait(&bars[B_M1ADONE], par, abort_flag, kBarChain, kNumChain))) break;
            tc_fence_after();
            DBG_CLK(4, 4)
            // ---- U^T (accumulated in TMEM) -> bf16 U^T and bf16 U^T diag(dl) (this thread: 32 tokens) ----
#pragma unroll 1
            for (int piece = 0; piece < 2; ++piece) {
                uint32_t u[16], pk[8];
                tmem_ld16(tm + lb + TM_DU + ch * 32 + piece * 16, u);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; i += 2)
                    pk[i >> 1] = pack_bf16x2(__uint_as_float(u[i]), __uint_as_float(u[i + 1]));
                tmem_st8(tm + lb + TM_UB + ch * 16 + piece * 8, pk);
#pragma unroll
                for (int i = 0; i < 16; i += 2)
                    pk[i >> 1] = pack_bf16x2(__uint_as_float(u[i]) * dlc[piece * 16 + i],
                                             __uint_as_float(u[i + 1]) * dlc[piece * 16 + i + 1]);
                tmem_st8(tm + lb + TM_UDB + ch * 16 + piece * 8, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            named_bar(kBarChain, kNumChain);
            if (ct == 0) arrive(&bars[B_UREADY]);
            DBG_CLK(4, 5)
            // gates of the next chunk, while this chunk's last MMAs run
            if (c + 1 < N) chain_gates(c + 1);
            DBG_CLK(4, 6)
        }
        if (ok && N > 0) {
            ok = role_wait(&bars[B_M2BDONE], (N - 1) & 1, abort_flag, kBarChain, kNumChain);
            if (ok) ok = role_wait(&bars[B_M2ADONE], (N - 1) & 1, abort_flag, kBarChain, kNumChain);
            tc_fence_after();
            if (ok && outputs) write_out(N - 1);
        }
        float *dst = nullptr;
        if (kind == 0)
            dst = (seg == p.nseg - 1 && p.S_final) ? p.S_final + (bh * kD + j) * (int64_t)kD : nullptr;
        else
            dst = (kind == 1 ? p.Bw : p.Mw) + ((bh * (p.nseg - 1) + seg) * kD + j) * (int64_t)kD;
        if (ok && dst) {
#pragma unroll 1
            for (int piece = 0; piece < 2; ++piece) {
                const int col0 = ch * 64 + piece * 32;
                uint32_t r[32];
                tmem_ld32(tm + lb + TM_S + col0, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4 *>(dst + col0 + i) =
                        make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]), __uint_as_float(r[i + 2]),
                                    __uint_as_float(r[i + 3]));
            }
        }
        if (ct == 0) bulk_wait0();  // every output store has completed
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) atomicExch(&g_tc_timeout, 1);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, 512);
    }
}

// ---------------------------------------------------------------- segment prefix
// Entry states of segments 1..nseg-1 from the segment transfers, in float32:
// S_{p+1} = S_p M_p + B_p with S_0 = S0 (or zero).  Rows of the state are
// independent, so one CTA owns 16 rows of one (b, h) and walks the segments
// in order.  A (b, h)'s transfers and entry states sit in consecutive slots;
// with a table (packed sequences, whose segment counts differ), CTA row x
// takes S0 [tab[x].x], slots tab[x].y .. tab[x].y + tab[x].z - 1; without
// one, (b, h) = x takes S0 [x] and slots x (nseg - 1) onwards.  The next
// needed M is bulk-copied into the second of two shared buffers while a step
// computes.  Where Mflag marks a transfer matrix as negligible (its bound is at
// most e^-40, see kNegligibleTransfer) the step is S_{p+1} = B_p: M_p is
// neither read nor multiplied, and all such steps are copied at once before
// the others run in order.
constexpr int kPrefixRows = 16;
constexpr int kPrefixThreads = 256;
constexpr int kPrefixLd = kD + 4;
constexpr size_t kPrefixSmem = (size_t)(2 * kD * kD + kPrefixRows * kPrefixLd) * sizeof(float) + 16;

__global__ void __launch_bounds__(kPrefixThreads, 1)
seg_prefix_kernel(const float *__restrict__ S0, const float *__restrict__ Bw, const float *__restrict__ Mw,
                  const int *__restrict__ Mflag, float *__restrict__ S_entry, int nseg,
                  const int4 *__restrict__ tab) {
    extern __shared__ __align__(128) float psm[];
    float *Ms = psm;                       // [2][128][128]
    float *Sr = psm + 2 * kD * kD;         // [16][kPrefixLd]
    uint64_t *full = reinterpret_cast<uint64_t *>(Sr + kPrefixRows * kPrefixLd);  // [2]
    int64_t bh, base;  // S0 row block and first slot
    int steps;
    if (tab) {
        const int4 w = tab[blockIdx.x];
        bh = w.x;
        base = w.y;
        steps = w.z;
    } else {
        bh = blockIdx.x;
        steps = nseg - 1;
        base = bh * steps;
    }
    const int r0 = blockIdx.y * kPrefixRows;
    const int tid = threadIdx.x;
    // this thread's row and columns ca..ca+3, cb..cb+3: consecutive threads read consecutive
    // 16-byte words of a row of M, without bank conflicts
    const int r = tid >> 4, ca = (tid & 15) * 4, cb = 64 + ca;
    auto needs_m = [&](int q) { return Mflag == nullptr || Mflag[base + q] == 0; };
    // the n-th matrix loaded goes to buffer n & 1 and completes phase (n >> 1) & 1 of full[n & 1]
    auto load_m = [&](int q, int n) {
        const float *M = Mw + (base + q) * (int64_t)kD * kD;
        float *dst = Ms + (n & 1) * kD * kD;
        fence_proxy_async_smem();  // the generic reads of this buffer two loads ago come first
        mbar_arrive_expect_tx(&full[n & 1], kD * kD * 4);
        for (int i = 0; i < 4; ++i) bulk_load(dst + i * 4096, M + i * 4096, 16384, &full[n & 1]);
    };
    // the first step at or after q that needs its M, or steps
    auto next_needed = [&](int q) {
        while (q < steps && !needs_m(q)) ++q;
        return q;
    };
    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_fence_init();
    }
    __syncthreads();
    int loaded = 0;  // matrices consumed so far
    // blocks with blockIdx.z > 0 only copy their share of the negligible steps (pass 1 below)
    int pending = blockIdx.z == 0 ? next_needed(0) : steps;  // the step whose M is in flight (steps: none)
    if (tid == 0 && pending < steps) load_m(pending, 0);
    for (int i = tid; i < kPrefixRows * (kD / 4); i += kPrefixThreads) {
        const int rr = i / (kD / 4), cc = (i % (kD / 4)) * 4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (S0) v = *reinterpret_cast<const float4 *>(S0 + (bh * kD + r0 + rr) * (int64_t)kD + cc);
        *reinterpret_cast<float4 *>(Sr + rr * kPrefixLd + cc) = v;
    }
    auto b_rows = [&](int q) { return Bw + ((base + q) * kD + r0 + r) * (int64_t)kD; };
    // pass 1: a step whose transfer matrix is negligible needs no state, S_{q+1} = B_q: all such
    // steps at once, spread over the gridDim.z blocks of these rows (steps z, z + gridDim.z, ...),
    // eight 16-byte loads in flight per thread
    if (Mflag) {
        constexpr int kUnits = kPrefixRows * (kD / 4);  // 16-byte units of this CTA's rows, per step
        const int zs = (int)gridDim.z, mine = (steps - (int)blockIdx.z + zs - 1) / zs;  // this block's steps
        const int total = mine * kUnits;
        for (int i0 = tid; i0 < total; i0 += 8 * kPrefixThreads) {
            float4 v[8];
            int64_t off[8];
            bool copy[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0 + u * kPrefixThreads;
                const int q = (int)blockIdx.z + (i / kUnits) * zs, rr = (i % kUnits) / (kD / 4),
                          cc = (i % (kD / 4)) * 4;
                copy[u] = i < total && !needs_m(q);
                off[u] = ((base + q) * kD + r0 + rr) * (int64_t)kD + cc;
                if (copy[u]) v[u] = *reinterpret_cast<const float4 *>(Bw + off[u]);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (copy[u]) *reinterpret_cast<float4 *>(S_entry + off[u]) = v[u];
        }
    }
    // pass 2: the steps that need their M, in order.  The state entering step q is S0 (q = 0), the
    // previous step's result still in Sr, or B_{q-1} when step q - 1 was negligible.
    int prev = -1;  // the step whose result Sr holds (-1: S0)
    while (pending < steps) {
        const int q = pending;
        // the next needed M goes into the other buffer, free since the step that read it ended
        const int nxt = next_needed(q + 1);
        if (tid == 0 && nxt < steps) load_m(nxt, loaded + 1);
        if (q > 0 && prev != q - 1) {
            __syncthreads();  // every thread is done with Sr
            for (int i = tid; i < kPrefixRows * (kD / 4); i += kPrefixThreads) {
                const int rr = i / (kD / 4), cc = (i % (kD / 4)) * 4;
                *reinterpret_cast<float4 *>(Sr + rr * kPrefixLd + cc) =
                    *reinterpret_cast<const float4 *>(Bw + ((base + q - 1) * kD + r0 + rr) * (int64_t)kD + cc);
            }
        }
        const float4 b0 = *reinterpret_cast<const float4 *>(b_rows(q) + ca);
        const float4 b1 = *reinterpret_cast<const float4 *>(b_rows(q) + cb);
        float acc[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
        // bounded wait; a timeout leaves the entry states unwritten rather than hanging
        const bool landed = mbar_wait(&full[loaded & 1], (loaded >> 1) & 1);
        if (!__syncthreads_and(landed)) break;  // also publishes the rows of Sr
        const float *M = Ms + (loaded & 1) * kD * kD;
#pragma unroll 4
        for (int k = 0; k < kD; ++k) {
            const float a = Sr[r * kPrefixLd + k];
            const float4 m0 = *reinterpret_cast<const float4 *>(M + k * kD + ca);
            const float4 m1 = *reinterpret_cast<const float4 *>(M + k * kD + cb);
            acc[0] = fmaf(a, m0.x, acc[0]); acc[1] = fmaf(a, m0.y, acc[1]);
            acc[2] = fmaf(a, m0.z, acc[2]); acc[3] = fmaf(a, m0.w, acc[3]);
            acc[4] = fmaf(a, m1.x, acc[4]); acc[5] = fmaf(a, m1.y, acc[5]);
            acc[6] = fmaf(a, m1.z, acc[6]); acc[7] = fmaf(a, m1.w, acc[7]);
        }
        ++loaded;
        __syncthreads();  // every thread is done reading this step's rows and M
        *reinterpret_cast<float4 *>(Sr + r * kPrefixLd + ca) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        *reinterpret_cast<float4 *>(Sr + r * kPrefixLd + cb) = make_float4(acc[4], acc[5], acc[6], acc[7]);
        float *dst = S_entry + ((base + q) * kD + r0 + r) * (int64_t)kD;
        *reinterpret_cast<float4 *>(dst + ca) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        *reinterpret_cast<float4 *>(dst + cb) = make_float4(acc[4], acc[5], acc[6], acc[7]);
        prev = q;
        pending = nxt;
    }
}

// ---------------------------------------------------------------- host side
}  // namespace

// Reads and clears the word the kernels of this file set when a bounded wait gave up
// (synchronous: it follows the work already enqueued on the legacy default stream's device).
bool take_tc_timeout() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc_timeout, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (v) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_tc_timeout, &zero, sizeof(int));
    }
    return v != 0;
}

#ifdef GDN_TC_DEBUG
extern "C" int gdn_debug_set_dump(float *ptr) {
    return cudaMemcpyToSymbol(g_dbg, &ptr, sizeof(ptr)) == cudaSuccess ? 0 : 1;
}
#endif

bool fwd_tc_supported(const FwdProblem &p) {
    return p.dtype == 1 && p.dk == kD && p.dv == kD && p.chunk == kC && p.T <= (int64_t)INT32_MAX / 2 &&
           p.B <= (int64_t)INT32_MAX && p.H <= (int64_t)INT32_MAX;
}

// Segments per (b, h): the count minimising a wave model of the passes, in
// units of half a chunk step of one CTA: transfers (nseg - 1 CTAs per head
// when both runs of a segment share a CTA, else 2 (nseg - 1)) and outputs
// (nseg CTAs per head), each CTA over ceil(chunks / nseg) chunks, plus the
// sequential prefix over segments (about half a chunk step per segment).
// GDN_SEGMENTS overrides the choice.
int fwd_tc_segments(const FwdProblem &p, int sm_count, bool paired_transfers) {
    const int64_t chunks = (p.T + kC - 1) / kC, heads = p.B * p.H;
    if (chunks <= 0 || heads <= 0) return 1;
    const char *env = getenv("GDN_SEGMENTS");
    if (env && atoi(env) >= 1) {
        int want = atoi(env);
        if (want > chunks) want = (int)chunks;
        const int64_t len = (chunks + want - 1) / want;
        return (int)((chunks + len - 1) / len);
    }
    auto waves = [&](int64_t ctas) { return (ctas + sm_count - 1) / sm_count; };
    int best = 1;
    int64_t best_cost = 2 * waves(heads) * chunks;
    for (int nseg = 2; nseg <= 64; ++nseg) {
        const int64_t len = (chunks + nseg - 1) / nseg;
        if (len < 4) break;
        const int64_t real = (chunks + len - 1) / len;
        const int64_t tr = (paired_transfers ? 1 : 2) * heads * (real - 1);
        const int64_t cost = 2 * (waves(tr) + waves(heads * real)) * len + (real - 1);
        if (cost < best_cost) {
            best_cost = cost;
            best = (int)real;
        }
    }
    return best;
}

size_t fwd_tc_workspace_bytes(const FwdProblem &p, int nseg) {
    if (nseg <= 1) return 0;
    return (size_t)3 * (size_t)(p.B * p.H / p.lead) * (size_t)(nseg - 1) * kD * kD * sizeof(float);
}

cudaError_t launch_seg_prefix(const float *S0, const float *Bw, const float *Mw, const int *Mflag, float *S_entry,
                              int64_t heads, int nseg, cudaStream_t stream, const int4 *tab) {
    static std::atomic<uint64_t> pconf{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(pconf.load() & bit)) {
        cudaError_t e =
            cudaFuncSetAttribute(seg_prefix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPrefixSmem);
        if (e != cudaSuccess) return e;
        pconf.fetch_or(bit);
    }
    {
        TimedLaunch tl_(GDN_KERNEL_PREFIX, stream);
        // with flags and many steps, up to three more blocks per row block share the copies of the
        // negligible steps
        const int zsi = Mflag ? (nseg - 1) / 8 : 1;
        const unsigned zs = zsi < 1 ? 1u : (zsi > 4 ? 4u : (unsigned)zsi);
        seg_prefix_kernel<<<dim3((unsigned)heads, kD / kPrefixRows, zs), kPrefixThreads, kPrefixSmem, stream>>>(
            S0, Bw, Mw, Mflag, S_entry, nseg, tab);
    }
    return cudaGetLastError();
}

cudaError_t launch_fwd_tc(const FwdProblem &p, int nseg, void *workspace, cudaStream_t stream) {
    CUtensorMap mq, mk, mv, mo;
    if (!make_map_bthd(&mq, p.q, p.B, p.T, p.H) || !make_map_bthd(&mk, p.k, p.B, p.T, p.H) ||
        !make_map_bthd(&mv, p.v, p.B, p.T, p.H) || !make_map_bthd(&mo, p.out, p.B, p.T, p.H))
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
    const int64_t chunks = (p.T + kC - 1) / kC, heads = p.B * p.H;
    if (nseg < 1) nseg = 1;
    a.seg_len = (int)((chunks + nseg - 1) / nseg);
    a.nseg = (int)((chunks + a.seg_len - 1) / a.seg_len);
    a.S_entry = nullptr;
    a.Bw = a.Mw = nullptr;
    if (a.nseg > 1) {
        if (!workspace) return cudaErrorInvalidValue;
        const size_t per = (size_t)heads * (a.nseg - 1) * kD * kD;
        a.Bw = static_cast<float *>(workspace);
        a.Mw = a.Bw + per;
        float *entry = a.Mw + per;
        a.S_entry = entry;
        // phase 1: segment transfers of segments 0..nseg-2
        a.mode = 1;
        {
            TimedLaunch tl_(GDN_KERNEL_TRANSFER, stream);
            fwd_tc_kernel<<<(unsigned)(heads * (a.nseg - 1) * 2), kThreadsTc, SMEM_TC, stream>>>(mq, mk, mv, mo, a);
        }
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        // phase 2: entry states of segments 1..nseg-1
        e = launch_seg_prefix(p.S0, a.Bw, a.Mw, nullptr, entry, heads, a.nseg, stream);
        if (e != cudaSuccess) return e;
    }
    // outputs of every segment from its entry state
    a.mode = 0;
    {
        TimedLaunch tl_(GDN_KERNEL_FUSED, stream);
        fwd_tc_kernel<<<(unsigned)(heads * a.nseg), kThreadsTc, SMEM_TC, stream>>>(mq, mk, mv, mo, a);
    }
    return cudaGetLastError();
}

}  // namespace gdn
