// fwd_split.cu -- chunkwise gated-delta forward on the 5th-generation tensor
// cores in two kernels: a chunk-parallel prep kernel and a chain kernel.
// bf16 q/k/v, dk = dv = 128, chunk C = 64.
//
// Operation: "ATMA: Long-Context Language Modeling via Polar Attention and
// Gated-Delta Compression Memory", Sec. 3.3 (gated-delta memory equation),
// computed in the chunkwise UT-transform form of the works that paper cites
// for the memory ("Gated delta networks"; "Parallelizing linear transformers
// with the delta rule over sequence length").  Per chunk of 64 tokens with
// chunk-local log-decay cumsum g_t, gamma_t = e^{g_t}, dl_s = e^{g_C - g_s}:
//
//   prep kernel (independent of the state; every chunk of every (b, h) in
//   parallel, persistent CTAs, three per SM):
//     G   = [Q; K] K^T                                          (tcgen05, M = 128)
//     P   = lower(e^{g_t - g_s} (Q K^T)_ts)                     -> workspace, bf16
//     A   = strict_lower(beta_t e^{g_t - g_s} (K K^T)_ts)
//     T   = (I + A)^{-1}: 16x16 diagonal blocks by substitution, merged 16 -> 32 -> 64
//           with warp-level TF32 MMAs (fp32 accumulation)
//     TB  = T diag(beta)                                        -> workspace, bf16
//     W^T = K^T (T diag(beta gamma))^T                          (tcgen05) -> workspace, bf16
//
//   chain kernel (sequential over the chunks of one (b, h) or segment; for long
//   sequences with few heads, the transfers of the segments come first from the
//   paired transfer kernel, and their prefix gives each segment's entry state):
//     Ut^T = V^T TB^T                               (tcgen05, off the critical path)
//     U^T  = Ut^T - S W^T                           (accumulated onto Ut^T, B negated)
//     S   <- gamma_C S + U^T (diag(dl) K)           (float32 state in tensor memory)
//     O^T  = S (diag(gamma) Q)^T + U^T P^T          (one accumulator, off the critical path)
//
// e^{g_t - g_s} is formed as e^{g_t - c} e^{c - g_s} (c = g_31) when every
// |g_t - c| < 60 in the chunk, else element by element; both are exact to a
// few ulp.  Workspace: per chunk P (8 KB), TB (8 KB) and W^T (16 KB), each a
// bf16 tile of 128-byte rows written and read by TMA with 128-byte swizzle,
// and the chunk's gates gamma_t and dl_s (512 B, float32).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <stdlib.h>

#include <string.h>

#include <algorithm>
#include <atomic>
#include <functional>
#include <queue>
#include <vector>

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
constexpr size_t kTileP = 64 * 64 * 2, kTileTB = 64 * 64 * 2, kTileW = 128 * 64 * 2;
// Gate record of one chunk, float32: [0, 64) gamma_t, [64, 128) dl_s = e^{g_63 - g_s}, [128] gamma_C,
// [129] rho_C, the chunk's transfer bound gamma_C prod_t max(1, |1 - beta_t |k_t|^2|) (see
// kNegligibleTransfer), [130, 132) zero.  With the input stage fused, gamma_t carries 1 / |q_t| and
// dl_s 1 / |k_s|, the scales of diag(gamma) Q and diag(dl) K in the chain, and |k_t| is the
// normalised key's.
constexpr int kRecFloats = 132;
constexpr size_t kGateRec = kRecFloats * 4;
constexpr size_t kWsPerChunk = kTileP + kTileTB + kTileW + kGateRec;  // 32.5 KB

__device__ int g_split_timeout;  // set when a bounded mbarrier wait gives up

#ifdef GDN_TC_DEBUG
// Debug builds only: per-phase clock stamps of CTA 0 for its first 8 work
// items, 8 rows of 16 int64 per item.
__device__ long long *g_split_dbg;
#define SDBG_INIT long long *const dbgp = (blockIdx.x == 0) ? g_split_dbg : nullptr;
#define SDBG(row, i) \
    if (dbgp != nullptr && it < 8) dbgp[(it * 8 + (row)) * 16 + (i)] = clock64();
#else
#define SDBG_INIT
#define SDBG(row, i)
#endif

// ============================================================================
// prep kernel
// ============================================================================
constexpr int kPrepThreads = 288;  // warp 0: TMA + MMA issue; warps 1-8: prep role
constexpr int kNumPrep = 256;
constexpr int kBarP = 1;
constexpr int LDM = 68;   // row stride (floats) of the fp32 64x64 tiles
constexpr int LDX2 = 40;  // row stride of the 32->64 merge scratch

// 73 KB in all, so that three CTAs share an SM.
constexpr uint32_t PO_QK = 0;        // 32 KB: per 64-column block j: [Q 8 KB | K 8 KB]
constexpr uint32_t PO_P = 0;         // 8 KB  P [t][s] staging, in the Q block 0 once G is done
constexpr uint32_t PO_TB = 32768;    // 8 KB  T diag(beta)       [t][s], 128-byte swizzle
constexpr uint32_t PO_TBG = 40960;   // 8 KB  T diag(beta gamma) [t][s]
constexpr uint32_t PO_AM = 49152;    // 17 KB A fp32 [64][LDM], overwritten by T in place; after the inverse:
                                     //       W^T bf16 [128][64] staging
constexpr uint32_t PO_XS = 66560;    // 5 KB  merge scratch
constexpr uint32_t PO_PG = 71680;    // gates per item parity: g, beta, gamma, e^{g-c}, e^{c-g}, beta gamma
                                     // (2 x 6 x 64)
constexpr int kPG = 384;             // floats per parity
constexpr uint32_t PO_NRM = 74752;   // input stage: 1 / |q_t|, 1 / |k_s|, g_s - ln(1 / |k_s|) (3 x 64)
constexpr uint32_t PO_BARS = 75520;  // mbarriers
constexpr uint32_t PO_MISC = 75584;  // tmem slot, abort flag, scan scratch, flags
constexpr uint32_t SMEM_PREP = 75648 + 1024;
constexpr int kPrepCtasPerSm = 3;
static_assert(PO_PG + 2 * kPG * 4 <= PO_NRM && PO_NRM + 3 * 64 * 4 <= PO_BARS,
              "prep-kernel gate buffers overflow their slot");
static_assert(kPrepCtasPerSm * (SMEM_PREP + 1024) <= 233472, "three prep CTAs no longer fit an SM");
constexpr int kBarMerge = 2;  // named barrier of the four 16->32 merge warps
constexpr int kBarGates = 3;  // named barrier of the two warps that form an item's gates

constexpr uint32_t TP_G = 0;   // 64 columns: [Q;K] K^T
constexpr uint32_t TP_W = 64;  // 64 columns: W^T

constexpr uint32_t IDESC_G = instr_desc_bf16(128, 64, 0, 0);     // [Q;K] . K^T
constexpr uint32_t IDESC_MN64 = instr_desc_bf16(128, 64, 1, 0);  // K^T / V^T (MN-major A) . T^T

enum PBar { PB_QFULL = 0, PB_KFULL, PB_GDONE, PB_GFREE, PB_TBREADY, PB_WDONE, PB_QFREE, PB_COUNT };

static_assert(PB_COUNT * 8 <= PO_MISC - PO_BARS, "prep-kernel mbarriers overflow their shared-memory slot");

// Packed variable-length sequences: chunk i of the packed tensor starts at
// token ctab[i].x and has ctab[i].y tokens (the last chunk of a sequence may be
// partial); work item i * H + h is chunk i of head h.
struct PrepArgs {
    const float *log_alpha, *beta;
    float *gate_rec;  // [items][kRecFloats]
    int64_t T, H;
    int64_t items;     // B * H * chunks, or (packed chunks) * H
    int chunks;        // chunks per (b, h) (fixed-length problems)
    const int2 *ctab;  // packed chunk table, or nullptr for fixed-length problems
    int raw_inputs;    // q, k not yet L2-normalised; log_alpha, beta hold the gate logits
    int group;         // grouped heads: k and the gates have H / group heads (head h / group)
    // one memory per key-value head (lead = group): only the items of query heads h % lead == 0 feed
    // the chain, so the others form P and their gate record alone (no inverse, TB or W^T)
    int lead;
    // or nullptr: T = (I + A)^{-1} of every item, bf16 [items][64][64] row-major (the backward's
    // recompute); only the lower triangle is written, the caller zeroes the rest
    __nv_bfloat16 *t_out;
};

// Writes entries (row, col) and (row, col + 1) (col even) of T diag(beta) and T diag(bgk) into
// their bf16 K-major 128-byte-swizzled tiles, and of T itself into `tout` (row-major, or nullptr).
__device__ __forceinline__ void store_tb_tbg(uint8_t *tb, uint8_t *tbg, int row, int col, float v0, float v1,
                                             const float *bet, const float *bgk, __nv_bfloat16 *tout) {
    const uint32_t off = sw128(row, col >> 3) + (col & 7) * 2;
    *reinterpret_cast<uint32_t *>(tb + off) = pack_bf16x2(v0 * bet[col], v1 * bet[col + 1]);
    *reinterpret_cast<uint32_t *>(tbg + off) = pack_bf16x2(v0 * bgk[col], v1 * bgk[col + 1]);
    if (tout) *reinterpret_cast<uint32_t *>(tout + row * 64 + col) = pack_bf16x2(v0, v1);
}

// kLead: one memory per key-value head (PrepArgs::lead > 1), with P-only items; a separate
// instantiation, so that the plain forward's kernel carries none of its branches.
template <bool kLead>
__global__ void __launch_bounds__(kPrepThreads, kPrepCtasPerSm)
fwd_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_tb,
                const __grid_constant__ CUtensorMap tm_w, PrepArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + PO_BARS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + PO_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + PO_MISC + 4);
    float *scan_tmp = reinterpret_cast<float *>(sm + PO_MISC + 8);
    int *nflags = reinterpret_cast<int *>(sm + PO_MISC + 16);  // [2 parities][2 warps]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t T = p.T, H = p.H;
    const int Hkv = (int)H / p.group;  // key-value heads (grouped heads), H otherwise
    SDBG_INIT
    // work items of this CTA: global chunk ids blockIdx.x, blockIdx.x + gridDim.x, ...
    const int nit = (blockIdx.x < p.items) ? (int)((p.items - 1 - blockIdx.x) / gridDim.x + 1) : 0;
    // items < 2^24 (checked on the host), so 32-bit index arithmetic suffices
    auto item = [&](int it) -> uint32_t { return blockIdx.x + (uint32_t)it * gridDim.x; };
    // (b, h, first token) of work item `it`
    // (b, h, first token, tokens) of work item `it`
    auto coords = [&](int it, int &b, int &h, int &t0, int &nt) {
        const uint32_t gi = item(it);
        if (p.ctab) {
            const uint32_t cid = gi / (uint32_t)H;
            const int2 e = p.ctab[cid];
            b = 0;
            h = (int)(gi - cid * (uint32_t)H);
            t0 = e.x;
            nt = e.y;
        } else {
            const uint32_t bh = gi / (uint32_t)p.chunks;
            const uint32_t hh = (uint32_t)H;
            b = (int)(bh / hh);
            h = (int)(bh - (uint32_t)b * hh);
            t0 = (int)(gi - bh * (uint32_t)p.chunks) * kC;
            nt = (T - t0 < kC) ? (int)(T - t0) : kC;
        }
    };
    // items that form P and the gate record alone
    auto p_only = [&](int it) -> bool {
        if (!kLead) return false;
        int b, h, t0, nt;
        coords(it, b, h, t0, nt);
        return h % p.lead != 0;
    };
    const uint32_t sbase = smem_u32(sm);

    if (tid == 0) {
        for (int i = 0; i < PB_COUNT; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;
    const uint32_t lb = (uint32_t)((warp & 3) * 32) << 16;  // this warp's TMEM lane quadrant

    if (warp == 0) {
        // ============================ issuer ============================
        if (lane == 0) {
            auto load_q = [&](int it) {
                int b, h, t0, nt;
                coords(it, b, h, t0, nt);
                mbar_arrive_expect_tx(&bars[PB_QFULL], 2 * 8192);
                for (int blk = 0; blk < 2; ++blk)
                    tma_load_4d(sm + PO_QK + blk * 16384, &tm_q, &bars[PB_QFULL], blk * 64, h, t0, b);
            };
            auto load_k = [&](int it) {
                int b, h, t0, nt;
                coords(it, b, h, t0, nt);
                mbar_arrive_expect_tx(&bars[PB_KFULL], 2 * 8192);
                for (int blk = 0; blk < 2; ++blk)
                    tma_load_4d(sm + PO_QK + blk * 16384 + 8192, &tm_k, &bars[PB_KFULL], blk * 64, h / p.group, t0,
                                b);
            };
            bool ok = true;
            if (nit > 0) {
                load_q(0);
                load_k(0);
            }
            uint32_t nw = 0;  // items with W^T so far (the phases of TBREADY and WDONE)
            for (int it = 0; it < nit && ok; ++it) {
                const uint32_t par = it & 1;
                SDBG(0, 0)
                if (!(ok = wait_bar(&bars[PB_QFULL], par, abort_flag))) break;
                if (!(ok = wait_bar(&bars[PB_KFULL], par, abort_flag))) break;
                if (it > 0 && !(ok = wait_bar(&bars[PB_GFREE], (it - 1) & 1, abort_flag))) break;
                SDBG(0, 1)
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t a = sbase + PO_QK + (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_ss(tm + TP_G, smem_desc_sw128(a, 16, 1024), smem_desc_sw128(a + 8192, 16, 1024), IDESC_G,
                           kk > 0);
                }
                mma_commit(&bars[PB_GDONE]);
                SDBG(0, 2)
                if (p_only(it)) {
                    // the Q block is free once the P tile staged in it has been stored, K once G is done
                    if (!(ok = wait_bar(&bars[PB_QFREE], par, abort_flag))) break;
                    if (it + 1 < nit) load_q(it + 1);
                    if (!(ok = wait_bar(&bars[PB_GDONE], par, abort_flag))) break;
                    if (it + 1 < nit) load_k(it + 1);
                    continue;
                }
                const uint32_t wpar = kLead ? (nw & 1) : par;  // every item has W^T unless kLead
                if (!(ok = wait_bar(&bars[PB_TBREADY], wpar, abort_flag))) break;
                SDBG(0, 3)
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss(tm + TP_W, smem_desc_sw128(sbase + PO_QK + 8192 + kk * 2048, 16384, 1024),
                           smem_desc_sw128(sbase + PO_TBG + kk * 32, 16, 1024), IDESC_MN64, kk > 0);
                mma_commit(&bars[PB_WDONE]);
                // the Q block is free once the P tile staged in it has been stored, K once W^T is done
                if (!(ok = wait_bar(&bars[PB_QFREE], par, abort_flag))) break;
                if (it + 1 < nit) load_q(it + 1);
                if (!(ok = wait_bar(&bars[PB_WDONE], wpar, abort_flag))) break;
                if (it + 1 < nit) load_k(it + 1);
                if (kLead) ++nw;
                SDBG(0, 4)
            }
        }
        __syncwarp();
    } else {
        // ============================== prep ==============================
        const int pt = tid - 32;          // 0..255
        const int pw = pt >> 5;           // role warp 0..7
        const int ch = pw >> 2;           // column half of the TMEM epilogues
        const int g8 = lane >> 2, t4 = lane & 3;  // MMA fragment coordinates
        float *Am = reinterpret_cast<float *>(sm + PO_AM);
        float *Tm = Am;  // T overwrites A block by block (see the merge steps)
        float *Xs = reinterpret_cast<float *>(sm + PO_XS);
        bool ok = true;
        // the upper triangles of the bf16 T tiles are never written below: zero both tiles once
#pragma unroll
        for (int i = 0; i < 4; ++i) reinterpret_cast<uint4 *>(sm + PO_TB)[pt + 256 * i] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
        // gates of work item `it` into buffer it & 1 (threads pt < 64 hold token pt)
        float la_next = 0.f, be_next = 0.f;
        // gates of token t of work item `it`; -1 past the chunk's tokens (they act as alpha = 1,
        // beta = 0, so they leave the chunk's recurrence unchanged)
        auto gate_index = [&](int it, int t) -> int64_t {
            int b, h, t0, nt;
            coords(it, b, h, t0, nt);
            if (t >= nt) return -1;
            return ((int64_t)b * T + t0 + t) * Hkv + (p.group == 1 ? h : h / p.group);
        };
        if (nit > 0 && pt < 64) {
            const int64_t x = gate_index(0, pt);
            if (x >= 0) {
                la_next = p.log_alpha[x];
                be_next = p.beta[x];
            }
        }
        // (threads pt < 64 alone, with their own barrier; the role's next 256-thread barrier, which
        // every caller reaches before the buffer is read, publishes what they write)
        auto prep_gates = [&](int it) {
            float *gb = reinterpret_cast<float *>(sm + PO_PG) + (it & 1) * kPG;
            if (pt < 64) {
                const bool valid = gate_index(it, pt) >= 0;
                float la = la_next, be = be_next;
                if (p.raw_inputs) {
                    // the input stage: log alpha = -softplus(x_alpha), beta = sigmoid(x_beta)
                    la = -(fmaxf(la, 0.f) + log1pf(expf(-fabsf(la))));
                    be = 1.f / (1.f + expf(-be));
                }
                const float x = valid ? fmaxf(la, kLogAlphaFloor) : 0.f;
                gb[64 + pt] = valid ? be : 0.f;
                const float s = chunk_cumsum(x, pt, scan_tmp, kBarGates, 64);
                SDBG(1, 8)
                gb[pt] = s;
                if (it + 1 < nit) {
                    const int64_t xn = gate_index(it + 1, pt);
                    la_next = xn >= 0 ? p.log_alpha[xn] : 0.f;
                    be_next = xn >= 0 ? p.beta[xn] : 0.f;
                }
                named_bar(kBarGates, 64);
                SDBG(1, 9)
                const float gt = gb[pt], cm = gb[31];
                const float gm = expf(gt);
                gb[128 + pt] = gm;
                gb[192 + pt] = expf(gt - cm);
                gb[256 + pt] = expf(cm - gt);
                gb[320 + pt] = gb[64 + pt] * gm;
                if (!p.raw_inputs) {
                    // the chunk's gate record: gamma_t, dl_s, gamma_C (with the input stage fused it is
                    // written once the norms are known)
                    float *rec = p.gate_rec + (int64_t)item(it) * kRecFloats;
                    rec[pt] = gm;
                    rec[64 + pt] = expf(gb[63] - gt);
                    // [128] gamma_C, [130, 132) zero; [129] is written after the G epilogue
                    if (pt >= 60 && pt != 62) rec[128 + 63 - pt] = (pt == 63) ? gb[63 + 128] : 0.f;
                }
                // e^{g_t - g_s} = e^{g_t - c} e^{c - g_s} while every |g_t - c| < 60, so that
                // neither factor overflows
                const bool nr = __all_sync(0xffffffffu, fabsf(gt - cm) < 60.f);
                if (lane == 0) nflags[(it & 1) * 2 + (pt >> 5)] = nr ? 1 : 0;
            }
        };
        if (nit > 0) prep_gates(0);
        uint32_t nw = 0;  // items with W^T so far (the phases of WDONE)
        for (int it = 0; it < nit && ok; ++it) {
            const uint32_t par = it & 1;
            const int gi = (int)item(it);
            const bool ponly = p_only(it);
            __nv_bfloat16 *const tout = p.t_out ? p.t_out + (int64_t)gi * 4096 : nullptr;
            float *g = reinterpret_cast<float *>(sm + PO_PG) + par * kPG;
            // beta, gamma, e^{g - c}, e^{c - g}, beta gamma (the last two carry 1 / |k_s| once the input
            // stage below has run)
            const float *bet = g + 64, *gam = g + 128, *ea = g + 192, *eb = g + 256, *bgm = g + 320;
            // the stores of the previous item have finished reading P, TB and the W^T staging
            if (pt == 0) {
                SDBG(1, 14)
                bulk_wait_read0();
                SDBG(1, 15)
            }
            SDBG(1, 0)
            // with the input stage fused these threads read the Q and K rows too: they also observe the
            // loads' own barriers (whose phases of this item completed before the G MMA was issued)
            {
                bool w = wait_bar(&bars[PB_GDONE], par, abort_flag);
                if (p.raw_inputs)
                    w = w && wait_bar(&bars[PB_QFULL], par, abort_flag) && wait_bar(&bars[PB_KFULL], par, abort_flag);
                if (!(ok = bar_and(kBarP, kNumPrep, w))) break;
            }
            tc_fence_after();
            // this item's gates and flags, published by the barrier above
            const bool narrow = nflags[par * 2] && nflags[par * 2 + 1];
            SDBG(1, 1)
            // ---- with the input stage fused: 1 / |q_t| and 1 / |k_s| (the thread pair of a row of
            //      [Q; K] reads its two 64-column boxes), folded into this item's gate buffers in place:
            //      e^{c - g_s} and beta_s gamma_s take 1 / |k_s|; the record's gamma_t takes 1 / |q_t|
            //      and dl_s 1 / |k_s|; the rows' factor enters the G epilogue below ----
            float *rq = reinterpret_cast<float *>(sm + PO_NRM), *rk = rq + 64, *gkn = rq + 128;
            const float *gk = p.raw_inputs ? gkn : g;
            if (p.raw_inputs) {
                const int r = pt >> 1, box = pt & 1;
                const uint4 *rowp =
                    reinterpret_cast<const uint4 *>(sm + PO_QK + box * 16384 + (r >> 6) * 8192 + (r & 63) * 128);
                // the 16-byte chunks in an order rotated by row and box, so that the eight lanes of
                // each quarter warp read eight different bank groups
                float ss = 0.f;
#pragma unroll 1
                for (int u = 0; u < 8; ++u) {
                    const uint4 w4 = rowp[(u + r + 4 * box) & 7];
                    const uint32_t ws[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ws[e]));
                        ss = fmaf(x.x, x.x, fmaf(x.y, x.y, ss));
                    }
                }
                ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                const float inv = rsqrtf(ss + kNormEps);
                float *rec = p.gate_rec + (int64_t)gi * kRecFloats;
                if (box == 0) {
                    if (r < 64) {
                        rq[r] = inv;
                        rec[r] = g[128 + r] * inv;  // gamma_t / |q_t|
                    } else {
                        const int c = r - 64;
                        rk[c] = inv;
                        gkn[c] = g[c] - logf(inv);
                        rec[64 + c] = expf(g[63] - g[c]) * inv;  // dl_s / |k_s|
                        g[256 + c] *= inv;
                        g[320 + c] *= inv;
                    }
                } else if (pt < 8 && (pt >> 1) != 1) {
                    rec[128 + (pt >> 1)] = (pt == 1) ? g[128 + 63] : 0.f;  // [128] gamma_C, [130, 132) 0
                }
                named_bar(kBarP, kNumPrep);
            }
            // ---- epilogue of G: rows 0..63 -> P (bf16), rows 64..127 -> A (fp32; not for P-only items);
            //      columns by half ----
            if ((warp & 3) < 2 || !ponly) {
                const int m = (warp & 3) * 32 + lane;  // TMEM lane = row of [Q; K]
                const int t = m & 63;
                // with the input stage fused, the factors 1 / |q_t| (rows of P) or 1 / |k_t| (rows of A)
                // and 1 / |k_s| enter through the decays: e^{g_t - g_s} -> e^{(g_t + ln rf_t) - (g_s - ln rk_s)}
                const float rf = p.raw_inputs ? ((m < 64) ? rq[t] : rk[t]) : 1.f;
                const float gt = p.raw_inputs ? g[t] + logf(rf) : g[t], at = ea[t] * rf, bt = bet[t];
#pragma unroll 1
                for (int piece = 0; piece < 2; ++piece) {
                    const int s0 = ch * 32 + piece * 16;
                    uint32_t r[16];
                    tmem_ld16(tm + lb + TP_G + s0, r);
                    tmem_wait_ld();
                    // e^{g_t - g_s} for the 16 columns s of this piece; in a wide chunk, __expf's few-ulp
                    // relative error (larger for large |x|, where the value is far below the bf16
                    // rounding of P and the TF32 inverse) does not show at the precision of the path
                    float d[16];
                    if (narrow) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) d[i] = at * eb[s0 + i];
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) d[i] = __expf(gt - gk[s0 + i]);
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
                            *reinterpret_cast<uint4 *>(sm + PO_P + sw128(t, (s0 >> 3) + cc)) =
                                make_uint4(pk[cc * 4], pk[cc * 4 + 1], pk[cc * 4 + 2], pk[cc * 4 + 3]);
                    } else {
                        // the diagonal beta_t |k_t|^2 (normalised key with the input stage fused) gives the
                        // token's transfer factor max(1, |1 - beta_t |k_t|^2|), reduced into rho_C below
                        float diag = 0.f;
#pragma unroll
                        for (int i = 0; i < 16; i += 4) {
                            float v[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float x = bt * d[i + e] * __uint_as_float(r[i + e]);
                                v[e] = (s0 + i + e < t) ? x : 0.f;
                                diag = (s0 + i + e == t) ? x : diag;
                            }
                            *reinterpret_cast<float4 *>(Am + t * LDM + s0 + i) = make_float4(v[0], v[1], v[2], v[3]);
                        }
                        if (t >= s0 && t < s0 + 16) Xs[t] = fmaxf(1.f, fabsf(1.f - diag));
                    }
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            named_bar(kBarP, kNumPrep);
            if (pt == 0) {
                arrive(&bars[PB_GFREE]);
                SDBG(1, 10)
                tma_store_2d(&tm_p, sm + PO_P, 0, (int)(gi * 64));
                bulk_commit();
                SDBG(1, 11)
            }
            if (ponly) {
                // the Q block is free once the P store has read its staging
                if (pt == 0) {
                    bulk_wait_read0();
                    arrive(&bars[PB_QFREE]);
                }
                if (it + 1 < nit) prep_gates(it + 1);
                continue;
            }
            SDBG(1, 2)
            // ---- T = (I + A)^{-1} ----
            // (1) 16x16 diagonal blocks by substitution: role warps 0..3, a column per lane, written over
            //     the block of A once every lane of the warp has read it.  Above the diagonal blocks A
            //     is zero, as T is.
            if (pw < 4) {
                const int o = pw * 16;
                float x[16];
                if (lane < 16) {
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
                }
                __syncwarp();
                if (lane < 16) {
#pragma unroll
                    for (int rr = 0; rr < 16; ++rr) Tm[(o + rr) * LDM + o + lane] = x[rr];
                }
            } else if (pw == 4) {
                // rho_C = gamma_C prod_t max(1, |1 - beta_t |k_t|^2|) into the gate record
                float pr = Xs[lane] * Xs[lane + 32];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) pr *= __shfl_xor_sync(0xffffffffu, pr, o);
                if (lane == 0) p.gate_rec[(int64_t)gi * kRecFloats + 129] = g[128 + 63] * pr;
            }
            __syncwarp();
            named_bar(kBarP, kNumPrep);
            SDBG(1, 3)
            // (2) 16 -> 32: T_10 = -T_11 (A_10 T_00) inside each 32x32 diagonal block; one warp per
            //     (block, 8-column tile).  Meanwhile role warps 4..7 write the four 16x16 diagonal
            //     blocks as bf16 T diag(beta) and T diag(beta gamma), one 16-byte unit per thread
            if (pw >= 4) {
                const int idx = pt - 128, row = idx >> 1, col = (row & ~15) + (idx & 1) * 8;
                const float4 x0 = *reinterpret_cast<const float4 *>(Tm + row * LDM + col);
                const float4 x1 = *reinterpret_cast<const float4 *>(Tm + row * LDM + col + 4);
                const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                uint32_t wb[4], wg[4];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    wb[e >> 1] = pack_bf16x2(xv[e] * bet[col + e], xv[e + 1] * bet[col + e + 1]);
                    wg[e >> 1] = pack_bf16x2(xv[e] * bgm[col + e], xv[e + 1] * bgm[col + e + 1]);
                }
                const uint32_t off = sw128(row, col >> 3);
                *reinterpret_cast<uint4 *>(sm + PO_TB + off) = make_uint4(wb[0], wb[1], wb[2], wb[3]);
                *reinterpret_cast<uint4 *>(sm + PO_TBG + off) = make_uint4(wg[0], wg[1], wg[2], wg[3]);
                if (tout)
                    *reinterpret_cast<uint4 *>(tout + row * 64 + col) =
                        make_uint4(pack_bf16x2(xv[0], xv[1]), pack_bf16x2(xv[2], xv[3]), pack_bf16x2(xv[4], xv[5]),
                                   pack_bf16x2(xv[6], xv[7]));
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
                // both warps of a block have read A_10 before either overwrites it with T_10
                named_bar(kBarMerge, 128);
                float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    uint32_t a[4], bb[2];
                    load_a(a, Tm, LDM, q0 + 16, q0 + 16 + 8 * kk, g8, t4);
                    load_b(bb, xs, 8, 8 * kk, 0, g8, t4);
                    mma_tf32(e, a, bb);
                }
                store_neg_d(Tm, LDM, q0 + 16, q0 + n0, e, g8, t4);
                store_tb_tbg(sm + PO_TB, sm + PO_TBG, q0 + 16 + g8, q0 + n0 + 2 * t4, -e[0], -e[1], bet, bgm, tout);
                store_tb_tbg(sm + PO_TB, sm + PO_TBG, q0 + 24 + g8, q0 + n0 + 2 * t4, -e[2], -e[3], bet, bgm, tout);
            }
            named_bar(kBarP, kNumPrep);
            SDBG(1, 4)
            // (3) 32 -> 64: X = A[32:64, 0:32] T[0:32, 0:32], then T[32:64, 0:32] = -T[32:64, 32:64] X;
            //     one warp per (16-row, 8-column) tile; T is lower triangular, so zero k-steps are skipped
            {
                const int mi = pw >> 2, ni = pw & 3;
                // [32][LDX2], reuses the 16->32 scratch (a barrier separates the two); the result goes to
                // the bf16 tiles only, so A[32:64, 0:32] is read in the first half alone
                float *x2 = Xs;
                float dacc[4] = {0.f, 0.f, 0.f, 0.f};
                for (int kk = ni; kk < 4; ++kk) {
                    uint32_t a[4], bb[2];
                    load_a(a, Am, LDM, 32 + 16 * mi, 8 * kk, g8, t4);
                    load_b(bb, Tm, LDM, 8 * kk, 8 * ni, g8, t4);
                    mma_tf32(dacc, a, bb);
                }
                store_d(x2, LDX2, 16 * mi, 8 * ni, dacc, g8, t4);
                named_bar(kBarP, kNumPrep);
                float e[4] = {0.f, 0.f, 0.f, 0.f};
                for (int kk = 0; kk <= 2 * mi + 1; ++kk) {
                    uint32_t a[4], bb[2];
                    load_a(a, Tm, LDM, 32 + 16 * mi, 32 + 8 * kk, g8, t4);
                    load_b(bb, x2, LDX2, 8 * kk, 8 * ni, g8, t4);
                    mma_tf32(e, a, bb);
                }
                store_tb_tbg(sm + PO_TB, sm + PO_TBG, 32 + 16 * mi + g8, 8 * ni + 2 * t4, -e[0], -e[1], bet, bgm, tout);
                store_tb_tbg(sm + PO_TB, sm + PO_TBG, 40 + 16 * mi + g8, 8 * ni + 2 * t4, -e[2], -e[3], bet, bgm, tout);
            }
            fence_proxy_async_smem();
            named_bar(kBarP, kNumPrep);
            if (pt == 0) {
                arrive(&bars[PB_TBREADY]);
                bulk_wait_read0();  // the P store has read its staging in the Q block
                arrive(&bars[PB_QFREE]);
                SDBG(1, 12)
                tma_store_2d(&tm_tb, sm + PO_TB, 0, (int)(gi * 64));
                bulk_commit();
                SDBG(1, 13)
            }
            SDBG(1, 5)
            // gates of the next item, while the W^T MMA runs
            if (it + 1 < nit) prep_gates(it + 1);
            SDBG(1, 6)
            // ---- W^T (bf16, rows = key dim i, 64 tokens per row) from TMEM into the staging tile ----
            if (!(ok = role_wait(&bars[PB_WDONE], kLead ? (nw & 1) : par, abort_flag, kBarP, kNumPrep))) break;
            if (kLead) ++nw;
            tc_fence_after();
            {
                const int i = (warp & 3) * 32 + lane;
                uint32_t r[32];
                tmem_ld32(tm + lb + TP_W + ch * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(r[cc * 8 + 0]), __uint_as_float(r[cc * 8 + 1]));
                    v.y = pack_bf16x2(__uint_as_float(r[cc * 8 + 2]), __uint_as_float(r[cc * 8 + 3]));
                    v.z = pack_bf16x2(__uint_as_float(r[cc * 8 + 4]), __uint_as_float(r[cc * 8 + 5]));
                    v.w = pack_bf16x2(__uint_as_float(r[cc * 8 + 6]), __uint_as_float(r[cc * 8 + 7]));
                    *reinterpret_cast<uint4 *>(sm + PO_AM + sw128(i, ch * 4 + cc)) = v;
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            named_bar(kBarP, kNumPrep);
            if (pt == 0) {
                tma_store_2d(&tm_w, sm + PO_AM, 0, (int)(gi * 128));
                bulk_commit();
            }
            SDBG(1, 7)
        }
        if (pt == 0) bulk_wait0();  // every workspace store has completed
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) atomicExch(&g_split_timeout, 1);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, 128);
    }
}

// ============================================================================
// chain kernel
// ============================================================================
constexpr int kChainThreads = 640;
// warp 0: TMA producer; warp 1: Ut^T MMA issuer; warp 2: output MMA issuer; warp 3: idle;
// warps 4-11: output role; warps 12-19: chain role, whose threads 0 and 32 issue the U^T and
// state-update MMAs themselves (the chain is latency-bound: a hand-off to another warp costs
// more than the issue)
constexpr int kOutWarp0 = 4, kNumOut = 256;
constexpr int kChnWarp0 = 12, kNumChn = 256;
constexpr int kBarOut = 1, kBarChn = 2;

// one pipeline stage (per chunk parity)
constexpr uint32_t ST_Q = 0;        // 16 KB: two [64 t][64 d] boxes
constexpr uint32_t ST_K = 16384;    // 16 KB
constexpr uint32_t ST_V = 32768;    // 16 KB
constexpr uint32_t ST_W = 49152;    // 16 KB: W^T [128 i][64 t]
constexpr uint32_t ST_P = 65536;    // 8 KB:  P [64 t][64 s]
constexpr uint32_t ST_TB = 73728;   // 8 KB:  TB [64 t][64 s]
constexpr uint32_t ST_GATE = 81920; // 528 B: the chunk's gate record
constexpr uint32_t ST_BYTES = 82944;
constexpr uint32_t CO_OST = 2 * ST_BYTES;     // 16 KB output staging: two [64 t][64 d] boxes
constexpr uint32_t CO_BARS = CO_OST + 16384;
constexpr uint32_t CO_MISC = CO_BARS + 256;
constexpr uint32_t SMEM_CHAIN = CO_MISC + 64 + 1024;

constexpr uint32_t TC_S = 0;      // 128  S float32 (row j in lane j)
constexpr uint32_t TC_SB = 128;   // 2 x 64  bf16 S (A operand), per chunk parity
constexpr uint32_t TC_DU = 256;   // 64   Ut^T, accumulated into U^T
constexpr uint32_t TC_UB = 320;   // 2 x 32  bf16 U^T (A operand), per chunk parity
constexpr uint32_t TC_O = 384;    // 64   O^T
constexpr uint32_t TC_DU2 = 448;  // 64   -S W^T over key dims 64..127

constexpr uint32_t IDESC_C64 = instr_desc_bf16(128, 64, 0, 0);               // S . Q^T, U^T . P^T
constexpr uint32_t IDESC_CMN = instr_desc_bf16(128, 64, 1, 0);               // V^T (MN-major A) . TB^T
constexpr uint32_t IDESC_CWNEG = instr_desc_bf16(128, 64, 0, 1) | (1u << 14); // S . (-W)^T, W^T MN-major
constexpr uint32_t IDESC_CS = instr_desc_bf16(128, 128, 0, 1);               // U^T . (dl K), MN-major B

enum CBar {
    CB_FULL0 = 0, CB_FULL1,        // stage tiles landed
    CB_EMPTY0, CB_EMPTY1,          // stage consumed by the three issuers (count 3)
    CB_QK0, CB_QK1,                // stage's Q and K scaled by the output role
    CB_UDONE0, CB_UDONE1,          // first half of the U^T MMA done (so the bf16 S copy is written)
    CB_SDONE0, CB_SDONE1,          // state update done (so the bf16 U^T is written)
    CB_O1DONE0, CB_O1DONE1,        // S Q^T MMA done (SB buffer free)
    CB_ODONE0, CB_ODONE1,          // U^T P^T MMA done (O complete, UB buffer free)
    CB_UTDONE,                     // Ut^T MMA done
    CB_UDONE2,                     // second half of the U^T MMA done
    CB_OFREE,                      // O read out
    CB_COUNT
};

// One CTA per (b, h, segment) computes the outputs of its chunk range from that
// segment's entry state (S0 for the first segment, else S_entry) and writes
// S_final from the last segment.  The segment transfers are the paired
// transfer kernel's.
static_assert(CB_COUNT * 8 <= CO_MISC - CO_BARS, "chain-kernel mbarriers overflow their shared-memory slot");

// Packed variable-length sequences: CTA i runs sequence ptab[i].x, head
// ptab[i].y, packed chunks ptab[i].z .. ptab[i].z + ptab[i].w - 1 of the chunk
// table ctab.  Sequences longer than the segment length run as segments:
// pseg[i] = {slot of S_entry holding the state entering the CTA's chunks, or -1
// for S0 [seq * H + head]; 1 if the chunks end the sequence (S_final [seq * H +
// head])}.  Transfer CTA i runs the full segment of seg_len chunks from packed
// chunk trtab[i].z of sequence trtab[i].x, head trtab[i].y, into slot
// trtab[i].w of Bw / Mw / Mflag.
struct ChainArgs {
    const float *gate_rec;  // [items][kRecFloats] from the prep kernel
    const float *S0;
    float *S_final;
    int64_t T, H;
    int chunks;  // chunks per (b, h) (fixed-length problems)
    int nseg, seg_len;
    const float *S_entry;  // [B*H][nseg-1][dv][dk]
    float *Bw, *Mw;        // [B*H][nseg-1][dv][dk] / [dk][dk]
    int *Mflag;            // [B*H][nseg-1]: 1 where the segment's transfer matrix is negligible (not written)
    const int4 *ptab;      // per-CTA work of packed sequences, or nullptr
    const int2 *pseg;      // packed: per-CTA entry slot and last flag, or nullptr (one CTA per sequence)
    const int4 *trtab;     // packed: per-CTA work of the segment transfers
    const int2 *ctab;      // packed chunk table, or nullptr
    __nv_bfloat16 *out;    // for the plain stores of partial packed chunks
    float *ckpt;           // fixed-length only, or nullptr: the state entering every chunk,
                           // [B*H][chunks][dv][dk] float32 (the backward's checkpoints)
    int ckpt_bf16;         // the checkpoints in bf16 instead (same layout)
    // one memory per key-value head (fixed-length problems): lead = group runs the transfers and the
    // chain for query heads hk * group only (the CTA's state index bh then counts (b, hk); S0,
    // S_final, the segment slots, the checkpoints and u_out follow it), 1 runs every head
    int lead;
    __nv_bfloat16 *u_out;  // or nullptr: U^T of every chunk, bf16 [bh][chunks][128][64]
    int group;             // grouped heads: k and v have H / group heads (head h / group)
};

__global__ void __launch_bounds__(kChainThreads, 1)
fwd_chain_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                 const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_tb,
                 const __grid_constant__ CUtensorMap tm_w, ChainArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + CO_BARS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + CO_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + CO_MISC + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t H = p.H;
    SDBG_INIT
    // work of this CTA: state index bh (S0 / S_final row block), segment, head and chunks; chunk c
    // starts at token tok0(c) of batch row b and is workspace item witem(c)
    int64_t bh;
    int b, h, c0, N;
    int64_t entry_slot;  // slot of S_entry holding the state entering the chunks, or -1 for S0
    bool last;           // the chunks end the sequence: S_final is written
    const bool packed = p.ptab != nullptr;
    if (packed) {
        const int4 w = p.ptab[blockIdx.x];
        bh = (int64_t)w.x * H + w.y;
        b = 0;
        h = w.y;
        c0 = w.z;
        N = w.w;
        const int2 sg = p.pseg ? p.pseg[blockIdx.x] : make_int2(-1, 1);
        entry_slot = sg.x;
        last = sg.y != 0;
    } else {
        bh = blockIdx.x / p.nseg;
        const int seg = (int)(blockIdx.x % p.nseg);
        const int64_t Hc = H / p.lead;  // memories per batch row
        b = (int)(bh / Hc);
        h = (int)(bh % Hc) * p.lead;
        c0 = seg * p.seg_len;
        N = (p.chunks - c0 < p.seg_len) ? (p.chunks - c0) : p.seg_len;
        entry_slot = seg == 0 ? -1 : bh * (p.nseg - 1) + seg - 1;
        last = seg == p.nseg - 1;
    }
    auto tok0 = [&](int c) -> int { return packed ? p.ctab[c0 + c].x : (c0 + c) * kC; };
    auto ntok = [&](int c) -> int { return packed ? p.ctab[c0 + c].y : kC; };  // TMA clips at T otherwise
    auto witem = [&](int c) -> int64_t {
        return packed ? (int64_t)(c0 + c) * H + h : ((int64_t)b * H + h) * p.chunks + c0 + c;
    };
    auto citem = [&](int c) -> int64_t { return bh * p.chunks + c0 + c; };  // checkpoints and u_out
    const uint32_t sbase = smem_u32(sm);

    if (tid == 0) {
        for (int i = 0; i < CB_COUNT; ++i) mbar_init(&bars[i], (i == CB_EMPTY0 || i == CB_EMPTY1) ? 3 : 1);
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
    const uint32_t lb = (uint32_t)((warp & 3) * 32) << 16;

    if (warp == 0) {
        // ============================ producer ============================
        if (lane == 0) {
            bool ok = true;
            const uint32_t bytes =
                16384 + 8192 + 16384 + 16384 + 16384 + 8192 + (uint32_t)kGateRec;
            for (int c = 0; c < N && ok; ++c) {
                const int s = c & 1;
                if (c >= 2 && !(ok = wait_bar(&bars[CB_EMPTY0 + s], ((c - 2) >> 1) & 1, abort_flag))) break;
                uint8_t *st = sm + s * ST_BYTES;
                uint64_t *full = &bars[CB_FULL0 + s];
                const int t0 = tok0(c);
                const int row = (int)witem(c);
                mbar_arrive_expect_tx(full, bytes);
                for (int blk = 0; blk < 2; ++blk) {
                    tma_load_4d(st + ST_Q + blk * 8192, &tm_q, full, blk * 64, h, t0, b);
                    tma_load_4d(st + ST_K + blk * 8192, &tm_k, full, blk * 64, h / p.group, t0, b);
                    tma_load_4d(st + ST_V + blk * 8192, &tm_v, full, blk * 64, h / p.group, t0, b);
                }
                tma_load_2d(st + ST_W, &tm_w, full, 0, row * 128);
                tma_load_2d(st + ST_P, &tm_p, full, 0, row * 64);
                tma_load_2d(st + ST_TB, &tm_tb, full, 0, row * 64);
                bulk_load(st + ST_GATE, p.gate_rec + (int64_t)row * kRecFloats, (uint32_t)kGateRec, full);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // =========================== Ut^T issuer ===========================
        if (lane == 0) {
            bool ok = true;
            for (int c = 0; c < N && ok; ++c) {
                const int s = c & 1;
                const uint32_t sp = (c >> 1) & 1;
                const uint32_t st = sbase + s * ST_BYTES;
                const int it = c;
                (void)it;
                SDBG(2, 0)
                if (!(ok = wait_bar(&bars[CB_FULL0 + s], sp, abort_flag))) break;
                // the previous chunk's state update is done, so its U^T has been read out of this
                // accumulator (and the tensor pipe is free while the chain converts the state)
                if (c > 0 && !(ok = wait_bar(&bars[CB_SDONE0 + ((c - 1) & 1)], ((c - 1) >> 1) & 1, abort_flag)))
                    break;
                SDBG(2, 1)
                tc_fence_after();
                // Ut^T = V^T TB^T
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss(tm + TC_DU, smem_desc_sw128(st + ST_V + kk * 2048, 8192, 1024),
                           smem_desc_sw128(st + ST_TB + kk * 32, 16, 1024), IDESC_CMN, kk > 0);
                mma_commit(&bars[CB_UTDONE]);
                SDBG(2, 2)
            }
        }
        __syncwarp();
    } else if (warp == 2) {
        // ========================= output issuer =========================
        if (lane == 0) {
            bool ok = true;
            for (int c = 0; c < N && ok; ++c) {
                const int s = c & 1;
                const uint32_t sp = (c >> 1) & 1;
                const uint32_t st = sbase + s * ST_BYTES;
                const uint32_t sb = TC_SB + (c & 1) * 64, ub = TC_UB + (c & 1) * 32;
                const int it = c;
                (void)it;
                SDBG(3, 0)
                // O^T is issued once the U^T MMA is done (the bf16 S copy exists, and the tensor pipe
                // is free while the chain role converts U^T), O2 once the state update is done
                if (!(ok = wait_bar(&bars[CB_QK0 + s], sp, abort_flag))) break;
                if (!(ok = wait_bar(&bars[CB_UDONE0 + (c & 1)], sp, abort_flag))) break;
                if (c > 0 && !(ok = wait_bar(&bars[CB_OFREE], (c - 1) & 1, abort_flag))) break;
                SDBG(3, 1)
                tc_fence_after();
                // O^T = S (diag(gamma) Q)^T
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tm + TC_O, tm + sb + kk * 8,
                           smem_desc_sw128(st + ST_Q + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), IDESC_C64,
                           kk > 0);
                mma_commit(&bars[CB_O1DONE0 + (c & 1)]);
                if (!(ok = wait_bar(&bars[CB_SDONE0 + (c & 1)], sp, abort_flag))) break;
                SDBG(3, 2)
                tc_fence_after();
                // O^T += U^T P^T
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(tm + TC_O, tm + ub + kk * 8, smem_desc_sw128(st + ST_P + kk * 32, 16, 1024), IDESC_C64,
                           1);
                mma_commit(&bars[CB_ODONE0 + (c & 1)]);
                mma_commit(&bars[CB_EMPTY0 + s]);
                SDBG(3, 3)
            }
        }
        __syncwarp();
    } else if (warp >= kOutWarp0 && warp < kChnWarp0) {
        // ============================ output role ============================
        // gates, diag(gamma) Q and diag(dl) K in place, then the outputs of the previous chunk
        const int ot = tid - kOutWarp0 * 32;         // 0..255
        const int j = (warp & 3) * 32 + lane;        // TMEM lane = value dim
        const int ch = (warp - kOutWarp0) >> 2;      // token half of the output tile
        bool ok = true;
        auto write_out = [&](int cprev) {
            if (ot == 0) bulk_wait_read0();  // the previous chunk's stores have read the staging buffer
            named_bar(kBarOut, kNumOut);
            const int par = j & 1, colw = j - par;  // this lane writes column pair (colw, colw + 1)
            uint8_t *stage = sm + CO_OST + (colw >> 6) * 8192;
            const uint32_t cbyte = (colw & 7) * 2, cchunk = (colw & 63) >> 3;
#pragma unroll 1
            for (int piece = 0; piece < 2; ++piece) {
                uint32_t r[16];
                tmem_ld16(tm + lb + TC_O + ch * 32 + piece * 16, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; i += 2) {
                    const float o0 = __uint_as_float(r[i]), o1 = __uint_as_float(r[i + 1]);
                    // even lanes keep row t and take the neighbour's column; odd lanes keep row t+1
                    const float send = par ? o0 : o1;
                    const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
                    const uint32_t word = par ? pack_bf16x2(recv, o1) : pack_bf16x2(o0, recv);
                    const int row = ch * 32 + piece * 16 + i + par;
                    *reinterpret_cast<uint32_t *>(stage + sw128(row, cchunk) + cbyte) = word;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(kBarOut, kNumOut);
            const int t0 = tok0(cprev), nt = ntok(cprev);
            if (nt == kC) {
                if (ot == 0) {
                    tma_store_4d(&tm_o, sm + CO_OST, 0, h, t0, b);
                    tma_store_4d(&tm_o, sm + CO_OST + 8192, 64, h, t0, b);
                    bulk_commit();
                }
            } else {
                // a partial chunk of a packed sequence: a 64-row box would write the next sequence's
                // rows, so its nt rows leave by plain 16-byte stores (unit u: box u >> 9, row
                // (u >> 3) & 63, 16-byte column chunk u & 7)
                __nv_bfloat16 *o = p.out;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int u = ot + 256 * i, box = u >> 9, row = (u >> 3) & 63, cc = u & 7;
                    if (row < nt) {
                        const uint4 v = *reinterpret_cast<const uint4 *>(sm + CO_OST + box * 8192 + sw128(row, cc));
                        *reinterpret_cast<uint4 *>(o + ((int64_t)(t0 + row) * H + h) * kD + box * 64 + cc * 8) = v;
                    }
                }
                named_bar(kBarOut, kNumOut);  // the staging buffer is read before the next chunk writes it
            }
        };
        for (int c = 0; c < N && ok; ++c) {
            const int s = c & 1;
            const uint32_t sp = (c >> 1) & 1;
            uint8_t *st = sm + s * ST_BYTES;
            const float *gam = reinterpret_cast<const float *>(st + ST_GATE), *dl = gam + 64;
            const int it = c;
            (void)it;
            SDBG(4, 0)
            if (!(ok = role_wait(&bars[CB_FULL0 + s], sp, abort_flag, kBarOut, kNumOut))) break;
            SDBG(4, 1)
            SDBG(4, 2)
            // ---- scale rows in place: Q row t by gamma_t, K row s by dl_s (16-byte units; a row
            //      of a 64-column box is one 128-byte line whatever the swizzle) ----
            {
                auto scale_tile = [&](uint8_t *tile, const float *f) {
                    uint4 v[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) v[i] = reinterpret_cast<const uint4 *>(tile)[ot + 256 * i];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float fr = f[((ot + 256 * i) >> 3) & 63];  // unit u covers bytes 16u.. of row (u/8) % 64
                        uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[e]));
                            w[e] = pack_bf16x2(x.x * fr, x.y * fr);
                        }
                        reinterpret_cast<uint4 *>(tile)[ot + 256 * i] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                };
                scale_tile(st + ST_K, dl);
                scale_tile(st + ST_Q, gam);
            }
            fence_proxy_async_smem();
            named_bar(kBarOut, kNumOut);
            if (ot == 0) arrive(&bars[CB_QK0 + s]);
            SDBG(4, 3)
            // ---- outputs of the previous chunk ----
            if (c > 0) {
                if (!(ok = role_wait(&bars[CB_ODONE0 + ((c - 1) & 1)], ((c - 1) >> 1) & 1, abort_flag, kBarOut,
                                     kNumOut)))
                    break;
                tc_fence_after();
                write_out(c - 1);  // ends with a role barrier after the O reads
                if (ot == 0) arrive(&bars[CB_OFREE]);
            }
            SDBG(4, 4)
        }
        if (ok && N > 0) {
            ok = role_wait(&bars[CB_ODONE0 + ((N - 1) & 1)], ((N - 1) >> 1) & 1, abort_flag, kBarOut, kNumOut);
            tc_fence_after();
            if (ok) write_out(N - 1);
        }
        if (ot == 0) bulk_wait0();  // every output store has completed
    } else if (warp >= kChnWarp0) {
        // ============================ chain role ============================
        // thread (j, ch) owns state row j and column half ch
        const int ct = tid - kChnWarp0 * 32;       // 0..255
        const int j = (warp & 3) * 32 + lane;      // TMEM lane / state row
        const int ch = (warp - kChnWarp0) >> 2;    // column half
        bool ok = true;
        // entry state -> TMEM: S0 (or zero) for the first segment, the prefix-scanned entry state for
        // later segments
        {
            const float *src = (entry_slot < 0) ? (p.S0 ? p.S0 + (bh * kD + j) * (int64_t)kD : nullptr)
                                                : p.S_entry + (entry_slot * kD + j) * (int64_t)kD;
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
                tmem_st32(tm + lb + TC_S + col0, r);
            }
            tmem_wait_st();
        }
        for (int c = 0; c < N && ok; ++c) {
            const int s = c & 1;
            const uint32_t sp = (c >> 1) & 1;
            const uint32_t st = sbase + s * ST_BYTES;
            const uint32_t sb = TC_SB + (c & 1) * 64, ub = TC_UB + (c & 1) * 32;
            const int it = c;
            (void)it;
            SDBG(5, 0)
            // the previous state update is done; the bf16 copy buffer of this parity was last read by
            // the output MMA of chunk c - 2; this chunk's stage (with its gates) has landed
            {
                bool w = c == 0 || wait_bar(&bars[CB_SDONE0 + ((c - 1) & 1)], ((c - 1) >> 1) & 1, abort_flag);
                w = w && (c < 2 || wait_bar(&bars[CB_O1DONE0 + (c & 1)], ((c - 2) >> 1) & 1, abort_flag));
                w = w && wait_bar(&bars[CB_FULL0 + (c & 1)], sp, abort_flag);
                if (!(ok = bar_and(kBarChn, kNumChn, w))) break;
            }
            const float gC = reinterpret_cast<const float *>(sm + (c & 1) * ST_BYTES + ST_GATE)[128];
            tc_fence_after();
            SDBG(5, 1)
            // ---- bf16 operand copy of S (row j, 64 columns) ----
#pragma unroll 1
            for (int piece = 0; piece < 2; ++piece) {
                const int col0 = ch * 64 + piece * 32;
                uint32_t r[32];
                tmem_ld32(tm + lb + TC_S + col0, r);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2)
                    pk[i >> 1] = pack_bf16x2(__uint_as_float(r[i]), __uint_as_float(r[i + 1]));
                if (p.ckpt && p.ckpt_bf16) {  // the state entering chunk c, as a bf16 checkpoint
                    uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.ckpt) +
                                                           (citem(c) * kD + j) * kD + col0);
#pragma unroll
                    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                } else if (p.ckpt) {  // the state entering chunk c, as a checkpoint
                    float4 *dst = reinterpret_cast<float4 *>(p.ckpt + (citem(c) * kD + j) * kD + col0);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                             __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
                }
                tmem_st16(tm + lb + sb + col0 / 2, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            named_bar(kBarChn, kNumChn);
            SDBG(5, 2)
            // ---- U^T = Ut^T - S W^T: key dims 0..63 into DU (onto Ut^T), 64..127 into DU2 ----
            if (ct == 0) {
                if (wait_bar(&bars[CB_UTDONE], c & 1, abort_flag)) {
                    SDBG(5, 5)
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(tm + TC_DU, tm + sb + kk * 8, smem_desc_sw128(st + ST_W + kk * 2048, 8192, 1024),
                               IDESC_CWNEG, 1u);
                    mma_commit(&bars[CB_UDONE0 + (c & 1)]);
                    SDBG(5, 6)
                }
            } else if (ct == 32) {
                tc_fence_after();
#pragma unroll
                for (int kk = 4; kk < 8; ++kk)
                    mma_ts(tm + TC_DU2, tm + sb + kk * 8, smem_desc_sw128(st + ST_W + kk * 2048, 8192, 1024),
                           IDESC_CWNEG, kk > 4 ? 1u : 0u);
                mma_commit(&bars[CB_UDONE2]);
                mma_commit(&bars[CB_EMPTY0 + s]);
            }
            // ---- S <- gamma_C S while the U^T MMAs run ----
#pragma unroll 1
            for (int piece = 0; piece < 2; ++piece) {
                const int col0 = ch * 64 + piece * 32;
                uint32_t r[32];
                tmem_ld32(tm + lb + TC_S + col0, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * gC);
                tmem_st32(tm + lb + TC_S + col0, r);
            }
            tmem_wait_st();
            SDBG(5, 7)
            // both U^T halves are done; the bf16 U^T buffer of this parity was last read by the
            // output MMA of chunk c - 2
            {
                bool w = wait_bar(&bars[CB_UDONE0 + (c & 1)], sp, abort_flag);
                SDBG(5, 8)
                w = w && wait_bar(&bars[CB_UDONE2], c & 1, abort_flag);
                SDBG(5, 9)
                w = w && (c < 2 || wait_bar(&bars[CB_ODONE0 + (c & 1)], ((c - 2) >> 1) & 1, abort_flag));
                if (!(ok = bar_and(kBarChn, kNumChn, w))) break;
            }
            tc_fence_after();
            SDBG(5, 10)
            SDBG(5, 3)
            // ---- U^T = DU + DU2 -> bf16 (this thread: 32 tokens) ----
#pragma unroll 1
            for (int piece = 0; piece < 2; ++piece) {
                uint32_t u[16], u2[16], pk[8];
                tmem_ld16(tm + lb + TC_DU + ch * 32 + piece * 16, u);
                tmem_ld16(tm + lb + TC_DU2 + ch * 32 + piece * 16, u2);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; i += 2)
                    pk[i >> 1] = pack_bf16x2(__uint_as_float(u[i]) + __uint_as_float(u2[i]),
                                             __uint_as_float(u[i + 1]) + __uint_as_float(u2[i + 1]));
                tmem_st8(tm + lb + ub + ch * 16 + piece * 8, pk);
                if (p.u_out) {  // U^T row j, tokens 32 ch + 16 piece .. + 15
                    uint4 *dst = reinterpret_cast<uint4 *>(p.u_out + (citem(c) * kD + j) * kC + ch * 32 + piece * 16);
                    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            named_bar(kBarChn, kNumChn);
            // ---- S += U^T (diag(dl) K) ----
            if (ct == 0) {
                if (wait_bar(&bars[CB_QK0 + s], sp, abort_flag)) {
                    SDBG(5, 11)
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(tm + TC_S, tm + ub + kk * 8, smem_desc_sw128(st + ST_K + kk * 2048, 8192, 1024),
                               IDESC_CS, 1);
                    mma_commit(&bars[CB_SDONE0 + (c & 1)]);
                    mma_commit(&bars[CB_EMPTY0 + s]);
                    SDBG(5, 12)
                }
            }
            SDBG(5, 4)
        }
        if (ok && N > 0) {
            ok = role_wait(&bars[CB_SDONE0 + ((N - 1) & 1)], ((N - 1) >> 1) & 1, abort_flag, kBarChn, kNumChn);
            tc_fence_after();
        }
        float *dst = (last && p.S_final) ? p.S_final + (bh * kD + j) * (int64_t)kD : nullptr;
        if (ok && dst) {
#pragma unroll 1
            for (int piece = 0; piece < 2; ++piece) {
                const int col0 = ch * 64 + piece * 32;
                uint32_t r[32];
                tmem_ld32(tm + lb + TC_S + col0, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4 *>(dst + col0 + i) =
                        make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]), __uint_as_float(r[i + 2]),
                                    __uint_as_float(r[i + 3]));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) atomicExch(&g_split_timeout, 1);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, 512);
    }
}

// ============================================================================
// paired transfer kernel (long sequences with few heads)
// ============================================================================
// One CTA per (b, h, segment < nseg - 1) computes the segment's affine transfer
// S_end = S_start M + B with two chains that share every load: group 0 runs the
// recurrence from the zero state (-> Bw), group 1 from the identity with v = 0
// (-> Mw; rows of the state evolve independently, so each row of M is a state
// row with no write term).  The two chains are independent, so each hides the
// other's latency.  Each group keeps S, the U^T accumulator and a second half
// accumulator in 256 TMEM columns; its bf16 operand copies of S and U^T live in
// shared memory.
//
// A segment whose chunks' transfer bounds rho_C multiply to at most e^-40 over
// its last m chunks (kNegligibleTransfer) needs neither run in full: the
// state entering the segment, and whatever the zero-state run gathered before
// those m chunks, reach the segment's end scaled by at most e^-40.  Such a CTA
// runs the zero-state run over the last m chunks only, skips the identity run
// and flags M as negligible for the prefix.
constexpr int kTrThreads = 640;
// warp 0: TMA producer; warp 1: Ut^T issuer (group 0); warps 2-3: K rows scaled by dl;
// warps 4-11: group 0; warps 12-19: group 1 (threads 0 and 32 of a group issue its MMAs)
constexpr int kTrGrpWarp0 = 4, kTrNumGrp = 256, kTrNumScale = 64;
constexpr int kBarGrp0 = 1, kBarScale = 3;  // group g uses named barrier kBarGrp0 + g

constexpr uint32_t TS_K = 0;         // 16 KB: two [64 t][64 d] boxes
constexpr uint32_t TS_V = 16384;     // 16 KB
constexpr uint32_t TS_W = 32768;     // 16 KB: W^T [128 i][64 t]
constexpr uint32_t TS_TB = 49152;    // 8 KB:  TB [64 t][64 s]
constexpr uint32_t TS_GATE = 57344;  // 528 B: the chunk's gate record
constexpr uint32_t TS_BYTES = 58368;
constexpr uint32_t TO_SB = 2 * TS_BYTES;        // 2 groups x 32 KB: bf16 S, two [128 j][64 i] boxes
constexpr uint32_t TO_UB = TO_SB + 2 * 32768;   // 2 groups x 16 KB: bf16 U^T, [128 j][64 t]
constexpr uint32_t TO_BARS = TO_UB + 2 * 16384;
constexpr uint32_t TO_MISC = TO_BARS + 256;
constexpr uint32_t SMEM_TR = TO_MISC + 64 + 1024;

constexpr uint32_t TT_S = 0;      // per group (base 256 g): 128  S float32
constexpr uint32_t TT_DU = 128;   //                          64   Ut^T - S W^T, key dims 0..63
constexpr uint32_t TT_DU2 = 192;  //                          64   -S W^T, key dims 64..127

constexpr uint32_t IDESC_TWNEG = instr_desc_bf16(128, 64, 0, 1) | (1u << 14);  // S . (-W)^T, W^T MN-major
constexpr uint32_t IDESC_TS = instr_desc_bf16(128, 128, 0, 1);                // U^T . (dl K), MN-major B

enum TBar {
    TB_FULL0 = 0, TB_FULL1,      // stage landed
    TB_EMPTY0, TB_EMPTY1,        // stage consumed (count 4: the U^T half and state update of each group)
    TB_KREADY0, TB_KREADY1,      // K scaled by dl
    TB_UTDONE,                   // Ut^T of group 0 done
    TB_SISSUED,                  // group 0's state update issued
    TB_UDONE0, TB_UDONE1,        // per group: first U^T half done
    TB_UDONE20, TB_UDONE21,      // per group: second U^T half done
    TB_SDONE0, TB_SDONE1,        // per group: state update done
    TB_COUNT
};
static_assert(TB_COUNT * 8 <= TO_MISC - TO_BARS, "transfer-kernel mbarriers overflow their shared-memory slot");
static_assert(SMEM_TR <= 232448, "transfer kernel exceeds the shared memory of a CTA");

__global__ void __launch_bounds__(kTrThreads, 1)
fwd_transfer_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_tb, const __grid_constant__ CUtensorMap tm_w,
                    ChainArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + TO_BARS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + TO_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + TO_MISC + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t H = p.H;
    // the segment: its first chunk cseg, its slot of Bw / Mw / Mflag, and the workspace item of chunk c
    // (a (b, h)'s chunk index for fixed-length problems, a packed chunk index for packed sequences)
    int b, h, cseg;
    int64_t slot, ibase, istride;
    if (p.trtab) {
        const int4 w = p.trtab[blockIdx.x];
        b = 0;
        h = w.y;
        cseg = w.z;
        slot = w.w;
        ibase = h;
        istride = H;
    } else {
        const int64_t bh = blockIdx.x / (p.nseg - 1);
        const int seg = (int)(blockIdx.x % (p.nseg - 1));
        const int64_t Hc = H / p.lead;
        b = (int)(bh / Hc);
        h = (int)(bh % Hc) * p.lead;
        cseg = seg * p.seg_len;  // segments 0..nseg-2 are full
        slot = bh * (p.nseg - 1) + seg;
        ibase = ((int64_t)b * H + h) * p.chunks;
        istride = 1;
    }
    auto item = [&](int c) -> int64_t { return ibase + (int64_t)c * istride; };
    auto tok0 = [&](int c) -> int { return p.trtab ? p.ctab[c].x : c * kC; };  // transfer chunks are full
    const uint32_t sbase = smem_u32(sm);
    volatile int *span = reinterpret_cast<volatile int *>(sm + TO_MISC + 8);  // chunks run, M negligible

    if (warp == 0) {
        // the shortest tail of the segment whose transfer bounds multiply to at most e^-40: warp-wide
        // suffix products over blocks of 32 chunk records, from the segment's end backwards
        int m = p.seg_len, negl = 0;
        float run = 1.f;
        for (int base = 0; base < p.seg_len; base += 32) {
            const int i = base + lane;  // i-th chunk from the end
            float x = (i < p.seg_len) ? p.gate_rec[item(cseg + p.seg_len - 1 - i) * kRecFloats + 129] : 1.f;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x *= y;
            }
            x *= run;
            const uint32_t hit = __ballot_sync(0xffffffffu, i < p.seg_len && x <= kNegligibleTransfer);
            if (hit) {
                m = base + __ffs(hit);
                negl = 1;
                break;
            }
            run = __shfl_sync(0xffffffffu, x, 31);
        }
        if (lane == 0) {
            span[0] = negl ? m : p.seg_len;
            span[1] = negl;
            p.Mflag[slot] = negl;
        }
        __syncwarp();
    }
    if (tid == 0) {
        __threadfence_block();
        // each group's U^T and state-update MMAs release a stage: two commits per running group
        const int cnt = span[1] ? 2 : 4;
        for (int i = 0; i < TB_COUNT; ++i) mbar_init(&bars[i], (i == TB_EMPTY0 || i == TB_EMPTY1) ? cnt : 1);
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
    const uint32_t lb = (uint32_t)((warp & 3) * 32) << 16;
    // the chunks run: the whole segment, or its last N chunks when its transfer matrix is negligible
    const int N = span[0];
    const bool negligible = span[1] != 0;
    const int c0 = cseg + (p.seg_len - N);

    if (warp == 0) {
        // ============================ producer ============================
        if (lane == 0) {
            bool ok = true;
            const uint32_t bytes = 16384 + 16384 + 16384 + 8192 + (uint32_t)kGateRec;
            for (int c = 0; c < N && ok; ++c) {
                const int s = c & 1;
                if (c >= 2 && !(ok = wait_bar(&bars[TB_EMPTY0 + s], ((c - 2) >> 1) & 1, abort_flag))) break;
                uint8_t *st = sm + s * TS_BYTES;
                uint64_t *full = &bars[TB_FULL0 + s];
                const int t0 = tok0(c0 + c);
                const int row = (int)item(c0 + c);
                mbar_arrive_expect_tx(full, bytes);
                for (int blk = 0; blk < 2; ++blk) {
                    tma_load_4d(st + TS_K + blk * 8192, &tm_k, full, blk * 64, h / p.group, t0, b);
                    tma_load_4d(st + TS_V + blk * 8192, &tm_v, full, blk * 64, h / p.group, t0, b);
                }
                tma_load_2d(st + TS_W, &tm_w, full, 0, row * 128);
                tma_load_2d(st + TS_TB, &tm_tb, full, 0, row * 64);
                bulk_load(st + TS_GATE, p.gate_rec + (int64_t)row * kRecFloats, (uint32_t)kGateRec, full);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ===================== Ut^T issuer (group 0) ======================
        // Ut^T = V^T TB^T of chunk c into group 0's DU2, queued behind that group's state update
        // of chunk c - 1
        if (lane == 0) {
            bool ok = true;
            for (int c = 0; c < N && ok; ++c) {
                const int s = c & 1;
                const uint32_t st = sbase + s * TS_BYTES;
                if (c > 0 && !(ok = wait_bar(&bars[TB_SISSUED], (c - 1) & 1, abort_flag))) break;
                if (!(ok = wait_bar(&bars[TB_FULL0 + s], (c >> 1) & 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss(tm + TT_DU2, smem_desc_sw128(st + TS_V + kk * 2048, 8192, 1024),
                           smem_desc_sw128(st + TS_TB + kk * 32, 16, 1024), IDESC_CMN, kk > 0);
                mma_commit(&bars[TB_UTDONE]);
            }
        }
        __syncwarp();
    } else if (warp < kTrGrpWarp0) {
        // ===================== K rows scaled by dl_s ======================
        const int kt = tid - 64;  // 0..63
        bool ok = true;
        for (int c = 0; c < N && ok; ++c) {
            const int s = c & 1;
            uint8_t *st = sm + s * TS_BYTES;
            if (!(ok = role_wait(&bars[TB_FULL0 + s], (c >> 1) & 1, abort_flag, kBarScale, kTrNumScale))) break;
            const float *dl = reinterpret_cast<const float *>(st + TS_GATE) + 64;
            uint4 *ktile = reinterpret_cast<uint4 *>(st + TS_K);
#pragma unroll 4
            for (int i = 0; i < 16; ++i) {
                const int u = kt + 64 * i;  // 16-byte unit u of K covers row (u / 8) % 64
                const float fr = dl[(u >> 3) & 63];
                const uint4 v = ktile[u];
                uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w4[e]));
                    w4[e] = pack_bf16x2(x.x * fr, x.y * fr);
                }
                ktile[u] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            fence_proxy_async_smem();
            named_bar(kBarScale, kTrNumScale);
            if (kt == 0) arrive(&bars[TB_KREADY0 + s]);
        }
    } else if (!negligible || warp < kTrGrpWarp0 + 8) {
        // ============================ chain groups ============================
        const int grp = (warp - kTrGrpWarp0) >> 3;              // 0: from zero (B), 1: from identity (M)
        const int gt = tid - (kTrGrpWarp0 + 8 * grp) * 32;       // 0..255
        const int j = (warp & 3) * 32 + lane;                    // TMEM lane / state row
        const int ch = ((warp - kTrGrpWarp0) >> 2) & 1;           // column half
        const int barg = kBarGrp0 + grp;
        const uint32_t tg = tm + (uint32_t)(256 * grp);          // this group's TMEM columns
        uint8_t *sbs = sm + TO_SB + grp * 32768;                 // bf16 S, [128 j][64 i] x 2 boxes
        uint8_t *ubs = sm + TO_UB + grp * 16384;                 // bf16 U^T, [128 j][64 t]
        const uint32_t sbs_a = sbase + TO_SB + grp * 32768, ubs_a = sbase + TO_UB + grp * 16384;
        bool ok = true;
        // entry state: zero for group 0, identity for group 1
#pragma unroll 1
        for (int piece = 0; piece < 2; ++piece) {
            const int col0 = ch * 64 + piece * 32;
            uint32_t r[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint((grp == 1 && col0 + i == j) ? 1.f : 0.f);
            tmem_st32(tg + lb + TT_S + col0, r);
        }
        tmem_wait_st();
        for (int c = 0; c < N && ok; ++c) {
            const int s = c & 1;
            const uint32_t sp = (c >> 1) & 1;
            const uint32_t st = sbase + s * TS_BYTES;
            // the previous state update is done (its operands in shared memory are free); this
            // chunk's stage has landed
            {
                bool w = c == 0 || wait_bar(&bars[TB_SDONE0 + grp], (c - 1) & 1, abort_flag);
                w = w && wait_bar(&bars[TB_FULL0 + s], sp, abort_flag);
                if (!(ok = bar_and(barg, kTrNumGrp, w))) break;
            }
            const float gC = reinterpret_cast<const float *>(sm + s * TS_BYTES + TS_GATE)[128];
            tc_fence_after();
            // ---- bf16 copy of S into shared memory (row j, 64 columns = one 128-byte row of a box) ----
#pragma unroll 1
            for (int piece = 0; piece < 2; ++piece) {
                const int col0 = ch * 64 + piece * 32;
                uint32_t r[32];
                tmem_ld32(tg + lb + TT_S + col0, r);
                tmem_wait_ld();
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(r[cc * 8 + 0]), __uint_as_float(r[cc * 8 + 1]));
                    v.y = pack_bf16x2(__uint_as_float(r[cc * 8 + 2]), __uint_as_float(r[cc * 8 + 3]));
                    v.z = pack_bf16x2(__uint_as_float(r[cc * 8 + 4]), __uint_as_float(r[cc * 8 + 5]));
                    v.w = pack_bf16x2(__uint_as_float(r[cc * 8 + 6]), __uint_as_float(r[cc * 8 + 7]));
                    *reinterpret_cast<uint4 *>(sbs + ch * 16384 + sw128(j, piece * 4 + cc)) = v;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(barg, kTrNumGrp);
            // ---- U^T = Ut^T - S W^T (key dims 0..63 from thread 0, 64..127 from thread 32) ----
            if (gt == 0) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss(tg + TT_DU, smem_desc_sw128(sbs_a + kk * 32, 16, 1024),
                           smem_desc_sw128(st + TS_W + kk * 2048, 8192, 1024), IDESC_TWNEG, kk > 0);
                mma_commit(&bars[TB_UDONE0 + grp]);
            } else if (gt == 32) {
                // group 0 accumulates onto its Ut^T; group 1 has v = 0 and starts fresh
                if (grp == 1 || wait_bar(&bars[TB_UTDONE], c & 1, abort_flag)) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 4; kk < 8; ++kk)
                        mma_ss(tg + TT_DU2, smem_desc_sw128(sbs_a + 16384 + (kk - 4) * 32, 16, 1024),
                               smem_desc_sw128(st + TS_W + kk * 2048, 8192, 1024), IDESC_TWNEG,
                               (grp == 0 || kk > 4) ? 1u : 0u);
                    mma_commit(&bars[TB_UDONE20 + grp]);
                    mma_commit(&bars[TB_EMPTY0 + s]);
                }
            }
            // ---- S <- gamma_C S while the U^T MMAs run ----
#pragma unroll 1
            for (int piece = 0; piece < 2; ++piece) {
                const int col0 = ch * 64 + piece * 32;
                uint32_t r[32];
                tmem_ld32(tg + lb + TT_S + col0, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * gC);
                tmem_st32(tg + lb + TT_S + col0, r);
            }
            tmem_wait_st();
            {
                bool w = wait_bar(&bars[TB_UDONE0 + grp], c & 1, abort_flag);
                w = w && wait_bar(&bars[TB_UDONE20 + grp], c & 1, abort_flag);
                if (!(ok = bar_and(barg, kTrNumGrp, w))) break;
            }
            tc_fence_after();
            // ---- U^T -> bf16 into shared memory (row j, tokens 32 ch .. 32 ch + 31) ----
#pragma unroll 1
            for (int piece = 0; piece < 2; ++piece) {
                uint32_t u[16], u2[16];
                tmem_ld16(tg + lb + TT_DU + ch * 32 + piece * 16, u);
                tmem_ld16(tg + lb + TT_DU2 + ch * 32 + piece * 16, u2);
                tmem_wait_ld();
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    uint32_t w4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = cc * 8 + 2 * e;
                        w4[e] = pack_bf16x2(__uint_as_float(u[i]) + __uint_as_float(u2[i]),
                                            __uint_as_float(u[i + 1]) + __uint_as_float(u2[i + 1]));
                    }
                    *reinterpret_cast<uint4 *>(ubs + sw128(j, ch * 4 + piece * 2 + cc)) =
                        make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(barg, kTrNumGrp);
            // ---- S += U^T (diag(dl) K) ----
            if (gt == 0) {
                if (wait_bar(&bars[TB_KREADY0 + s], sp, abort_flag)) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss(tg + TT_S, smem_desc_sw128(ubs_a + kk * 32, 16, 1024),
                               smem_desc_sw128(st + TS_K + kk * 2048, 8192, 1024), IDESC_TS, 1);
                    mma_commit(&bars[TB_SDONE0 + grp]);
                    mma_commit(&bars[TB_EMPTY0 + s]);
                }
                if (grp == 0) arrive(&bars[TB_SISSUED]);
            }
        }
        if (ok && N > 0) {
            ok = role_wait(&bars[TB_SDONE0 + grp], (N - 1) & 1, abort_flag, barg, kTrNumGrp);
            tc_fence_after();
        }
        float *dst = (grp == 0 ? p.Bw : p.Mw) + (slot * kD + j) * (int64_t)kD;
        if (ok) {
#pragma unroll 1
            for (int piece = 0; piece < 2; ++piece) {
                const int col0 = ch * 64 + piece * 32;
                uint32_t r[32];
                tmem_ld32(tg + lb + TT_S + col0, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4 *>(dst + col0 + i) =
                        make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]), __uint_as_float(r[i + 2]),
                                    __uint_as_float(r[i + 3]));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) atomicExch(&g_split_timeout, 1);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, 512);
    }
}

bool configure_once(const void *fn, uint32_t smem, std::atomic<uint64_t> &done) {
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (done.load() & bit) return true;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) return false;
    done.fetch_or(bit);
    return true;
}

}  // namespace

// Reads and clears the word the kernels of this file set when a bounded wait gave up
// (synchronous: it follows the work already enqueued on the legacy default stream's device).
bool take_split_timeout() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_split_timeout, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (v) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_split_timeout, &zero, sizeof(int));
    }
    return v != 0;
}

#ifdef GDN_TC_DEBUG
extern "C" int gdn_debug_set_split_dump(long long *ptr) {
    return cudaMemcpyToSymbol(g_split_dbg, &ptr, sizeof(ptr)) == cudaSuccess ? 0 : 1;
}
#endif

bool fwd_split_supported(const FwdProblem &p) {
    if (!fwd_tc_supported(p)) return false;
    const int64_t items = p.B * p.H * ((p.T + kC - 1) / kC);
    return items * 128 < ((int64_t)1 << 31);  // tile-row coordinates of the workspace maps fit in int32
}

// Flags of the segment transfers (one int per head and segment boundary), after the segment scratch.
size_t seg_flag_bytes(const FwdProblem &p, int nseg) {
    return nseg > 1 ? (((size_t)(p.B * p.H / p.lead) * (size_t)(nseg - 1) * sizeof(int) + 255) & ~(size_t)255) : 0;
}

const float *fwd_split_ws_gates(const void *workspace, int64_t items) {
    return reinterpret_cast<const float *>(static_cast<const uint8_t *>(workspace) +
                                           items * (kTileP + kTileTB + kTileW));
}

void fwd_split_ws_tiles(void *workspace, int64_t items, void **p_tiles, void **tb_tiles) {
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    *p_tiles = ws;
    *tb_tiles = ws + items * kTileP;
}

size_t fwd_split_workspace_bytes(const FwdProblem &p, int nseg) {
    const size_t items = (size_t)(p.B * p.H) * (size_t)((p.T + kC - 1) / kC);
    return items * kWsPerChunk + fwd_tc_workspace_bytes(p, nseg) + seg_flag_bytes(p, nseg);
}

cudaError_t launch_fwd_split(const FwdProblem &p, int nseg, int sm_count, void *workspace, cudaStream_t stream) {
    const int64_t chunks = (p.T + kC - 1) / kC, items = p.B * p.H * chunks;
    if (p.lead < 1 || p.H % p.lead || (p.lead > 1 && p.lead != p.group)) return cudaErrorInvalidValue;
    const int64_t heads = p.B * p.H / p.lead;  // memories: the transfer, prefix and chain CTAs' (b, h)
    if (items == 0) return cudaSuccess;
    if (!workspace) return cudaErrorInvalidValue;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint8_t *ws_p = ws, *ws_tb = ws + items * kTileP, *ws_w = ws_tb + items * kTileTB;
    float *ws_gates = reinterpret_cast<float *>(ws_w + items * kTileW);
    float *seg_ws = reinterpret_cast<float *>(ws + items * kWsPerChunk);
    CUtensorMap mq, mk, mv, mo, mp, mtb, mw;
    if (p.group < 1 || p.H % p.group) return cudaErrorInvalidValue;
    if (!make_map_bthd(&mq, p.q, p.B, p.T, p.H) || !make_map_bthd(&mk, p.k, p.B, p.T, p.H / p.group) ||
        !make_map_bthd(&mv, p.v, p.B, p.T, p.H / p.group) || !make_map_bthd(&mo, p.out, p.B, p.T, p.H) ||
        !make_map_tiles(&mp, ws_p, items, 64) || !make_map_tiles(&mtb, ws_tb, items, 64) ||
        !make_map_tiles(&mw, ws_w, items, 128))
        return cudaErrorInvalidValue;
    static std::atomic<uint64_t> conf_prep{0}, conf_prep_lead{0}, conf_chain{0}, conf_tr{0};
    if (!configure_once((const void *)fwd_prep_kernel<false>, SMEM_PREP, conf_prep) ||
        !configure_once((const void *)fwd_prep_kernel<true>, SMEM_PREP, conf_prep_lead) ||
        !configure_once((const void *)fwd_chain_kernel, SMEM_CHAIN, conf_chain) ||
        !configure_once((const void *)fwd_transfer_kernel, SMEM_TR, conf_tr))
        return cudaErrorInvalidValue;

    PrepArgs pa;
    pa.log_alpha = p.log_alpha;
    pa.beta = p.beta;
    pa.gate_rec = ws_gates;
    pa.T = p.T;
    pa.H = p.H;
    pa.items = items;
    pa.chunks = (int)chunks;
    pa.ctab = nullptr;
    pa.raw_inputs = p.raw_inputs;
    pa.group = p.group;
    pa.lead = p.lead;
    pa.t_out = static_cast<__nv_bfloat16 *>(p.t_out);
    const int64_t pgrid =
        items < kPrepCtasPerSm * (int64_t)sm_count ? items : kPrepCtasPerSm * (int64_t)sm_count;
    {
        TimedLaunch tl_(GDN_KERNEL_PREP, stream);
        if (p.lead > 1)
            fwd_prep_kernel<true><<<(unsigned)pgrid, kPrepThreads, SMEM_PREP, stream>>>(mq, mk, mp, mtb, mw, pa);
        else
            fwd_prep_kernel<false><<<(unsigned)pgrid, kPrepThreads, SMEM_PREP, stream>>>(mq, mk, mp, mtb, mw, pa);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    ChainArgs a;
    a.gate_rec = ws_gates;
    a.S0 = p.S0;
    a.S_final = p.S_final;
    a.T = p.T;
    a.H = p.H;
    a.chunks = (int)chunks;
    if (nseg < 1) nseg = 1;
    a.seg_len = (int)((chunks + nseg - 1) / nseg);
    a.nseg = (int)((chunks + a.seg_len - 1) / a.seg_len);
    a.S_entry = nullptr;
    a.Bw = a.Mw = nullptr;
    a.Mflag = nullptr;
    a.ptab = nullptr;
    a.pseg = nullptr;
    a.trtab = nullptr;
    a.ctab = nullptr;
    a.out = static_cast<__nv_bfloat16 *>(p.out);
    a.ckpt = p.ckpt;
    a.ckpt_bf16 = p.ckpt_bf16;
    a.lead = p.lead;
    a.u_out = static_cast<__nv_bfloat16 *>(p.u_out);
    a.group = p.group;
    if (a.nseg > 1) {
        const size_t per = (size_t)heads * (a.nseg - 1) * kD * kD;
        a.Bw = seg_ws;
        a.Mw = a.Bw + per;
        float *entry = a.Mw + per;
        a.S_entry = entry;
        a.Mflag = reinterpret_cast<int *>(entry + per);
        // segment transfers of segments 0..nseg-2, both runs of a segment in one CTA
        {
            TimedLaunch tl_(GDN_KERNEL_TRANSFER, stream);
            fwd_transfer_kernel<<<(unsigned)(heads * (a.nseg - 1)), kTrThreads, SMEM_TR, stream>>>(mk, mv, mtb, mw,
                                                                                                  a);
        }
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        e = launch_seg_prefix(p.S0, a.Bw, a.Mw, a.Mflag, entry, heads, a.nseg, stream);
        if (e != cudaSuccess) return e;
    }
    // outputs of every segment from its entry state
    {
        TimedLaunch tl_(GDN_KERNEL_CHAIN, stream);
        fwd_chain_kernel<<<(unsigned)(heads * a.nseg), kChainThreads, SMEM_CHAIN, stream>>>(mq, mk, mv, mo, mp, mtb, mw,
                                                                                            a);
    }
    return cudaGetLastError();
}

// Tables after the per-chunk tiles: the chunk table (int2 entries), then, from the next 256-byte
// boundary, the per-CTA table (int4 entries, read with 16-byte loads).
namespace {

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

// Makespan of CTAs of the given lengths on sm_count SMs, one CTA per SM at a time, launched
// longest first onto the SM that frees first.
int64_t list_makespan(std::vector<int64_t> &len, int sm_count) {
    std::sort(len.begin(), len.end(), std::greater<int64_t>());
    std::priority_queue<int64_t, std::vector<int64_t>, std::greater<int64_t>> free_at;
    for (int i = 0; i < sm_count; ++i) free_at.push(0);
    int64_t end = 0;
    for (int64_t l : len) {
        const int64_t t = free_at.top() + l;
        free_at.pop();
        free_at.push(t);
        end = t > end ? t : end;
    }
    return end;
}

}  // namespace

// The segment length of packed sequences: the one minimising a model of the three passes, in
// units of half a chunk step of one CTA: the transfer pass (segments but the last of each cut
// sequence, L chunks each) and the output pass (every segment), each as a list schedule over the
// SMs, plus the sequential prefix (about half a chunk step per segment of the most-cut
// sequence).  Candidates cut the longest sequence into 2..64 segments of at least 4 chunks.
bool plan_packed(const int64_t *cu_seqlens, int64_t N, int64_t H, int sm_count, PackedPlan *pl) {
    pl->H = H;
    pl->sm_count = sm_count;
    std::vector<int> first((size_t)N), n((size_t)N);
    int64_t chunks = 0, nmax = 0;
    for (int64_t i = 0; i < N; ++i) {
        const int64_t len = cu_seqlens[i + 1] - cu_seqlens[i];
        if (len < 0) return false;
        const int64_t ni = (len + kC - 1) / kC;
        first[(size_t)i] = (int)chunks;
        n[(size_t)i] = (int)ni;
        chunks += ni;
        nmax = ni > nmax ? ni : nmax;
    }
    if (chunks * H * 128 >= ((int64_t)1 << 31)) return false;  // workspace tile rows stay in int32
    pl->chunks = chunks;
    // chunk lengths of the output CTAs of one head when sequences above L chunks are cut
    auto segments_of = [&](int64_t ni, int64_t L) -> int64_t { return (L > 0 && ni > L) ? (ni + L - 1) / L : 1; };
    int64_t L = 0;
    const char *env = getenv("GDN_SEGMENTS");
    if (env && atoi(env) >= 1) {
        const int64_t k = atoi(env);
        if (k > 1 && nmax > 1) L = (nmax + k - 1) / k;
    } else if (nmax * sm_count > H * chunks && N * H * 64 <= ((int64_t)1 << 20)) {
        // the longest sequence outlasts the average load of an SM: try cutting it
        auto cost = [&](int64_t Lc) {
            std::vector<int64_t> out_len;
            int64_t ntr = 0, steps = 0;
            for (int64_t i = 0; i < N; ++i) {
                const int64_t m = segments_of(n[(size_t)i], Lc);
                for (int64_t q = 0; q < m; ++q) {
                    const int64_t cl = (q + 1 < m) ? Lc : n[(size_t)i] - (m - 1) * Lc;
                    for (int64_t h = 0; h < H; ++h) out_len.push_back(cl);
                }
                ntr += m - 1;
                steps = (m - 1) > steps ? (m - 1) : steps;
            }
            const int64_t waves = (ntr * H + sm_count - 1) / sm_count;
            return 2 * (waves * Lc + list_makespan(out_len, sm_count)) + steps;
        };
        int64_t best = cost(0);
        for (int64_t m = 2; m <= 64; ++m) {
            const int64_t Lc = (nmax + m - 1) / m;
            if (Lc < 4) break;
            const int64_t c = cost(Lc);
            if (c < best) {
                best = c;
                L = Lc;
            }
        }
    }
    pl->seg_len = (int)L;
    // tables: chunk table; output CTAs (longest first) with their entry slot and last flag; transfer
    // CTAs; prefix rows.  The transfers and entry states of a (sequence, head) take consecutive slots.
    std::vector<int2> ctab;
    ctab.reserve((size_t)chunks);
    struct OutCta { int4 w; int2 sg; };
    std::vector<OutCta> outs;
    std::vector<int4> trs, pfs;
    int64_t slot0 = 0;
    for (int64_t i = 0; i < N; ++i) {
        const int64_t t0 = cu_seqlens[i], len = cu_seqlens[i + 1] - t0, ni = n[(size_t)i];
        for (int64_t c = 0; c < ni; ++c) {
            const int64_t rest = len - c * kC;
            ctab.push_back(make_int2((int)(t0 + c * kC), (int)(rest < kC ? rest : kC)));
        }
        const int64_t m = segments_of(ni, L);
        for (int64_t h = 0; h < H; ++h) {
            const int64_t base = slot0 + h * (m - 1);
            for (int64_t q = 0; q < m; ++q) {
                const int64_t c0 = first[(size_t)i] + q * L, cl = (q + 1 < m) ? L : ni - q * L;
                outs.push_back({make_int4((int)i, (int)h, (int)c0, (int)cl),
                                make_int2(q == 0 ? -1 : (int)(base + q - 1), q == m - 1 ? 1 : 0)});
                if (q + 1 < m) trs.push_back(make_int4((int)i, (int)h, (int)c0, (int)(base + q)));
            }
            if (m > 1) pfs.push_back(make_int4((int)(i * H + h), (int)base, (int)(m - 1), 0));
        }
        slot0 += H * (m - 1);
    }
    std::stable_sort(outs.begin(), outs.end(), [](const OutCta &x, const OutCta &y) { return x.w.w > y.w.w; });
    pl->slots = slot0;
    pl->n_chain = (int64_t)outs.size();
    pl->n_transfer = (int64_t)trs.size();
    pl->n_prefix = (int64_t)pfs.size();
    pl->off_chain = round256(ctab.size() * sizeof(int2));
    pl->off_seg = pl->off_chain + round256(outs.size() * sizeof(int4));
    pl->off_transfer = pl->off_seg + round256(outs.size() * sizeof(int2));
    pl->off_prefix = pl->off_transfer + round256(trs.size() * sizeof(int4));
    pl->tables.assign(pl->off_prefix + round256(pfs.size() * sizeof(int4)), 0);
    uint8_t *t = pl->tables.data();
    if (!ctab.empty()) memcpy(t, ctab.data(), ctab.size() * sizeof(int2));
    for (size_t x = 0; x < outs.size(); ++x) {
        memcpy(t + pl->off_chain + x * sizeof(int4), &outs[x].w, sizeof(int4));
        memcpy(t + pl->off_seg + x * sizeof(int2), &outs[x].sg, sizeof(int2));
    }
    if (!trs.empty()) memcpy(t + pl->off_transfer, trs.data(), trs.size() * sizeof(int4));
    if (!pfs.empty()) memcpy(t + pl->off_prefix, pfs.data(), pfs.size() * sizeof(int4));
    return true;
}

// Workspace of a packed launch: the per-chunk tiles, the segment scratch (transfers, entry states;
// 3 x 64 KiB per slot), the flags of the transfers, then the tables.
size_t packed_workspace_bytes(const PackedPlan &pl) {
    const size_t items = (size_t)pl.chunks * (size_t)pl.H;
    return items * kWsPerChunk + (size_t)3 * (size_t)pl.slots * kD * kD * sizeof(float) +
           round256((size_t)pl.slots * sizeof(int)) + pl.tables.size();
}

cudaError_t launch_fwd_split_packed(const FwdProblem &p, const PackedPlan &pl, void *workspace,
                                    cudaStream_t stream) {
    const int64_t H = p.H, chunks = pl.chunks, items = chunks * H;
    if (pl.n_chain == 0) return cudaSuccess;
    if (!workspace || pl.H != H) return cudaErrorInvalidValue;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint8_t *ws_p = ws, *ws_tb = ws + items * kTileP, *ws_w = ws_tb + items * kTileTB;
    float *ws_gates = reinterpret_cast<float *>(ws_w + items * kTileW);
    const size_t per = (size_t)pl.slots * kD * kD;
    float *Bw = reinterpret_cast<float *>(ws + items * kWsPerChunk), *Mw = Bw + per, *S_entry = Mw + per;
    int *Mflag = reinterpret_cast<int *>(S_entry + per);
    uint8_t *dtab = reinterpret_cast<uint8_t *>(Mflag) + round256((size_t)pl.slots * sizeof(int));
    const int2 *d_ctab = reinterpret_cast<const int2 *>(dtab);
    cudaError_t e = cudaMemcpyAsync(dtab, pl.tables.data(), pl.tables.size(), cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return e;
    const int64_t rows = items > 0 ? items : 1;  // tile maps need a non-empty extent
    CUtensorMap mq, mk, mv, mo, mp, mtb, mw;
    if (!make_map_bthd(&mq, p.q, 1, p.T, p.H) || !make_map_bthd(&mk, p.k, 1, p.T, p.H) ||
        !make_map_bthd(&mv, p.v, 1, p.T, p.H) || !make_map_bthd(&mo, p.out, 1, p.T, p.H) ||
        !make_map_tiles(&mp, ws_p, rows, 64) || !make_map_tiles(&mtb, ws_tb, rows, 64) ||
        !make_map_tiles(&mw, ws_w, rows, 128))
        return cudaErrorInvalidValue;
    static std::atomic<uint64_t> conf_prep{0}, conf_prep_lead{0}, conf_chain{0}, conf_tr{0};
    if (!configure_once((const void *)fwd_prep_kernel<false>, SMEM_PREP, conf_prep) ||
        !configure_once((const void *)fwd_prep_kernel<true>, SMEM_PREP, conf_prep_lead) ||
        !configure_once((const void *)fwd_chain_kernel, SMEM_CHAIN, conf_chain) ||
        !configure_once((const void *)fwd_transfer_kernel, SMEM_TR, conf_tr))
        return cudaErrorInvalidValue;
    const int64_t sm_count = pl.sm_count;
    if (items > 0) {
        PrepArgs pa;
        pa.log_alpha = p.log_alpha;
        pa.beta = p.beta;
        pa.gate_rec = ws_gates;
        pa.T = p.T;
        pa.H = p.H;
        pa.items = items;
        pa.chunks = 0;
        pa.ctab = d_ctab;
        pa.raw_inputs = p.raw_inputs;
        pa.group = 1;
        pa.lead = 1;
        pa.t_out = nullptr;
        const int64_t pgrid =
            items < kPrepCtasPerSm * (int64_t)sm_count ? items : kPrepCtasPerSm * (int64_t)sm_count;
        TimedLaunch tl_(GDN_KERNEL_PREP, stream);
        fwd_prep_kernel<false><<<(unsigned)pgrid, kPrepThreads, SMEM_PREP, stream>>>(mq, mk, mp, mtb, mw, pa);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ChainArgs a;
    a.gate_rec = ws_gates;
    a.S0 = p.S0;
    a.S_final = p.S_final;
    a.T = p.T;
    a.H = p.H;
    a.chunks = 0;
    a.nseg = 1;
    a.seg_len = pl.seg_len;
    a.S_entry = S_entry;
    a.Bw = Bw;
    a.Mw = Mw;
    a.Mflag = Mflag;
    a.ptab = reinterpret_cast<const int4 *>(dtab + pl.off_chain);
    a.pseg = reinterpret_cast<const int2 *>(dtab + pl.off_seg);
    a.trtab = reinterpret_cast<const int4 *>(dtab + pl.off_transfer);
    a.ctab = d_ctab;
    a.out = static_cast<__nv_bfloat16 *>(p.out);
    a.ckpt = nullptr;
    a.ckpt_bf16 = 0;
    a.lead = 1;
    a.u_out = nullptr;
    a.group = 1;
    if (pl.n_transfer > 0) {
        // transfers of every segment but the last of each cut sequence, then the entry states
        {
            TimedLaunch tl_(GDN_KERNEL_TRANSFER, stream);
            fwd_transfer_kernel<<<(unsigned)pl.n_transfer, kTrThreads, SMEM_TR, stream>>>(mk, mv, mtb, mw, a);
        }
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        e = launch_seg_prefix(p.S0, Bw, Mw, Mflag, S_entry, pl.n_prefix, 0, stream,
                              reinterpret_cast<const int4 *>(dtab + pl.off_prefix));
        if (e != cudaSuccess) return e;
    }
    {
        TimedLaunch tl_(GDN_KERNEL_CHAIN, stream);
        fwd_chain_kernel<<<(unsigned)pl.n_chain, kChainThreads, SMEM_CHAIN, stream>>>(mq, mk, mv, mo, mp, mtb, mw,
                                                                                     a);
    }
    return cudaGetLastError();
}

}  // namespace gdn
