// bwd_tc.cu -- reverse mode of the chunkwise gated-delta forward on the tensor
// cores: bf16 inputs, dk = dv = 128, chunk = 64, every contraction a tcgen05
// MMA (bf16 operands, float32 accumulators in tensor memory).
//
// The forward is the Sec. 3.3 recurrence of "ATMA: Long-Context Language
// Modeling via Polar Attention and Gated-Delta Compression Memory" in its
// chunkwise form (notation as in bwd_simt.cu: entry state S, chunk-local
// log-decay cumsum g_t, gamma_t = e^{g_t}, dl_s = e^{g_C - g_s}, E_ts =
// e^{g_t - g_s}, T = (I + A)^{-1}, Y = V - diag(gamma) K S^T, U = T diag(beta) Y,
// P = E o Q K^T (s <= t)).  Given dO and the adjoint dS' of the state leaving a
// chunk:
//     dU = P^T dO + diag(dl) K dS'^T,   dR = T^T dU,   dV = diag(beta) dR,
//     dS = gamma_C dS' + dO^T diag(gamma) Q - dR^T diag(beta gamma) K      (entering the chunk),
//     dP = dO U^T (s <= t),   dA = -dR U^T (s < t),   F = dA o beta_t E,
//     dQ = diag(gamma) dO S + (dP o E) K,
//     dK = (dP o E)^T Q + (F + F^T) K - diag(beta gamma) dR S + diag(dl) U dS',
// with dbeta and d log alpha gathered from the same products.
//
// After a forward recompute (the two-kernel forward, asked for bf16
// checkpoints of the state entering every chunk and for T of every chunk),
// two passes:
//   1. bwd_chain_kernel, one CTA per (b, h) and segment, walks the chunks
//      backwards with dS in tensor memory: per chunk dU^T, dR^T and the dS
//      update as three rounds of MMAs, while a tenth warp prepares the next
//      chunk's gates and gamma-scaled Q.  It writes dV, and for pass 2 dS'
//      (bf16) and dR (bf16) of every chunk, through TMA stores.  Long
//      sequences with few heads are cut into the forward's segments: a
//      transfer launch of the same kernel gives each segment's map of the
//      adjoint (dS -> dS X_p + B'_p, X_p the transpose of the segment's
//      forward transfer), the forward's prefix kernel chains them from
//      dS_final, and every segment then walks at once.
//   2. bwd_grad_kernel, chunk-parallel (persistent CTAs over the chunks of
//      every (b, h)): from S, dS', dR and the chunk's tiles it forms
//      [Q;K] K^T, [Q;K] S^T, dS' K^T, U^T, [dO; dR] U^T and finally
//      [dQ; dK] as one 128-row accumulator fed by three products, then dbeta
//      and d log alpha.
// Both kernels run their rounds in lock step (one thread issues, all wait on
// the MMA's mbarrier with a bounded wait), so each round's latency shows; the
// chunk-parallel pass hides it behind the other SMs' chunks.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

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
constexpr int kRecFloats = 132;  // the forward prep kernel's gate record per chunk; [129] is rho_C

__device__ int g_bwd_timeout;  // set when a bounded mbarrier wait gives up

#ifdef GDN_TC_DEBUG
// Debug builds only: per-phase clock stamps of the gradient pass's CTA 0 for its first 8 items, 16 int64
// per item.
__device__ long long *g_bwd_dbg;
#define BDBG(i) \
    if (dbgp != nullptr && nd < 8 && tid == 0) dbgp[nd * 16 + (i)] = clock64();
// and of the reverse chain's CTA 0 for its first 8 chunks
__device__ long long *g_bwd1_dbg;
#define B1DBG(i) \
    if (blockIdx.x == 0 && g_bwd1_dbg != nullptr && idx < 8 && tid == 0) g_bwd1_dbg[idx * 16 + (i)] = clock64();
#else
#define BDBG(i)
#define B1DBG(i)
#endif

// [rows][128] bf16 viewed as a 2-D tensor; box = 64 columns x box_rows rows, 128-byte swizzle.
inline bool make_map_rows128(CUtensorMap *m, const void *base, int64_t rows, uint32_t box_rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[2] = {128, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {128 * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

__device__ __forceinline__ void unpack8(const uint4 &w, float *f) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u[i]));
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}

__device__ __forceinline__ uint16_t bf16_bits(float x) {
    const __nv_bfloat16 b = __float2bfloat16_rn(x);
    return *reinterpret_cast<const uint16_t *>(&b);
}

// Element (r, c) of a bf16 tile stored as 64-column, 128-byte-swizzled boxes of `box_rows` rows.
__device__ __forceinline__ uint32_t tile_off(uint32_t r, uint32_t c, uint32_t box_bytes) {
    return (c >> 6) * box_bytes + sw128(r, (c & 63) >> 3) + (c & 7) * 2;
}

// The sum over the warp's 32 lanes of column `lane` of v[0..31] (v is destroyed): five exchange
// rounds, each halving the columns a lane keeps.
__device__ __forceinline__ float warp_colsum32(float (&v)[32]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        const bool up = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
            const float send = up ? v[i] : v[i + off];
            const float keep = up ? v[i + off] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    return v[0];
}

// Chunk-local inclusive cumsum g_t of the clamped log-decays (zero past the n valid tokens) and
// beta_t, by threads 0..63 of a group of `nthreads` that share named barrier `bar_id`; every thread
// of the group calls it.  g[], bet[] receive 64 entries.
// chunk_gates_from takes this thread's raw gates (log alpha unclamped, zero past the valid tokens).
__device__ __forceinline__ void chunk_gates_from(float la, float be, int n, int tid, float *g, float *bet,
                                                 float *scratch, int bar_id, int nthreads) {
    la = (tid < 64 && tid < n) ? fmaxf(la, kLogAlphaFloor) : 0.f;
    be = (tid < 64 && tid < n) ? be : 0.f;
    float s = la;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, s, off);
        if ((tid & 31) >= off) s += y;
    }
    if (tid == 31) scratch[0] = s;
    named_bar(bar_id, nthreads);
    if (tid >= 32 && tid < 64) s += scratch[0];
    if (tid < 64) {
        g[tid] = s;
        bet[tid] = be;
    }
    named_bar(bar_id, nthreads);
}
__device__ __forceinline__ void chunk_gates(const float *log_alpha, const float *beta, int64_t gbase, int64_t H,
                                            int t0, int n, int tid, float *g, float *bet, float *scratch,
                                            int bar_id, int nthreads) {
    float la = 0.f, be = 0.f;
    if (tid < 64 && tid < n) {
        la = log_alpha[gbase + (int64_t)(t0 + tid) * H];
        be = beta[gbase + (int64_t)(t0 + tid) * H];
    }
    chunk_gates_from(la, be, n, tid, g, bet, scratch, bar_id, nthreads);
}

constexpr uint32_t IDESC_64_MN_MN = instr_desc_bf16(128, 64, 1, 1);
constexpr uint32_t IDESC_64_KK = instr_desc_bf16(128, 64, 0, 0);
constexpr uint32_t IDESC_64_K_MN = instr_desc_bf16(128, 64, 0, 1);
constexpr uint32_t IDESC_64_MN_K = instr_desc_bf16(128, 64, 1, 0);
constexpr uint32_t IDESC_128_MN_MN = instr_desc_bf16(128, 128, 1, 1);
constexpr uint32_t IDESC_128_K_MN = instr_desc_bf16(128, 128, 0, 1);
constexpr uint32_t IDESC_128_KK = instr_desc_bf16(128, 128, 0, 0);

// ============================================================================
// pass 1: reverse chain
// ============================================================================
constexpr int kP1Threads = 320;  // warps 0-7: the chain, two per TMEM lane quadrant (value dim j = lane
                                 // 32 (w & 3) + lane, column half w >> 2); warp 8: TMA; warp 9: each chunk's
                                 // gates and gamma-scaled Q, one chunk ahead of the chain
constexpr int kP1Compute = 256;
constexpr int kBarP1 = 1;

constexpr uint32_t S1_DO = 0;       // 16 KB: dO, two [64 t][64 j] boxes
constexpr uint32_t S1_Q = 16384;    // 16 KB: Q, scaled by gamma in place
constexpr uint32_t S1_K = 32768;    // 16 KB: K
constexpr uint32_t S1_P = 49152;    // 8 KB:  P [t][s]
constexpr uint32_t S1_T = 57344;    // 8 KB:  T [s][t]
constexpr uint32_t S1_BYTES = 65536;
// staging of the outputs for TMA stores (128-byte swizzle): dS' [128 j][128 i] as two [128][64] boxes,
// dR and dV [64 t][128 j] as two [64][64] boxes each
constexpr uint32_t O1_DSST = 2 * S1_BYTES;    // 32 KB
constexpr uint32_t O1_DRST = O1_DSST + 32768;  // 16 KB
constexpr uint32_t O1_DVST = O1_DRST + 16384;  // 16 KB
constexpr uint32_t O1_GATE = O1_DVST + 16384;  // per chunk parity: bet[64], gam[64], dl[64], gamma_C (1 KB)
constexpr uint32_t O1_BARS = O1_GATE + 2048;
constexpr uint32_t O1_MISC = O1_BARS + 128;
constexpr uint32_t SMEM_P1 = O1_MISC + 64 + 1024;
static_assert(SMEM_P1 <= 232448, "pass-1 kernel exceeds the shared memory of a CTA");

// READY: a chunk's gates are in their buffer and its stage has landed with Q scaled; GFREE: the chain is done
// with a gate buffer (both per chunk parity)
enum P1Bar {
    B1_FULL0 = 0,
    B1_FULL1,
    B1_EMPTY0,
    B1_EMPTY1,
    B1_MMA,
    B1_READY0,
    B1_READY1,
    B1_GFREE0,
    B1_GFREE1,
    B1_COUNT
};
static_assert(B1_COUNT * 8 <= O1_MISC - O1_BARS, "pass-1 mbarriers overflow their slot");

// tensor memory of pass 1
constexpr uint32_t T1_DS = 0;     // 128 dS float32 (row j in lane j)
constexpr uint32_t T1_DSB = 128;  // 64  dS in bf16 (A operand)
constexpr uint32_t T1_DU = 192;   // 64  dO^T P
constexpr uint32_t T1_D2 = 256;   // 64  dS K^T
constexpr uint32_t T1_DUB = 320;  // 32  dU^T in bf16 (A operand)
constexpr uint32_t T1_DR = 352;   // 64  dR^T
constexpr uint32_t T1_DRB = 416;  // 32  -beta gamma dR^T in bf16 (A operand)

struct BwdArgs {
    const float *log_alpha, *beta;
    const float *dS_final;   // [B*H][128][128] or nullptr
    float *dS0;              // or nullptr
    __nv_bfloat16 *dv;       // [B, T, H, 128]
    __nv_bfloat16 *dq, *dk;  // [B, T, H, 128]
    float *dlog_alpha, *dbeta;  // [B, T, H]
    __nv_bfloat16 *ds_ws;    // [items][128][128]: dS' of every chunk (pass 1 -> pass 2)
    __nv_bfloat16 *dr_ws;    // [items][64][128]:  dR of every chunk
    int64_t T, H, items;
    int chunks;
    // Segments: chunks [p seg_len, (p + 1) seg_len) of each (b, h) form segment p (nseg = 1: one
    // segment).  The adjoint leaving a segment maps to the one entering it by dS -> dS X_p + B'_p,
    // X_p = M_p^T the transpose of the segment's forward transfer (S -> S M_p + B_p).
    int nseg, seg_len;
    // 0: one CTA per (b, h) and segment walks its chunks backwards from the adjoint leaving the segment
    //    (dS_final for the last one, else `entry`) and writes every output (dS0 for segment 0);
    // 1: transfers, a CTA pair per (b, h) and segment p >= 1 writing only the adjoint it reaches at the
    //    segment's start: run 0 from zero with dO (B'_p), run 1 from the identity without dO (X_p).
    int mode;
    const float *gate_rec;  // the forward's gate records: rho_C at [129] bounds the chunks' transfers
    const float *entry;     // [B*H][nseg - 1][128][128]: the prefix's result, slot q for segment nseg - 2 - q
    float *xb, *xm;         // [B*H][nseg - 1][128][128]: B'_p and X_p in slot q = nseg - 1 - p
    int *xflag;             // [B*H][nseg - 1]: X_p negligible (slot q)
};

__global__ void __launch_bounds__(kP1Threads, 1)
bwd_chain_kernel(const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_q,
                 const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_p,
                 const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_dsw,
                 const __grid_constant__ CUtensorMap tm_drw, const __grid_constant__ CUtensorMap tm_dv, BwdArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + O1_BARS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + O1_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + O1_MISC + 4);
    float *gbuf = reinterpret_cast<float *>(sm + O1_GATE);  // [2][256]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t H = p.H, T = p.T;
    int64_t bh;
    int seg, run = 0;
    if (p.mode == 0) {
        bh = blockIdx.x / p.nseg;
        seg = (int)(blockIdx.x % p.nseg);
    } else {
        bh = (blockIdx.x >> 1) / (p.nseg - 1);
        seg = 1 + (int)((blockIdx.x >> 1) % (p.nseg - 1));
        run = (int)(blockIdx.x & 1);
    }
    const int b = (int)(bh / H), h = (int)(bh % H);
    const int nch = p.chunks;
    const int c_lo = seg * p.seg_len, c_hi = (c_lo + p.seg_len < nch) ? c_lo + p.seg_len : nch;
    const bool idrun = p.mode == 1 && run == 1;  // the identity run: no dO
    const int64_t slot = bh * (p.nseg - 1) + (p.nseg - 1 - seg);
    volatile int *span = reinterpret_cast<volatile int *>(sm + O1_MISC + 8);  // chunks walked
    const uint32_t sbase = smem_u32(sm);

    if (warp == 0) {
        int nrun = c_hi - c_lo;
        if (p.mode == 1) {
            // the shortest head of the segment whose transfer bounds multiply to at most e^-40: the
            // chunks after it reach the segment's start scaled by at most that, so the zero run walks
            // the head alone and X_p is negligible (warp-wide prefix products over blocks of 32 records)
            const int len = c_hi - c_lo;
            int m = len, negl = 0;
            float acc = 1.f;
            for (int base = 0; base < len; base += 32) {
                const int i = base + lane;
                float x = (i < len) ? p.gate_rec[(bh * nch + c_lo + i) * kRecFloats + 129] : 1.f;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x, o);
                    if (lane >= o) x *= y;
                }
                x *= acc;
                const uint32_t hit = __ballot_sync(0xffffffffu, i < len && x <= kNegligibleTransfer);
                if (hit) {
                    m = base + __ffs(hit);
                    negl = 1;
                    break;
                }
                acc = __shfl_sync(0xffffffffu, x, 31);
            }
            nrun = idrun ? (negl ? 0 : len) : m;
            if (idrun && lane == 0) p.xflag[slot] = negl;
        }
        if (lane == 0) span[0] = nrun;
        __syncwarp();
    }
    if (tid == 0) {
        for (int i = 0; i < B1_COUNT; ++i) mbar_init(&bars[i], 1);
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
    const int nrun = span[0];
    const int c_top = c_lo + nrun - 1;  // the walk's first chunk

    if (warp == 8) {
        // ============================ producer ============================
        if (lane == 0) {
            bool ok = true;
            for (int idx = 0; idx < nrun && ok; ++idx) {
                const int c = c_top - idx, s = idx & 1;
                if (idx >= 2 && !(ok = wait_bar(&bars[B1_EMPTY0 + s], ((idx - 2) >> 1) & 1, abort_flag))) break;
                uint8_t *st = sm + s * S1_BYTES;
                uint64_t *full = &bars[B1_FULL0 + s];
                const int t0 = c * kC;
                const int row = (int)(bh * nch + c) * 64;
                // the identity run needs neither dO nor the products that carry it (Q, P)
                mbar_arrive_expect_tx(full, idrun ? 16384 + 8192 : 3 * 16384 + 2 * 8192);
                for (int blk = 0; blk < 2; ++blk) {
                    if (!idrun) {
                        tma_load_4d(st + S1_DO + blk * 8192, &tm_do, full, blk * 64, h, t0, b);
                        tma_load_4d(st + S1_Q + blk * 8192, &tm_q, full, blk * 64, h, t0, b);
                    }
                    tma_load_4d(st + S1_K + blk * 8192, &tm_k, full, blk * 64, h, t0, b);
                }
                if (!idrun) tma_load_2d(st + S1_P, &tm_p, full, 0, row);
                tma_load_2d(st + S1_T, &tm_t, full, 0, row);
            }
        }
        __syncwarp();
    } else if (warp == 9) {
        // ============================ prepare ============================
        // chunk idx's gates into buffer idx & 1 (once the chain is done with chunk idx - 2's), then its
        // stage's Q rows scaled by gamma_t in place once the stage has landed (16-byte unit u: box u >> 9,
        // row (u >> 3) & 63)
        bool ok = true;
        for (int idx = 0; idx < nrun && ok; ++idx) {
            const int c = c_top - idx, s = idx & 1;
            const int t0 = c * kC;
            const int n = (T - t0 < kC) ? (int)(T - t0) : kC;
            // the raw gates of tokens lane and lane + 32 (zero past the valid tokens)
            float la[2], be[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int t = lane + 32 * k;
                const int64_t x = ((int64_t)b * T + t0 + t) * H + h;
                la[k] = t < n ? fmaxf(p.log_alpha[x], kLogAlphaFloor) : 0.f;
                be[k] = t < n ? p.beta[x] : 0.f;
            }
            // inclusive cumsum over the 64 tokens: each half by shuffles, the first half's total then
            // added to the second
            float s0 = la[0], s1 = la[1];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y0 = __shfl_up_sync(0xffffffffu, s0, o), y1 = __shfl_up_sync(0xffffffffu, s1, o);
                if (lane >= o) {
                    s0 += y0;
                    s1 += y1;
                }
            }
            s1 += __shfl_sync(0xffffffffu, s0, 31);
            const float g63 = __shfl_sync(0xffffffffu, s1, 31);
            if (idx >= 2 && !(ok = wait_bar(&bars[B1_GFREE0 + s], ((idx - 2) >> 1) & 1, abort_flag))) break;
            float *gb = gbuf + s * 256;
            gb[lane] = be[0];
            gb[32 + lane] = be[1];
            gb[64 + lane] = expf(s0);
            gb[96 + lane] = expf(s1);
            gb[128 + lane] = expf(g63 - s0);
            gb[160 + lane] = expf(g63 - s1);
            if (lane == 0) gb[192] = expf(g63);
            if (!(ok = wait_bar(&bars[B1_FULL0 + s], (idx >> 1) & 1, abort_flag))) break;
            __syncwarp();
            if (!idrun) {
                uint4 *q = reinterpret_cast<uint4 *>(sm + s * S1_BYTES + S1_Q);
#pragma unroll 4
                for (int i = 0; i < 32; ++i) {
                    const int u = lane + 32 * i;
                    float f[8];
                    unpack8(q[u], f);
                    const float x = gb[64 + ((u >> 3) & 63)];
                    q[u] = make_uint4(pack_bf16x2(f[0] * x, f[1] * x), pack_bf16x2(f[2] * x, f[3] * x),
                                      pack_bf16x2(f[4] * x, f[5] * x), pack_bf16x2(f[6] * x, f[7] * x));
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) arrive(&bars[B1_READY0 + s]);
        }
    } else {
        // ============================ the chain ============================
        const int j = (warp & 3) * 32 + lane;  // value dim = TMEM lane
        const int ch = warp >> 2;             // column half
        const uint32_t lb = (uint32_t)((warp & 3) * 32) << 16;
        bool ok = true;
        uint32_t mph = 0;  // phase of the next wait on B1_MMA
        // dS <- the adjoint leaving the walk: dS_final (or zero) for the last segment, the prefix's
        // entry for the others; zero for the transfer's zero run, the identity for its identity run
        const float *ent = nullptr;
        if (p.mode == 0) {
            if (seg == p.nseg - 1)
                ent = p.dS_final ? p.dS_final + bh * kD * kD : nullptr;
            else
                ent = p.entry + (bh * (p.nseg - 1) + (p.nseg - 2 - seg)) * kD * kD;
        }
#pragma unroll 1
        for (int pc = 2 * ch; pc < 2 * ch + 2; ++pc) {
            uint32_t r[32];
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (ent) x = *reinterpret_cast<const float4 *>(ent + (int64_t)j * kD + 32 * pc + i);
                r[i] = __float_as_uint(x.x);
                r[i + 1] = __float_as_uint(x.y);
                r[i + 2] = __float_as_uint(x.z);
                r[i + 3] = __float_as_uint(x.w);
            }
            if (idrun) {
#pragma unroll
                for (int i = 0; i < 32; ++i) r[i] = __float_as_uint((32 * pc + i == j) ? 1.f : 0.f);
            }
            tmem_st32(tm + lb + T1_DS + 32 * pc, r);
        }
        tmem_wait_st();
        auto mma_round = [&]() {  // every compute thread: wait for the MMAs committed to B1_MMA
            const bool w = wait_bar(&bars[B1_MMA], mph, abort_flag);
            mph ^= 1u;
            const bool r = bar_and(kBarP1, kP1Compute, w);
            ok = ok && r;
            tc_fence_after();
        };
        auto sync_after_tmem_st = [&]() {
            tmem_wait_st();
            tc_fence_before();
            named_bar(kBarP1, kP1Compute);
            tc_fence_after();
        };
#pragma unroll 1
        for (int idx = 0; idx < nrun && ok; ++idx) {
            B1DBG(0)
            const int c = c_top - idx, s = idx & 1;
            const int t0 = c * kC;
            const int64_t item = bh * nch + c;
            const uint32_t sta = sbase + s * S1_BYTES;
            // this chunk's gates, and its stage (landed, Q scaled), from the prepare warp
            {
                const bool w = wait_bar(&bars[B1_READY0 + s], (idx >> 1) & 1, abort_flag);
                if (!(ok = bar_and(kBarP1, kP1Compute, w) && ok)) break;
            }
            const float *bet = gbuf + s * 256, *gam = bet + 64, *dl = bet + 128;
            const float gC = bet[192];
            // ---- dS (the adjoint of the state leaving chunk c): bf16 copy into TMEM and to the
            //      workspace, then dS <- gamma_C dS ----
            {
#pragma unroll 1
                for (int pc = 2 * ch; pc < 2 * ch + 2; ++pc) {
                    uint32_t r[32];
                    tmem_ld32(tm + lb + T1_DS + 32 * pc, r);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 2)
                        pk[i >> 1] = pack_bf16x2(__uint_as_float(r[i]), __uint_as_float(r[i + 1]));
                    tmem_st16(tm + lb + T1_DSB + 16 * pc, pk);
                    if (p.mode == 0) {
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            *reinterpret_cast<uint4 *>(sm + O1_DSST + ch * 16384 + sw128(j, (pc & 1) * 4 + i)) =
                                make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(gC * __uint_as_float(r[i]));
                    tmem_st32(tm + lb + T1_DS + 32 * pc, r);
                }
            }
            if (p.mode == 0) fence_proxy_async_smem();
            sync_after_tmem_st();
            if (p.mode == 0 && tid == 0) {
                // dS' of this chunk to the workspace (pass 2 reads it)
                for (int blk = 0; blk < 2; ++blk)
                    tma_store_2d(&tm_dsw, sm + O1_DSST + blk * 16384, blk * 64, (int)(item * 128));
                bulk_commit();
            }
            B1DBG(1)
            // ---- dO^T P and dS K^T ----
            if (tid == 0) {
                // the issuing thread observes the stage's loads itself (complete long since: the prepare
                // warp saw them before this chunk was ready)
                wait_bar(&bars[B1_FULL0 + s], (idx >> 1) & 1, abort_flag);
                if (!idrun) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss(tm + T1_DU, smem_desc_sw128(sta + S1_DO + kk * 2048, 8192, 1024),
                               smem_desc_sw128(sta + S1_P + kk * 2048, 8192, 1024), IDESC_64_MN_MN, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tm + T1_D2, tm + T1_DSB + kk * 8,
                           smem_desc_sw128(sta + S1_K + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), IDESC_64_KK,
                           kk > 0);
                mma_commit(&bars[B1_MMA]);
            }
            mma_round();
            B1DBG(2)
            if (!ok) break;
            // ---- dU^T = dO^T P + (dS K^T) diag(dl), in bf16 ----
            {
                const int pc = ch;
                uint32_t a[32], d2[32];
                tmem_ld32(tm + lb + T1_DU + 32 * pc, a);
                tmem_ld32(tm + lb + T1_D2 + 32 * pc, d2);
                tmem_wait_ld();
                if (idrun) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) a[i] = 0u;
                }
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const float u0 = fmaf(dl[32 * pc + i], __uint_as_float(d2[i]), __uint_as_float(a[i]));
                    const float u1 = fmaf(dl[32 * pc + i + 1], __uint_as_float(d2[i + 1]), __uint_as_float(a[i + 1]));
                    pk[i >> 1] = pack_bf16x2(u0, u1);
                }
                tmem_st16(tm + lb + T1_DUB + 16 * pc, pk);
            }
            sync_after_tmem_st();
            B1DBG(3)
            // ---- dR^T = dU^T T ----
            if (tid == 0) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(tm + T1_DR, tm + T1_DUB + kk * 8, smem_desc_sw128(sta + S1_T + kk * 2048, 8192, 1024),
                           IDESC_64_K_MN, kk > 0);
                mma_commit(&bars[B1_MMA]);
            }
            mma_round();
            B1DBG(4)
            if (!ok) break;
            // ---- -beta gamma dR^T in bf16 for the state update; then, while that runs, dV = diag(beta) dR
            //      (output) and dR (workspace) ----
            uint32_t r[32];
            tmem_ld32(tm + lb + T1_DR + 32 * ch, r);
            tmem_wait_ld();
            {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const int t = 32 * ch + i;
                    pk[i >> 1] = pack_bf16x2(-bet[t] * gam[t] * __uint_as_float(r[i]),
                                             -bet[t + 1] * gam[t + 1] * __uint_as_float(r[i + 1]));
                }
                tmem_st16(tm + lb + T1_DRB + 16 * ch, pk);
            }
            // the previous chunk's dR / dV stores have read their staging before it is written again below
            if (tid == 0) bulk_wait_read0();
            sync_after_tmem_st();
            B1DBG(5)
            // ---- dS += dO^T (diag(gamma) Q) - dR^T diag(beta gamma) K ----
            if (tid == 0) {
                if (!idrun) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss(tm + T1_DS, smem_desc_sw128(sta + S1_DO + kk * 2048, 8192, 1024),
                               smem_desc_sw128(sta + S1_Q + kk * 2048, 8192, 1024), IDESC_128_MN_MN, 1u);
                }
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(tm + T1_DS, tm + T1_DRB + kk * 8, smem_desc_sw128(sta + S1_K + kk * 2048, 8192, 1024),
                           IDESC_128_K_MN, 1u);
                mma_commit(&bars[B1_EMPTY0 + s]);
                mma_commit(&bars[B1_MMA]);
            }
            if (p.mode == 0) {
                // thread j holds column j of dR (tokens 32 ch ..): element (t, j) of the staged [64 t][128 j]
                // tiles sits in box j / 64, row t, 16-byte chunk (j % 64) / 8.  Lanes j, j ^ 1 trade one value
                // per token pair so that each writes two adjacent columns of one row: the even lane columns
                // j, j + 1 of row t, the odd lane columns j - 1, j of row t + 1.
                const bool odd = (lane & 1) != 0;
                const int j0 = j & ~1;
                const uint32_t col = (uint32_t)(j0 >> 6) * 8192, cj = (uint32_t)((j0 & 63) >> 3), bj = (j0 & 7) * 2;
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const int t = 32 * ch + i;
                    const float x0 = __uint_as_float(r[i]), x1 = __uint_as_float(r[i + 1]);
                    const float got = __shfl_xor_sync(0xffffffffu, odd ? x0 : x1, 1);
                    const int row = odd ? t + 1 : t;
                    const float lo = odd ? got : x0, hi = odd ? x1 : got, bt = bet[row];
                    const uint32_t o = col + sw128(row, cj) + bj;
                    *reinterpret_cast<uint32_t *>(sm + O1_DRST + o) = pack_bf16x2(lo, hi);
                    *reinterpret_cast<uint32_t *>(sm + O1_DVST + o) = pack_bf16x2(bt * lo, bt * hi);
                }
                fence_proxy_async_smem();
            }
            named_bar(kBarP1, kP1Compute);
            if (tid == 0) {
                arrive(&bars[B1_GFREE0 + s]);  // this chunk's gates are no longer read
                if (p.mode == 0) {
                    // dR to the workspace, dV to the output (its rows past the sequence's end are outside
                    // the tensor and not written)
                    for (int blk = 0; blk < 2; ++blk) {
                        tma_store_2d(&tm_drw, sm + O1_DRST + blk * 8192, blk * 64, (int)(item * 64));
                        tma_store_4d(&tm_dv, sm + O1_DVST + blk * 8192, blk * 64, h, t0, b);
                    }
                    bulk_commit();
                }
            }
            B1DBG(6)
            mma_round();
            B1DBG(7)
        }
        // the adjoint reached at the walk's start: dS0 (the state entering chunk 0) for segment 0, B'_p or
        // X_p for a transfer run
        float *exitp = nullptr;
        if (p.mode == 0)
            exitp = (seg == 0 && p.dS0) ? p.dS0 + bh * kD * kD : nullptr;
        else if (nrun > 0)
            exitp = (idrun ? p.xm : p.xb) + slot * kD * kD;
        if (ok && exitp) {
#pragma unroll 1
            for (int pc = 2 * ch; pc < 2 * ch + 2; ++pc) {
                uint32_t r[32];
                tmem_ld32(tm + lb + T1_DS + 32 * pc, r);
                tmem_wait_ld();
                float4 *dst = reinterpret_cast<float4 *>(exitp + (int64_t)j * kD + 32 * pc);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                         __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
            }
        }
        if (!ok) *abort_flag = 1;
        if (tid == 0) bulk_wait0();  // every dS', dR and dV store has completed
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) atomicExch(&g_bwd_timeout, 1);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, 512);
    }
}

// ============================================================================
// pass 2: chunk-parallel gradients
// ============================================================================
constexpr int kP2Threads = 256;  // two threads per TMEM lane: row m = 32 (w & 3) + lane, column half w >> 2

constexpr uint32_t R_QK = 0;        // 32 KB: box b = [Q rows 0-63 | K rows 64-127] x columns 64b..64b+63
constexpr uint32_t R_DOR = 32768;   // 32 KB: box b = [dO rows 0-63 | dR rows 64-127]
constexpr uint32_t R_V = 65536;     // 16 KB: V [64 t][64 j] x 2 boxes, overwritten by Y = V - diag(gamma) K S^T
constexpr uint32_t R_S = 81920;     // 32 KB: S (bf16) [128 j][64 i] x 2 boxes
constexpr uint32_t R_DS = 114688;   // 32 KB: dS' (bf16), same layout
constexpr uint32_t R_UT = 147456;   // 16 KB: U^T [128 j][64 s]
constexpr uint32_t R_TB = 163840;   // 8 KB:  T diag(beta) [t][s]
constexpr uint32_t R_A1 = 172032;   // 32 KB: [[0, dP o E], [(dP o E)^T, F + F^T]], [128 m][64 k] x 2 boxes
constexpr uint32_t R_F = 204800;    // floats: g, bet, gam, dl, dg, db, colsum [64 each], misc [16], keep [64]
constexpr uint32_t R_BARS = R_F + 8 * 256 + 64;
constexpr uint32_t R_MISC = R_BARS + 64;
constexpr uint32_t SMEM_P2 = R_MISC + 64 + 1024;
static_assert(SMEM_P2 <= 232448, "pass-2 kernel exceeds the shared memory of a CTA");

// B2_LOAD: Q, K, dO, dR, S, dS' of an item; B2_LOADE: its V and T diag(beta), which load as soon as the
// previous item's round 2 has read its own
enum P2Bar { B2_LOAD = 0, B2_LOADE, B2_MMA, B2_COUNT };

// tensor memory of pass 2 (the last round reuses columns 0..383)
constexpr uint32_t T2_G = 0;     // 64:  [Q; K] K^T
constexpr uint32_t T2_Z = 64;    // 128: [Q; K] S^T
constexpr uint32_t T2_D2 = 192;  // 64:  dS' K^T (rows j)
constexpr uint32_t T2_U = 256;   // 64:  U^T (rows j)
constexpr uint32_t T2_DG = 320;  // 64:  [dO; dR] U^T
constexpr uint32_t T2_H1 = 0;    // 128: A1 [Q; K]
constexpr uint32_t T2_H2 = 128;  // 128: [dO; dR] S
constexpr uint32_t T2_H3 = 256;  // 128: [*; U] dS'

__global__ void __launch_bounds__(kP2Threads, 1)
bwd_grad_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_dr, const __grid_constant__ CUtensorMap tm_s,
                const __grid_constant__ CUtensorMap tm_ds, const __grid_constant__ CUtensorMap tm_tb,
                const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_dk, BwdArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + R_BARS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + R_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + R_MISC + 4);
    float *g = reinterpret_cast<float *>(sm + R_F), *bet = g + 64, *gam = g + 128, *dl = g + 192, *dg = g + 256,
          *db = g + 320, *colsum = g + 384, *misc = g + 448;  // misc: scan scratch, <dS', S>, sum of w, ...
    // keep: log alpha_t at or above the forward's floor (its gradient passes)
    float *keep = g + 464;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t H = p.H, T = p.T;
    const int nch = p.chunks;
    const uint32_t sbase = smem_u32(sm);
    const int m = (warp & 3) * 32 + lane;  // TMEM lane / row of the 128-row tiles
    const int ch = warp >> 2;              // column half
    const uint32_t lb = (uint32_t)((warp & 3) * 32) << 16;

    if (tid == 0) {
        for (int i = 0; i < B2_COUNT; ++i) mbar_init(&bars[i], 1);
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

    auto issue_loads = [&](int64_t item) {  // thread 0
        const int64_t bh = item / nch;
        const int c = (int)(item % nch), b = (int)(bh / H), h = (int)(bh % H), t0 = c * kC;
        uint64_t *full = &bars[B2_LOAD];
        mbar_arrive_expect_tx(full, 32768 * 4);
        for (int blk = 0; blk < 2; ++blk) {
            tma_load_4d(sm + R_QK + blk * 16384, &tm_q, full, blk * 64, h, t0, b);
            tma_load_4d(sm + R_QK + blk * 16384 + 8192, &tm_k, full, blk * 64, h, t0, b);
            tma_load_4d(sm + R_DOR + blk * 16384, &tm_do, full, blk * 64, h, t0, b);
            tma_load_2d(sm + R_DOR + blk * 16384 + 8192, &tm_dr, full, blk * 64, (int)(item * 64));
            tma_load_2d(sm + R_S + blk * 16384, &tm_s, full, blk * 64, (int)(item * 128));
            tma_load_2d(sm + R_DS + blk * 16384, &tm_ds, full, blk * 64, (int)(item * 128));
        }
    };
    auto issue_loads_early = [&](int64_t item) {  // thread 0
        const int64_t bh = item / nch;
        const int c = (int)(item % nch), b = (int)(bh / H), h = (int)(bh % H), t0 = c * kC;
        uint64_t *full = &bars[B2_LOADE];
        mbar_arrive_expect_tx(full, 16384 + 8192);
        for (int blk = 0; blk < 2; ++blk) tma_load_4d(sm + R_V + blk * 8192, &tm_v, full, blk * 64, h, t0, b);
        tma_load_2d(sm + R_TB, &tm_tb, full, 0, (int)(item * 64));
    };
    if (tid == 0 && (int64_t)blockIdx.x < p.items) {
        issue_loads_early(blockIdx.x);
        issue_loads(blockIdx.x);
    }
#ifdef GDN_TC_DEBUG
    long long *const dbgp = (blockIdx.x == 0) ? g_bwd_dbg : nullptr;
    int nd = 0;
#endif

    bool ok = true;
    uint32_t lph = 0, mph = 0;
    auto mma_round = [&]() {
        const bool w = wait_bar(&bars[B2_MMA], mph, abort_flag);
        mph ^= 1u;
        ok = __syncthreads_and(w);
        tc_fence_after();
    };
    auto publish_smem = [&]() {  // generic-proxy shared-memory writes -> the next MMAs
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    };

#pragma unroll 1
    for (int64_t item = blockIdx.x; item < p.items && ok; item += gridDim.x) {
        const int64_t bh = item / nch;
        const int c = (int)(item % nch), b = (int)(bh / H), h = (int)(bh % H), t0 = c * kC;
        const int n = (T - t0 < kC) ? (int)(T - t0) : kC;
        const int64_t gbase = (int64_t)b * T * H + h;
        BDBG(0)
        // ---- gates (while the loads fly) ----
        chunk_gates(p.log_alpha, p.beta, gbase, H, t0, n, tid, g, bet, misc, 1, kP2Threads);
        if (tid < 64) {
            gam[tid] = expf(g[tid]);
            dl[tid] = expf(g[63] - g[tid]);
            dg[tid] = 0.f;
            db[tid] = 0.f;
            colsum[tid] = 0.f;
            // the clamp test of the d log alpha step below, its load in flight with the tiles'
            keep[tid] = (tid < n && p.log_alpha[gbase + (int64_t)(t0 + tid) * H] >= kLogAlphaFloor) ? 1.f : 0.f;
        }
        if (tid == 0) {
            misc[1] = 0.f;
            misc[2] = 0.f;
        }
        {
            const bool w = wait_bar(&bars[B2_LOAD], lph, abort_flag) && wait_bar(&bars[B2_LOADE], lph, abort_flag);
            lph ^= 1u;
            if (!(ok = __syncthreads_and(w))) break;  // also publishes the gates
        }
        BDBG(1)
        const float gC = expf(g[63]);
        // ---- round 1: G = [Q; K] K^T, Z = [Q; K] S^T, D2 = dS' K^T ----
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ka = sbase + R_QK + (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_ss(tm + T2_G, smem_desc_sw128(ka, 16, 1024), smem_desc_sw128(ka + 8192, 16, 1024), IDESC_64_KK,
                       kk > 0);
                mma_ss(tm + T2_Z, smem_desc_sw128(ka, 16, 1024),
                       smem_desc_sw128(sbase + R_S + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024), IDESC_128_KK,
                       kk > 0);
                mma_ss(tm + T2_D2, smem_desc_sw128(sbase + R_DS + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                       smem_desc_sw128(ka + 8192, 16, 1024), IDESC_64_KK, kk > 0);
            }
            mma_commit(&bars[B2_MMA]);
        }
        // <dS'_j, S_j> for d g_C, while round 1 runs (row j = m of both bf16 tiles, this thread's
        // 64-column box)
        {
            float acc = 0.f;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint32_t off = ch * 16384 + sw128(m, q);
                float x[8], y[8];
                unpack8(*reinterpret_cast<const uint4 *>(sm + R_DS + off), x);
                unpack8(*reinterpret_cast<const uint4 *>(sm + R_S + off), y);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc = fmaf(x[e], y[e], acc);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if ((tid & 31) == 0) atomicAdd(&misc[1], acc);
        }
        mma_round();
        if (!ok) break;
        BDBG(2)
        // ---- epilogue 1: rows t: d g_t from the outputs' gamma_t Q S^T term; rows 64 + t: X, Y ----
        if (m < 64) {
            const int t = m;
            float acc = 0.f;
#pragma unroll 1
            for (int pc = 2 * ch; pc < 2 * ch + 2; ++pc) {
                uint32_t z[32];
                tmem_ld32(tm + lb + T2_Z + 32 * pc, z);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int j0 = 32 * pc + 8 * q;
                    float o[8];
                    unpack8(*reinterpret_cast<const uint4 *>(sm + R_DOR + tile_off(t, j0, 16384)), o);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc = fmaf(__uint_as_float(z[8 * q + e]), o[e], acc);
                }
            }
            atomicAdd(&dg[t], gam[t] * acc);
        } else {
            const int t = m - 64;
            const float gt = gam[t], bt = bet[t];
            float ry = 0.f, rx = 0.f;
#pragma unroll 1
            for (int pc = 2 * ch; pc < 2 * ch + 2; ++pc) {
                uint32_t z[32];
                tmem_ld32(tm + lb + T2_Z + 32 * pc, z);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int j0 = 32 * pc + 8 * q;
                    uint4 *vp = reinterpret_cast<uint4 *>(sm + R_V + tile_off(t, j0, 8192));
                    float v[8], r[8], y[8];
                    unpack8(*vp, v);
                    unpack8(*reinterpret_cast<const uint4 *>(sm + R_DOR + tile_off(64 + t, j0, 16384)), r);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float x = gt * __uint_as_float(z[8 * q + e]);
                        y[e] = v[e] - x;
                        ry = fmaf(r[e], y[e], ry);
                        rx = fmaf(r[e], x, rx);
                    }
                    *vp = make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                                     pack_bf16x2(y[6], y[7]));
                }
            }
            atomicAdd(&db[t], ry);
            atomicAdd(&dg[t], -bt * rx);
        }
        publish_smem();
        BDBG(3)
        // ---- round 2: U^T = Y^T (T diag(beta))^T ----
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_ss(tm + T2_U, smem_desc_sw128(sbase + R_V + kk * 2048, 8192, 1024),
                       smem_desc_sw128(sbase + R_TB + kk * 32, 16, 1024), IDESC_64_MN_K, kk > 0);
            mma_commit(&bars[B2_MMA]);
        }
        mma_round();
        if (!ok) break;
        // round 2 has read this item's V (now Y) and T diag(beta): the next item's may land
        if (tid == 0 && item + gridDim.x < p.items) issue_loads_early(item + gridDim.x);
        BDBG(4)
        // ---- epilogue 2 (row j = tid): U^T into shared memory in bf16; w_s = dl_s sum_j U^T_js D2_js ----
        {
            const int j = m;
            {
                const int pc = ch;
                uint32_t u[32], d2[32];
                tmem_ld32(tm + lb + T2_U + 32 * pc, u);
                tmem_ld32(tm + lb + T2_D2 + 32 * pc, d2);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4 *>(sm + R_UT + sw128(j, 4 * pc + q)) =
                        make_uint4(pack_bf16x2(__uint_as_float(u[8 * q]), __uint_as_float(u[8 * q + 1])),
                                   pack_bf16x2(__uint_as_float(u[8 * q + 2]), __uint_as_float(u[8 * q + 3])),
                                   pack_bf16x2(__uint_as_float(u[8 * q + 4]), __uint_as_float(u[8 * q + 5])),
                                   pack_bf16x2(__uint_as_float(u[8 * q + 6]), __uint_as_float(u[8 * q + 7])));
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(u[i]) * __uint_as_float(d2[i]);
                atomicAdd(&colsum[32 * pc + lane], warp_colsum32(v));
            }
        }
        publish_smem();  // also publishes colsum
        if (tid < 64) {
            const float w = dl[tid] * colsum[tid];
            colsum[tid] = 0.f;
            atomicAdd(&dg[tid], -w);
            float x = w;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
            if ((tid & 31) == 0) atomicAdd(&misc[2], x);
        }
        BDBG(5)
        // the previous item's dQ / dK stores have read their staging in the A1 tile, which epilogue 3 writes
        if (tid == 0) bulk_wait_read0();
        // ---- round 3: [dO; dR] U^T ----
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_ss(tm + T2_DG, smem_desc_sw128(sbase + R_DOR + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                       smem_desc_sw128(sbase + R_UT + kk * 2048, 8192, 1024), IDESC_64_K_MN, kk > 0);
            mma_commit(&bars[B2_MMA]);
        }
        mma_round();
        if (!ok) break;
        BDBG(6)
        // ---- epilogue 3: dP o E, F, their d g and dbeta terms; the A1 operand of round 4 ----
        if (m < 64) {
            const int t = m;
            const float gt = g[t];
            float rs = 0.f;
            // A1 row t, columns 0..63: zero (each thread of the row half of them)
#pragma unroll
            for (int q = 4 * ch; q < 4 * ch + 4; ++q)
                *reinterpret_cast<uint4 *>(sm + R_A1 + sw128(t, q)) = make_uint4(0, 0, 0, 0);
            {
                const int pc = ch;
                uint32_t a[32], qk[32];
                tmem_ld32(tm + lb + T2_DG + 32 * pc, a);
                tmem_ld32(tm + lb + T2_G + 32 * pc, qk);
                tmem_wait_ld();
                float pe[32], cv[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int s = 32 * pc + i;
                    const float e = (s <= t) ? expf(gt - g[s]) : 0.f;
                    const float dp = __uint_as_float(a[i]);
                    const float gp = dp * e * __uint_as_float(qk[i]);  // dP_ts P_ts
                    rs += gp;
                    cv[i] = gp;
                    pe[i] = dp * e;
                    // (dP o E)^T: A1 row 64 + s, column t
                    *reinterpret_cast<uint16_t *>(sm + R_A1 + sw128(64 + s, t >> 3) + (t & 7) * 2) = bf16_bits(pe[i]);
                }
                // dP o E: A1 row t, columns 64 + s
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4 *>(sm + R_A1 + 16384 + sw128(t, 4 * pc + q)) =
                        make_uint4(pack_bf16x2(pe[8 * q], pe[8 * q + 1]), pack_bf16x2(pe[8 * q + 2], pe[8 * q + 3]),
                                   pack_bf16x2(pe[8 * q + 4], pe[8 * q + 5]), pack_bf16x2(pe[8 * q + 6], pe[8 * q + 7]));
                atomicAdd(&colsum[32 * pc + lane], warp_colsum32(cv));
            }
            atomicAdd(&dg[t], rs);
        } else {
            const int t = m - 64;
            const float gt = g[t], bt = bet[t];
            float rs = 0.f, bs = 0.f;
            {
                const int pc = ch;
                uint32_t a[32], kk2[32];
                tmem_ld32(tm + lb + T2_DG + 32 * pc, a);
                tmem_ld32(tm + lb + T2_G + 32 * pc, kk2);
                tmem_wait_ld();
                float cv[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int s = 32 * pc + i;
                    float f = 0.f, ga = 0.f;
                    if (s < t) {
                        const float e = expf(gt - g[s]);
                        const float da = -__uint_as_float(a[i]);     // dA_ts
                        const float ek = e * __uint_as_float(kk2[i]);  // E_ts (k_t . k_s)
                        bs = fmaf(da, ek, bs);
                        ga = da * bt * ek;  // dA_ts A_ts
                        f = da * bt * e;
                        // (F + F^T): row 64 + s, column 64 + t
                        *reinterpret_cast<uint16_t *>(sm + R_A1 + 16384 + sw128(64 + s, t >> 3) + (t & 7) * 2) =
                            bf16_bits(f);
                    }
                    rs += ga;
                    cv[i] = ga;
                    // (F + F^T): row 64 + t, column 64 + s for s <= t (F_ts, zero on the diagonal)
                    if (s <= t)
                        *reinterpret_cast<uint16_t *>(sm + R_A1 + 16384 + sw128(64 + t, s >> 3) + (s & 7) * 2) =
                            bf16_bits(f);
                }
                atomicAdd(&colsum[32 * pc + lane], warp_colsum32(cv));
            }
            atomicAdd(&dg[t], rs);
            atomicAdd(&db[t], bs);
        }
        publish_smem();  // A1 and colsum
        BDBG(7)
        if (tid < 64) atomicAdd(&dg[tid], -colsum[tid]);
        // ---- round 4: [dQ; dK] = A1 [Q; K] + (scaled) [dO; dR] S + [*; U] dS' ----
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                mma_ss(tm + T2_H1, smem_desc_sw128(sbase + R_A1 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                       smem_desc_sw128(sbase + R_QK + kk * 2048, 16384, 1024), IDESC_128_K_MN, kk > 0);
                mma_ss(tm + T2_H2, smem_desc_sw128(sbase + R_DOR + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                       smem_desc_sw128(sbase + R_S + kk * 2048, 16384, 1024), IDESC_128_K_MN, kk > 0);
                // A MN-major over two 64-row blocks: block 0 (rows 0..63, not used) any finite tile, block 1
                // (rows 64..127) U^T
                mma_ss(tm + T2_H3, smem_desc_sw128(sbase + R_S + 16384 + kk * 2048, R_UT - (R_S + 16384), 1024),
                       smem_desc_sw128(sbase + R_DS + kk * 2048, 16384, 1024), IDESC_128_MN_MN, kk > 0);
            }
            mma_commit(&bars[B2_MMA]);
        }
        mma_round();
        if (!ok) break;
        BDBG(8)
        // every MMA of this item is done: the next item's tiles may land while this one finishes
        if (tid == 0 && item + gridDim.x < p.items) issue_loads(item + gridDim.x);
        // ---- epilogue 4: dQ (rows t), dK (rows 64 + s), staged in the A1 tile (free once round 4 is done:
        //      [dQ box 0 | dQ box 1 | dK box 0 | dK box 1], 64 rows x 64 columns each) for TMA stores ----
        {
            const int r = m & 63;
            const bool isq = m < 64;
            const float f2 = isq ? gam[r] : -bet[r] * gam[r], f3 = dl[r];
            uint8_t *const stg = sm + R_A1 + ((isq ? 0 : 2) + ch) * 8192;
#pragma unroll 1
            for (int pc = 2 * ch; pc < 2 * ch + 2; ++pc) {
                uint32_t x1[32], x2[32], x3[32];
                tmem_ld32(tm + lb + T2_H1 + 32 * pc, x1);
                tmem_ld32(tm + lb + T2_H2 + 32 * pc, x2);
                tmem_ld32(tm + lb + T2_H3 + 32 * pc, x3);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    float v0 = fmaf(f2, __uint_as_float(x2[i]), __uint_as_float(x1[i]));
                    float v1 = fmaf(f2, __uint_as_float(x2[i + 1]), __uint_as_float(x1[i + 1]));
                    if (!isq) {
                        v0 = fmaf(f3, __uint_as_float(x3[i]), v0);
                        v1 = fmaf(f3, __uint_as_float(x3[i + 1]), v1);
                    }
                    pk[i >> 1] = pack_bf16x2(v0, v1);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4 *>(stg + sw128(r, 4 * (pc - 2 * ch) + q)) =
                        make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            // rows past the sequence's end are outside the tensor and not written
            for (int blk = 0; blk < 2; ++blk) {
                tma_store_4d(&tm_dq, sm + R_A1 + blk * 8192, blk * 64, h, t0, b);
                tma_store_4d(&tm_dk, sm + R_A1 + (2 + blk) * 8192, blk * 64, h, t0, b);
            }
            bulk_commit();
        }
        BDBG(9)
        // ---- dbeta and d log alpha_r = sum_{t >= r} dg_t + dg_C (zero where log alpha was clamped):
        //      a suffix sum over the two warps' 32 tokens each, then warp 0 adds warp 1's total ----
        if (tid < 64) {
            float x = dg[tid];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_down_sync(0xffffffffu, x, o);
                if (lane + o < 32) x += y;
            }
            if (tid == 32) misc[3] = x;
            named_bar(2, 64);
            if (tid < 32) x += misc[3];
            if (tid < n) {
                const int64_t gi = gbase + (int64_t)(t0 + tid) * H;
                p.dlog_alpha[gi] = keep[tid] != 0.f ? x + (gC * misc[1] + misc[2]) : 0.f;
                p.dbeta[gi] = db[tid];
            }
        }
        tc_fence_before();
        __syncthreads();  // TMEM and the gate buffers are free for the next item
        tc_fence_after();
        BDBG(10)
#ifdef GDN_TC_DEBUG
        ++nd;
#endif
    }
    if (!ok) *abort_flag = 1;
    if (tid == 0) {
        bulk_wait0();  // every dQ / dK store has completed
        // after an abort, tile loads of the next item may still be in flight: bounded waits for them
        if (!ok) {
            mbar_wait(&bars[B2_LOADE], lph, 1u << 20);
            mbar_wait(&bars[B2_LOAD], lph, 1u << 20);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) atomicExch(&g_bwd_timeout, 1);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, 512);
    }
}

bool configure(const void *fn, uint32_t smem, std::atomic<uint64_t> &done) {
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (done.load() & bit) return true;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) return false;
    done.fetch_or(bit);
    return true;
}

struct TcLayout {
    size_t fwd_ws, fwd_out, ckpt, tt, ds, dr, seg, total;
    int nseg;               // segments asked of the forward recompute
    int seg_len, nseg_run;  // chunks per segment and the segments they make (the forward's own rounding)
};

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

TcLayout tc_layout(const BwdProblem &p, int sm_count) {
    const FwdProblem &f = p.f;
    const int64_t nch = (f.T + kC - 1) / kC, items = f.B * f.H * nch, ntok = f.B * f.T * f.H;
    TcLayout l;
    l.nseg = fwd_tc_segments(f, sm_count, true);
    l.fwd_ws = round256(fwd_split_workspace_bytes(f, l.nseg));
    l.fwd_out = round256((size_t)ntok * kD * 2);
    l.ckpt = round256((size_t)items * kD * kD * 2);
    l.tt = round256((size_t)items * kC * kC * 2);
    l.ds = round256((size_t)items * kD * kD * 2);
    l.dr = round256((size_t)items * kC * kD * 2);
    l.seg_len = (int)((nch + l.nseg - 1) / l.nseg);
    l.nseg_run = (int)((nch + l.seg_len - 1) / l.seg_len);
    // reverse segments: B', X and the entry adjoints of every transfer slot, and their flags
    const size_t slots = (size_t)(f.B * f.H) * (size_t)(l.nseg_run - 1);
    l.seg = l.nseg_run > 1 ? round256(3 * slots * kD * kD * sizeof(float)) + round256(slots * sizeof(int)) : 0;
    l.total = l.fwd_ws + l.fwd_out + l.ckpt + l.tt + l.ds + l.dr + l.seg;
    return l;
}

}  // namespace

#ifdef GDN_TC_DEBUG
extern "C" int gdn_debug_set_bwd_dump(long long *ptr) {
    return cudaMemcpyToSymbol(g_bwd_dbg, &ptr, sizeof(ptr)) == cudaSuccess ? 0 : 1;
}
extern "C" int gdn_debug_set_bwd1_dump(long long *ptr) {
    return cudaMemcpyToSymbol(g_bwd1_dbg, &ptr, sizeof(ptr)) == cudaSuccess ? 0 : 1;
}
#endif

bool take_bwd_timeout() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_bwd_timeout, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (v) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_bwd_timeout, &zero, sizeof(int));
    }
    return v != 0;
}

// The tensor-core backward takes the shapes of the two-kernel forward with one head per memory,
// unless GDN_BWD_PATH=simt or GDN_BWD_RECOMPUTE=simt asks for the CUDA-core one.
bool bwd_tc_supported(const BwdProblem &p) {
    const char *e1 = getenv("GDN_BWD_PATH"), *e2 = getenv("GDN_BWD_RECOMPUTE");
    if ((e1 && strcmp(e1, "simt") == 0) || (e2 && strcmp(e2, "simt") == 0)) return false;
    const FwdProblem &f = p.f;
    const int64_t nch = (f.T + kC - 1) / kC, items = f.B * f.H * nch;
    return f.dtype == GDN_BF16 && f.dk == kD && f.dv == kD && f.chunk == kC && f.group == 1 && !f.raw_inputs &&
           fwd_split_supported(f) && items * 128 < ((int64_t)1 << 31) && nch < ((int64_t)1 << 24);
}

size_t bwd_tc_workspace_bytes(const BwdProblem &p, int sm_count) { return tc_layout(p, sm_count).total; }

cudaError_t launch_bwd_tc(const BwdProblem &p, int sm_count, void *workspace, cudaStream_t stream) {
    const FwdProblem &f = p.f;
    if (f.B * f.H == 0 || f.T == 0) return cudaSuccess;
    if (!workspace) return cudaErrorInvalidValue;
    const TcLayout l = tc_layout(p, sm_count);
    const int64_t nch = (f.T + kC - 1) / kC, items = f.B * f.H * nch;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint8_t *fwd_ws = ws, *fwd_out = ws + l.fwd_ws, *ckpt = fwd_out + l.fwd_out, *tt = ckpt + l.ckpt,
            *dsw = tt + l.tt, *drw = dsw + l.ds, *segw = drw + l.dr;
    cudaError_t e;
    // forward recompute: bf16 checkpoints, T of every chunk, P and T diag(beta) in the workspace
    if ((e = cudaMemsetAsync(tt, 0, (size_t)items * kC * kC * 2, stream)) != cudaSuccess) return e;
    FwdProblem fc = f;
    fc.out = fwd_out;
    fc.S_final = nullptr;
    fc.ckpt = reinterpret_cast<float *>(ckpt);
    fc.ckpt_bf16 = 1;
    fc.t_out = tt;
    fc.raw_inputs = 0;
    if ((e = launch_fwd_split(fc, l.nseg, sm_count, fwd_ws, stream)) != cudaSuccess) return e;
    void *p_tiles = nullptr, *tb_tiles = nullptr;
    fwd_split_ws_tiles(fwd_ws, items, &p_tiles, &tb_tiles);

    CUtensorMap mq, mk, mv, mdo, mp, mt, mtb, mdr, ms, mds, mdq, mdk, mdv;
    if (!make_map_bthd(&mq, f.q, f.B, f.T, f.H) || !make_map_bthd(&mk, f.k, f.B, f.T, f.H) ||
        !make_map_bthd(&mv, f.v, f.B, f.T, f.H) || !make_map_bthd(&mdo, p.d_out, f.B, f.T, f.H) ||
        !make_map_bthd(&mdq, p.dq, f.B, f.T, f.H) || !make_map_bthd(&mdk, p.dk, f.B, f.T, f.H) ||
        !make_map_bthd(&mdv, p.dv, f.B, f.T, f.H) ||
        !make_map_tiles(&mp, p_tiles, items, 64) || !make_map_tiles(&mt, tt, items, 64) ||
        !make_map_tiles(&mtb, tb_tiles, items, 64) || !make_map_rows128(&mdr, drw, items * 64, 64) ||
        !make_map_rows128(&ms, ckpt, items * 128, 128) || !make_map_rows128(&mds, dsw, items * 128, 128))
        return cudaErrorInvalidValue;
    static std::atomic<uint64_t> conf1{0}, conf2{0};
    if (!configure((const void *)bwd_chain_kernel, SMEM_P1, conf1) ||
        !configure((const void *)bwd_grad_kernel, SMEM_P2, conf2))
        return cudaErrorInvalidValue;
    BwdArgs a;
    a.log_alpha = f.log_alpha;
    a.beta = f.beta;
    a.dS_final = p.dS_final;
    a.dS0 = p.dS0;
    a.dv = static_cast<__nv_bfloat16 *>(p.dv);
    a.dq = static_cast<__nv_bfloat16 *>(p.dq);
    a.dk = static_cast<__nv_bfloat16 *>(p.dk);
    a.dlog_alpha = p.dlog_alpha;
    a.dbeta = p.dbeta;
    a.ds_ws = reinterpret_cast<__nv_bfloat16 *>(dsw);
    a.dr_ws = reinterpret_cast<__nv_bfloat16 *>(drw);
    a.T = f.T;
    a.H = f.H;
    a.items = items;
    a.chunks = (int)nch;
    a.nseg = l.nseg_run;
    a.seg_len = l.seg_len;
    a.gate_rec = fwd_split_ws_gates(fwd_ws, items);
    a.entry = nullptr;
    a.xb = a.xm = nullptr;
    a.xflag = nullptr;
    const int64_t heads = f.B * f.H;
    if (l.nseg_run > 1) {
        // long sequences with few heads: the segments' reverse transfers, their prefix from dS_final
        // (the adjoint leaving every segment), then every segment's walk at once
        const size_t per = (size_t)heads * (size_t)(l.nseg_run - 1) * kD * kD;
        a.xb = reinterpret_cast<float *>(segw);
        a.xm = a.xb + per;
        float *entry = a.xm + per;
        a.xflag = reinterpret_cast<int *>(segw + round256(3 * per * sizeof(float)));
        a.mode = 1;
        {
            TimedLaunch tl_(GDN_KERNEL_TRANSFER, stream);
            bwd_chain_kernel<<<(unsigned)(heads * (l.nseg_run - 1) * 2), kP1Threads, SMEM_P1, stream>>>(
                mdo, mq, mk, mp, mt, mds, mdr, mdv, a);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if ((e = launch_seg_prefix(p.dS_final, a.xb, a.xm, a.xflag, entry, heads, l.nseg_run, stream, nullptr)) !=
            cudaSuccess)
            return e;
        a.entry = entry;
    }
    a.mode = 0;
    {
        TimedLaunch tl_(GDN_KERNEL_BACKWARD, stream);
        bwd_chain_kernel<<<(unsigned)(heads * l.nseg_run), kP1Threads, SMEM_P1, stream>>>(mdo, mq, mk, mp, mt, mds,
                                                                                       mdr, mdv, a);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    {
        const int64_t grid = items < (int64_t)sm_count ? items : (int64_t)sm_count;
        TimedLaunch tl_(GDN_KERNEL_BACKWARD, stream);
        bwd_grad_kernel<<<(unsigned)grid, kP2Threads, SMEM_P2, stream>>>(mq, mk, mv, mdo, mdr, ms, mds, mtb, mdq,
                                                                          mdk, a);
    }
    return cudaGetLastError();
}

}  // namespace gdn
