// grouped_out.cu -- outputs of the query heads that share a key-value head's
// memory, on the tensor cores (bf16, d = 128, chunk = 64).
//
// With grouped heads (8 query / 2 key-value heads in ATMA, Sec. 3.1; the
// memory is the Sec. 3.3 recurrence of "ATMA: Long-Context Language Modeling
// via Polar Attention and Gated-Delta Compression Memory"), the memory of
// key-value head hk is written by that head's k, v and gates only, so every
// query head of the group reads the same states S and the same chunk
// corrections U.  The two-kernel forward in lead mode runs one chain per
// key-value head (query head hk * G) and leaves behind, per chunk, the state
// entering it (bf16) and U^T (bf16).  This kernel forms, chunk-parallel, the
// outputs of the other query heads r = 1 .. G - 1 of each group:
//     O^T = S (diag(gamma) Q_r)^T + U^T P_r^T
// with Q_r the query head's tile, P_r its decayed, masked Q_r K^T tile and
// gamma its gate scales, both from the prep kernel's workspace item of that
// query head.  Two MMAs into one 128 x 64 accumulator per chunk; persistent
// CTAs, three per SM, each over a contiguous range of (memory chunk, query
// head) steps with the query head fastest, so that S and U^T load once for the
// query heads of a group that a CTA takes in a row.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

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
constexpr int kGrpThreads = 128;  // thread j = TMEM lane = value dim j
constexpr int kRecFloats = 132;   // the prep kernel's gate record: gamma_t (with 1 / |q_t| folded in) first

constexpr uint32_t G_S = 0;       // 32 KB: S (bf16) [128 j][64 i] x 2 boxes
constexpr uint32_t G_U = 32768;   // 16 KB: U^T [128 j][64 s]
constexpr uint32_t G_Q = 49152;   // 16 KB: Q [64 t][64 i] x 2 boxes, scaled by gamma in place
constexpr uint32_t G_P = 65536;   // 8 KB:  P [t][s]
constexpr uint32_t G_GAM = 73728;  // 64 floats
constexpr uint32_t G_BARS = G_GAM + 256;
constexpr uint32_t G_MISC = G_BARS + 64;
constexpr uint32_t SMEM_GRP = G_MISC + 64 + 1024;
static_assert(3 * (SMEM_GRP + 1024) <= 233472, "three output CTAs no longer fit an SM");

constexpr uint32_t IDESC_O = instr_desc_bf16(128, 64, 0, 0);

__device__ int g_grp_timeout;

struct GrpArgs {
    const float *gates;  // [items][kRecFloats]: the prep kernel's records, every query head
    __nv_bfloat16 *out;  // [B, T, H, 128]
    int64_t T, H, items;  // items: B * Hkv * chunks * (G - 1), the query head fastest
    int64_t per;          // items per CTA (a contiguous range)
    int chunks, group;
};

__global__ void __launch_bounds__(kGrpThreads, 3)
grouped_out_kernel(const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CUtensorMap tm_u,
                   const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_p, GrpArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + G_BARS);  // [0] loads, [1] MMA
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + G_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + G_MISC + 4);
    float *gam = reinterpret_cast<float *>(sm + G_GAM);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int j = tid;
    const uint32_t lb = (uint32_t)(warp * 32) << 16;
    const uint32_t sbase = smem_u32(sm);
    const int64_t H = p.H, T = p.T;
    const int G = p.group, nch = p.chunks;
    const int64_t Hkv = H / G;

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 64);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;

    // item -> (b, hk, c, r): query head h = hk * G + r, memory index m = b * Hkv + hk; the memory chunk
    // m * nch + c is item / (G - 1)
    struct Coord {
        int b, h, c;
        int64_t m, wi;  // memory index, the query head's workspace item
    };
    auto coord = [&](int64_t it) {
        Coord x;
        const int r = 1 + (int)(it % (G - 1));
        int64_t rest = it / (G - 1);
        x.c = (int)(rest % nch);
        rest /= nch;
        const int hk = (int)(rest % Hkv);
        x.b = (int)(rest / Hkv);
        x.h = hk * G + r;
        x.m = (int64_t)x.b * Hkv + hk;
        x.wi = ((int64_t)x.b * H + x.h) * nch + x.c;
        return x;
    };
    // this CTA's range of items
    const int64_t first = (int64_t)blockIdx.x * p.per;
    const int64_t last = (first + p.per < p.items) ? first + p.per : p.items;
    // S and U^T of item `it`'s memory chunk load unless the item before it in this range had them
    auto issue_loads = [&](int64_t it) {  // thread 0
        const Coord x = coord(it);
        const bool su = it == first || it / (G - 1) != (it - 1) / (G - 1);
        mbar_arrive_expect_tx(&bars[0], (su ? 32768 + 16384 : 0) + 16384 + 8192);
        if (su) {
            const int64_t ci = x.m * nch + x.c;  // checkpoint / U^T index of the memory
            for (int blk = 0; blk < 2; ++blk)
                tma_load_2d(sm + G_S + blk * 16384, &tm_s, &bars[0], blk * 64, (int)(ci * 128));
            tma_load_2d(sm + G_U, &tm_u, &bars[0], 0, (int)(ci * 128));
        }
        for (int blk = 0; blk < 2; ++blk)
            tma_load_4d(sm + G_Q + blk * 8192, &tm_q, &bars[0], blk * 64, x.h, x.c * kC, x.b);
        tma_load_2d(sm + G_P, &tm_p, &bars[0], 0, (int)(x.wi * 64));
    };
    if (tid == 0 && first < last) issue_loads(first);

    bool ok = true;
    uint32_t ph = 0;
#pragma unroll 1
    for (int64_t it = first; it < last && ok; ++it, ph ^= 1u) {
        const Coord x = coord(it);
        const int t0 = x.c * kC;
        const int n = (T - t0 < kC) ? (int)(T - t0) : kC;
        if (tid < 64) gam[tid] = p.gates[x.wi * kRecFloats + tid];
        if (!(ok = __syncthreads_and(wait_bar(&bars[0], ph, abort_flag)))) break;
        // Q rows scaled by gamma_t in place (16-byte unit u: box u >> 9, row (u >> 3) & 63)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int u = tid + 128 * i;
            uint4 *ptr = reinterpret_cast<uint4 *>(sm + G_Q) + u;
            const uint4 w = *ptr;
            const float f = gam[(u >> 3) & 63];
            const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&wv[e]));
                o[e] = pack_bf16x2(v.x * f, v.y * f);
            }
            *ptr = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_ss(tm, smem_desc_sw128(sbase + G_S + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                       smem_desc_sw128(sbase + G_Q + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), IDESC_O, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_ss(tm, smem_desc_sw128(sbase + G_U + kk * 32, 16, 1024),
                       smem_desc_sw128(sbase + G_P + kk * 32, 16, 1024), IDESC_O, 1u);
            mma_commit(&bars[1]);
        }
        if (!(ok = __syncthreads_and(wait_bar(&bars[1], ph, abort_flag)))) break;
        tc_fence_after();
        // the tiles are read: the next item's loads may land while this one's outputs leave
        if (tid == 0 && it + 1 < last) issue_loads(it + 1);
        // O^T row j -> out[b, t0 + t, h, j]
        __nv_bfloat16 *dst = p.out + (((int64_t)x.b * T + t0) * H + x.h) * kD + j;
#pragma unroll 1
        for (int pc = 0; pc < 2; ++pc) {
            uint32_t r[32];
            tmem_ld32(tm + lb + 32 * pc, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int t = 32 * pc + i;
                if (t < n) dst[(int64_t)t * H * kD] = __float2bfloat16_rn(__uint_as_float(r[i]));
            }
        }
        tc_fence_before();
        __syncthreads();  // TMEM and gam are free for the next item
        tc_fence_after();
    }
    if (!ok) *abort_flag = 1;
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) atomicExch(&g_grp_timeout, 1);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, 64);
    }
}

inline bool make_map_rows(CUtensorMap *m, const void *base, int64_t rows, uint32_t cols, uint32_t box_rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[2] = {cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool take_grouped_timeout() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_grp_timeout, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (v) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_grp_timeout, &zero, sizeof(int));
    }
    return v != 0;
}

cudaError_t launch_grouped_outputs(const FwdProblem &p, const void *ckpt, const void *u, const void *p_tiles,
                                   const float *gates, int sm_count, cudaStream_t stream) {
    const int G = p.group;
    if (G < 2 || p.H % G) return cudaErrorInvalidValue;
    const int64_t nch = (p.T + kC - 1) / kC, Hkv = p.H / G;
    const int64_t mems = p.B * Hkv * nch, items = p.B * Hkv * (G - 1) * nch;
    if (items == 0) return cudaSuccess;
    if (mems * 128 >= ((int64_t)1 << 31) || p.B * p.H * nch * 64 >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    CUtensorMap ms, mu, mq, mp;
    if (!make_map_rows(&ms, ckpt, mems * 128, 128, 128) || !make_map_rows(&mu, u, mems * 128, 64, 128) ||
        !make_map_bthd(&mq, p.q, p.B, p.T, p.H) || !make_map_rows(&mp, p_tiles, p.B * p.H * nch * 64, 64, 64))
        return cudaErrorInvalidValue;
    static std::atomic<uint64_t> conf{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(conf.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(grouped_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SMEM_GRP);
        if (e != cudaSuccess) return e;
        conf.fetch_or(bit);
    }
    GrpArgs a;
    a.gates = gates;
    a.out = static_cast<__nv_bfloat16 *>(p.out);
    a.T = p.T;
    a.H = p.H;
    a.items = items;
    a.chunks = (int)nch;
    a.group = G;
    const int64_t ctas = items < 3 * (int64_t)sm_count ? items : 3 * (int64_t)sm_count;
    a.per = (items + ctas - 1) / ctas;
    const int64_t grid = (items + a.per - 1) / a.per;
    {
        TimedLaunch tl_(GDN_KERNEL_GROUP_OUT, stream);
        grouped_out_kernel<<<(unsigned)grid, kGrpThreads, SMEM_GRP, stream>>>(ms, mu, mq, mp, a);
    }
    return cudaGetLastError();
}

}  // namespace gdn
