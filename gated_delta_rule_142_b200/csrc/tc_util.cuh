// tc_util.cuh -- helpers shared by the tcgen05 forward kernels: role
// hand-offs (bounded mbarrier waits, named barriers), the 128-byte swizzle
// address of a shared-memory tile, warp-level TF32 MMA fragments for the
// 64x64 triangular inverse, the 64-token chunk cumsum, and host-side TMA
// tensor-map encoding.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "sm100.cuh"

namespace gdn {
namespace tcu {

using namespace sm100;

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

// ---- warp-level TF32 MMA (m16n8k8, fp32 accumulate) for the 64x64 inverse ----
// Fragment ownership, g = lane / 4, t = lane % 4:
//   A 16x8: a0 (g, t), a1 (g+8, t), a2 (g, t+4), a3 (g+8, t+4)
//   B  8x8: b0 (t, g), b1 (t+4, g)
//   D 16x8: d0 (g, 2t), d1 (g, 2t+1), d2 (g+8, 2t), d3 (g+8, 2t+1)
__device__ __forceinline__ uint32_t tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// A fragment from a row-major fp32 matrix M (row stride ld), rows r0.., columns k0..
__device__ __forceinline__ void load_a(uint32_t (&a)[4], const float *M, int ld, int r0, int k0, int g, int t) {
    a[0] = tf32(M[(r0 + g) * ld + k0 + t]);
    a[1] = tf32(M[(r0 + g + 8) * ld + k0 + t]);
    a[2] = tf32(M[(r0 + g) * ld + k0 + t + 4]);
    a[3] = tf32(M[(r0 + g + 8) * ld + k0 + t + 4]);
}
// B fragment (K x N) from a row-major fp32 matrix M: element (k, n) = M[k0 + k][n0 + n]
__device__ __forceinline__ void load_b(uint32_t (&b)[2], const float *M, int ld, int k0, int n0, int g, int t) {
    b[0] = tf32(M[(k0 + t) * ld + n0 + g]);
    b[1] = tf32(M[(k0 + t + 4) * ld + n0 + g]);
}
// Store -D (16x8 fragment) into a row-major fp32 matrix at (r0, c0).
__device__ __forceinline__ void store_neg_d(float *M, int ld, int r0, int c0, const float (&d)[4], int g, int t) {
    *reinterpret_cast<float2 *>(M + (r0 + g) * ld + c0 + 2 * t) = make_float2(-d[0], -d[1]);
    *reinterpret_cast<float2 *>(M + (r0 + g + 8) * ld + c0 + 2 * t) = make_float2(-d[2], -d[3]);
}
__device__ __forceinline__ void store_d(float *M, int ld, int r0, int c0, const float (&d)[4], int g, int t) {
    *reinterpret_cast<float2 *>(M + (r0 + g) * ld + c0 + 2 * t) = make_float2(d[0], d[1]);
    *reinterpret_cast<float2 *>(M + (r0 + g + 8) * ld + c0 + 2 * t) = make_float2(d[2], d[3]);
}

// Writes entries (row, col) and (row, col + 1) (col even) of T diag(beta) and
// T diag(beta gamma) into their bf16 K-major 128-byte-swizzled tiles.
__device__ __forceinline__ void store_t_pair(uint8_t *tb, uint8_t *tbg, int row, int col, float v0, float v1,
                                             const float *bet, const float *gam) {
    const uint32_t off = sw128(row, col >> 3) + (col & 7) * 2;
    const float b0 = bet[col], b1 = bet[col + 1];
    *reinterpret_cast<uint32_t *>(tb + off) = pack_bf16x2(v0 * b0, v1 * b1);
    *reinterpret_cast<uint32_t *>(tbg + off) = pack_bf16x2(v0 * b0 * gam[col], v1 * b1 * gam[col + 1]);
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

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
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
inline bool make_map_bthd(CUtensorMap *m, const void *base, int64_t B, int64_t T, int64_t H) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {128 * 2, (cuuint64_t)(H * 128 * 2), (cuuint64_t)(T * H * 128 * 2)};
    const cuuint32_t box[4] = {64, 1, 64, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A stack of bf16 tiles of `rows_per_tile` rows x 64 columns (128-byte rows),
// `ntiles` of them back to back, viewed as one [ntiles * rows_per_tile][64]
// matrix; box = one whole tile, 128-byte swizzle.
inline bool make_map_tiles(CUtensorMap *m, const void *base, int64_t ntiles, uint32_t rows_per_tile) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[2] = {64, (cuuint64_t)(ntiles * rows_per_tile)};
    const cuuint64_t strides[1] = {64 * 2};
    const cuuint32_t box[2] = {64, rows_per_tile};
    const cuuint32_t estr[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tcu
}  // namespace gdn
