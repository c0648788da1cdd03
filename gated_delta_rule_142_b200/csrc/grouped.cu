// grouped.cu -- state copies for grouped heads.
//
// With grouped heads (H query heads reading the memories of H / group
// key-value heads), the forward kernels keep one state per query head: each
// query head of a group recomputes its group's memory.  These two copies
// translate between the caller's per-key-value-head states and those:
//     expand:  dst[b, h]  = src[b, h / group]     h  < H
//     pick:    dst[b, hk] = src[b, hk * group]    hk < H / group
// with n floats per state.  Both are plain HBM copies.
#include "gdn.h"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kCopyThreads = 256;

__global__ void __launch_bounds__(kCopyThreads)
copy_states_kernel(const float *__restrict__ src, float *__restrict__ dst, int64_t n_dst_states, int64_t H,
                   int group, int64_t n4, bool expand) {
    const int64_t Hkv = H / group;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_dst_states * n4;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t st = i / n4, e = i % n4;
        int64_t from;
        if (expand) {  // dst state (b, h) <- src (b, h / group)
            const int64_t b = st / H, h = st % H;
            from = b * Hkv + h / group;
        } else {  // dst state (b, hk) <- src (b, hk * group)
            const int64_t b = st / Hkv, hk = st % Hkv;
            from = b * H + hk * group;
        }
        reinterpret_cast<float4 *>(dst)[i] = reinterpret_cast<const float4 *>(src)[from * n4 + e];
    }
}

cudaError_t launch(const float *src, float *dst, int64_t states, int64_t H, int group, int64_t n, bool expand,
                   cudaStream_t stream) {
    if (states <= 0 || n <= 0) return cudaSuccess;
    const int64_t n4 = n / 4, total = states * n4;
    const int64_t blocks = (total + kCopyThreads - 1) / kCopyThreads;
    copy_states_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), kCopyThreads, 0, stream>>>(src, dst, states, H,
                                                                                             group, n4, expand);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_expand_states(const float *src, float *dst, int64_t B, int64_t H, int group, int64_t n,
                                 cudaStream_t stream) {
    return launch(src, dst, B * H, H, group, n, true, stream);
}

cudaError_t launch_pick_states(const float *src, float *dst, int64_t B, int64_t H, int group, int64_t n,
                               cudaStream_t stream) {
    return launch(src, dst, B * (H / group), H, group, n, false, stream);
}

}  // namespace gdn
