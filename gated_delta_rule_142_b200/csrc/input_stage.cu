// input_stage.cu -- the memory's input stage as a pass of its own.
//
// The gated-delta memory ("ATMA: Long-Context Language Modeling via Polar
// Attention and Gated-Delta Compression Memory", Sec. 3.3; App. A.2 takes
// ||q_t|| = ||k_t|| = 1) reads unit-norm queries and keys, a decay alpha_t in
// (0, 1) and a write strength beta_t in (0, 1).  From the layer's raw
// projections this pass forms
//     q_t / sqrt(|q_t|^2 + eps),  k_t / sqrt(|k_t|^2 + eps),
//     log alpha_t = -softplus(x_alpha),  beta_t = sigmoid(x_beta),
// for every (token, head) row.  The two-kernel tensor-core forward and the
// decode step fold this stage into their own loads; the other forwards run
// this pass first, into scratch.  It is bound by HBM: each row is read once
// and written once.
//
// Mapping: a row of dk elements is held by dk/4 consecutive lanes, four
// elements per lane; a warp covers 32/(dk/4) rows per step, grid-stride.
#include "common.cuh"
#include "gdn.h"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kStageThreads = 256;

__device__ __forceinline__ void store4(float *p, float4 x) { *reinterpret_cast<float4 *>(p) = x; }
__device__ __forceinline__ void store4(__nv_bfloat16 *p, float4 x) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(x.x, x.y), hi = __floats2bfloat162_rn(x.z, x.w);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t *>(&lo);
    u.y = *reinterpret_cast<const uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(p) = u;
}

__device__ __forceinline__ float4 scale4(float4 x, float s) { return make_float4(x.x * s, x.y * s, x.z * s, x.w * s); }

template <typename Tin, int DK>
__global__ void __launch_bounds__(kStageThreads)
input_stage_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const float *__restrict__ x_alpha,
                   const float *__restrict__ x_beta, Tin *__restrict__ qn, Tin *__restrict__ kn,
                   float *__restrict__ log_alpha, float *__restrict__ beta, int64_t rows) {
    constexpr int LPR = DK / 4;    // lanes per row
    constexpr int RPW = 32 / LPR;  // rows per warp per step
    const int lane = threadIdx.x & 31, grp = lane / LPR, gl = lane % LPR;
    const int64_t warps = (int64_t)gridDim.x * (kStageThreads / 32);
    // the loop bound is the same for every lane of a warp, so all of them take the shuffles below;
    // rows past the end only skip the memory accesses
    for (int64_t base = ((int64_t)blockIdx.x * (kStageThreads / 32) + (threadIdx.x >> 5)) * RPW; base < rows;
         base += warps * RPW) {
        const int64_t r = base + grp;
        const bool live = r < rows;
        const int64_t off = r * DK + 4 * gl;
        const float4 qf = live ? load4(q + off) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 kf = live ? load4(k + off) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float qq = group_sum<LPR>(dot4(qf, qf)), kk = group_sum<LPR>(dot4(kf, kf));
        if (!live) continue;
        store4(qn + off, scale4(qf, rsqrtf(qq + kNormEps)));
        store4(kn + off, scale4(kf, rsqrtf(kk + kNormEps)));
        if (gl == 0) {
            const float xa = x_alpha[r], xb = x_beta[r];
            log_alpha[r] = -(fmaxf(xa, 0.f) + log1pf(expf(-fabsf(xa))));
            beta[r] = 1.f / (1.f + expf(-xb));
        }
    }
}

template <typename Tin, int DK>
cudaError_t launch_t(const void *q, const void *k, const float *xa, const float *xb, void *qn, void *kn, float *la,
                     float *be, int64_t rows, cudaStream_t stream) {
    constexpr int rows_per_cta = (kStageThreads / 32) * (32 / (DK / 4));
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t need = (rows + rows_per_cta - 1) / rows_per_cta;
    const int64_t cap = (int64_t)sms * 8;
    const unsigned grid = (unsigned)(need < cap ? need : cap);
    TimedLaunch tl_(GDN_KERNEL_INPUT, stream);
    input_stage_kernel<Tin, DK><<<grid, kStageThreads, 0, stream>>>(
        static_cast<const Tin *>(q), static_cast<const Tin *>(k), xa, xb, static_cast<Tin *>(qn),
        static_cast<Tin *>(kn), la, be, rows);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_dtype(const void *q, const void *k, const float *xa, const float *xb, void *qn, void *kn,
                         float *la, float *be, int64_t rows, int64_t dk, cudaStream_t stream) {
    switch (dk) {
        case 16: return launch_t<Tin, 16>(q, k, xa, xb, qn, kn, la, be, rows, stream);
        case 32: return launch_t<Tin, 32>(q, k, xa, xb, qn, kn, la, be, rows, stream);
        case 64: return launch_t<Tin, 64>(q, k, xa, xb, qn, kn, la, be, rows, stream);
        case 128: return launch_t<Tin, 128>(q, k, xa, xb, qn, kn, la, be, rows, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_input_stage(const void *q, const void *k, const float *x_alpha, const float *x_beta, void *qn,
                               void *kn, float *log_alpha, float *beta, int64_t rows, int64_t dk, int dtype,
                               cudaStream_t stream) {
    if (rows <= 0) return cudaSuccess;
    if (dtype == GDN_F32)
        return launch_dtype<float>(q, k, x_alpha, x_beta, qn, kn, log_alpha, beta, rows, dk, stream);
    return launch_dtype<__nv_bfloat16>(q, k, x_alpha, x_beta, qn, kn, log_alpha, beta, rows, dk, stream);
}

}  // namespace gdn
