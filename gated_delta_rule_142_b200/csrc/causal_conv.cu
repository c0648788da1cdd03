// causal_conv.cu -- the short depthwise causal convolution applied to q, k
// and v before the memory.
//
// "ATMA: Long-Context Language Modeling via Polar Attention and Gated-Delta
// Compression Memory", Sec. 3, applies depthwise causal ("Canon")
// convolutions to q, k and v.  Per channel c (C = heads x head dim channels)
// and token t of each batch row:
//     y_t[c] = sum_{j < W} w[c][j] * x_{t-j}[c],
// where x_{-1}, x_{-2}, ... come from the carried state (the last W - 1
// inputs of the previous call, oldest first) or are zero.  The state after
// the call is the last W - 1 inputs (state, then this call's tokens).
//
// One thread owns one channel of one batch row over a tile of tokens and
// slides a W - 1 window in registers, so x is read once (plus a W - 1 halo
// per tile) and y written once: an HBM-bound pass with consecutive threads
// on consecutive channels.
#include "common.cuh"
#include "gdn.h"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kConvThreads = 256;
constexpr int kConvTile = 128;  // tokens per thread

template <typename Tin>
__device__ __forceinline__ float ld1(const Tin *p) { return to_f32(*p); }

template <typename Tin, int W>
__global__ void __launch_bounds__(kConvThreads)
causal_conv_kernel(const Tin *__restrict__ x, const float *__restrict__ w, const float *__restrict__ state_in,
                   Tin *__restrict__ y, float *__restrict__ state_out, int64_t B, int64_t T, int64_t C,
                   int64_t ntiles) {
    const int64_t gid = (int64_t)blockIdx.x * kConvThreads + threadIdx.x;
    const int64_t per_row = ntiles * C;
    if (gid >= B * per_row) return;
    const int64_t b = gid / per_row, rem = gid % per_row, tile = rem / C, c = rem % C;
    const int64_t t0 = tile * kConvTile, t1 = (t0 + kConvTile < T) ? t0 + kConvTile : T;
    float wc[W];
#pragma unroll
    for (int j = 0; j < W; ++j) wc[j] = w[c * W + j];
    // window h[j] = x_{t-1-j} for the token t about to be produced
    float h[W > 1 ? W - 1 : 1];
#pragma unroll
    for (int j = 0; j < W - 1; ++j) {
        const int64_t tt = t0 - 1 - j;
        if (tt >= 0) h[j] = ld1(x + (b * T + tt) * C + c);
        else h[j] = state_in ? state_in[(b * (W - 1) + (W - 1 + tt)) * C + c] : 0.f;
    }
    for (int64_t t = t0; t < t1; ++t) {
        const float xt = ld1(x + (b * T + t) * C + c);
        float acc = wc[0] * xt;
#pragma unroll
        for (int j = 1; j < W; ++j) acc = fmaf(wc[j], h[j - 1], acc);
        y[(b * T + t) * C + c] = from_f32<Tin>(acc);
#pragma unroll
        for (int j = W - 2; j >= 1; --j) h[j] = h[j - 1];
        if (W > 1) h[0] = xt;
    }
    // the state after the call: the last W - 1 inputs, oldest first (written by the last tile)
    if (state_out && tile == ntiles - 1) {
#pragma unroll
        for (int j = 0; j < W - 1; ++j) {
            const int64_t tt = T - (W - 1) + j;  // token index of state slot j
            float val;
            if (tt >= 0) val = ld1(x + (b * T + tt) * C + c);
            else val = state_in ? state_in[(b * (W - 1) + (W - 1 + tt)) * C + c] : 0.f;
            state_out[(b * (W - 1) + j) * C + c] = val;
        }
    }
}

template <typename Tin, int W>
cudaError_t launch_w(const void *x, const float *w, const float *s_in, void *y, float *s_out, int64_t B, int64_t T,
                     int64_t C, cudaStream_t stream) {
    const int64_t ntiles = T > 0 ? (T + kConvTile - 1) / kConvTile : 1;
    const int64_t threads = B * ntiles * C;
    const int64_t blocks = (threads + kConvThreads - 1) / kConvThreads;
    TimedLaunch tl_(GDN_KERNEL_INPUT, stream);
    causal_conv_kernel<Tin, W><<<(unsigned)blocks, kConvThreads, 0, stream>>>(
        static_cast<const Tin *>(x), w, s_in, static_cast<Tin *>(y), s_out, B, T, C, ntiles);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_t(const void *x, const float *w, const float *s_in, void *y, float *s_out, int64_t B, int64_t T,
                     int64_t C, int W, cudaStream_t stream) {
    switch (W) {
        case 1: return launch_w<Tin, 1>(x, w, s_in, y, s_out, B, T, C, stream);
        case 2: return launch_w<Tin, 2>(x, w, s_in, y, s_out, B, T, C, stream);
        case 3: return launch_w<Tin, 3>(x, w, s_in, y, s_out, B, T, C, stream);
        case 4: return launch_w<Tin, 4>(x, w, s_in, y, s_out, B, T, C, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_causal_conv(const void *x, const float *w, const float *state_in, void *y, float *state_out,
                               int64_t B, int64_t T, int64_t C, int W, int dtype, cudaStream_t stream) {
    if (B * C == 0) return cudaSuccess;
    if (dtype == GDN_F32) return launch_t<float>(x, w, state_in, y, state_out, B, T, C, W, stream);
    return launch_t<__nv_bfloat16>(x, w, state_in, y, state_out, B, T, C, W, stream);
}

}  // namespace gdn
