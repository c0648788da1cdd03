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
// An HBM-bound pass: x is read once (plus a W - 1 row halo per token tile)
// and y written once, the window of the last W - 1 inputs sliding in
// registers.  The wide kernel gives each thread one 16-byte word of a row
// (8 bf16 or 4 float32 channels) and keeps 8 rows' loads in flight, so a warp
// moves 512 contiguous bytes per instruction; it takes up to three tensors
// (q, k, v) in one launch.  The narrow kernel (one channel per thread) takes
// channel counts or pointers that do not allow 16-byte words.
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

// ---------------------------------------------------------------- wide kernel
constexpr int kWideTile = 64;  // tokens per thread
constexpr int kWideUnroll = 8; // rows loaded before any is used
constexpr int kWideThreads = 128;  // ~150 registers a thread: three blocks (12 warps) per SM

struct ConvJobs {
    const void *x[3];
    const float *w[3];
    const float *s_in[3];
    void *y[3];
    int64_t C[3];
};

__device__ __forceinline__ void unpack16(const uint4 &r, float *f, const float *) {
    f[0] = __uint_as_float(r.x);
    f[1] = __uint_as_float(r.y);
    f[2] = __uint_as_float(r.z);
    f[3] = __uint_as_float(r.w);
}
__device__ __forceinline__ void unpack16(const uint4 &r, float *f, const __nv_bfloat16 *) {
    const uint32_t u[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u[i]));
        f[2 * i] = v.x;
        f[2 * i + 1] = v.y;
    }
}
__device__ __forceinline__ uint4 pack16(const float *f, const float *) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
}
__device__ __forceinline__ uint4 pack16(const float *f, const __nv_bfloat16 *) {
    uint32_t u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        u[i] = *reinterpret_cast<const uint32_t *>(&v);
    }
    return make_uint4(u[0], u[1], u[2], u[3]);
}

// Tensor blockIdx.y of the jobs; one thread per (b, token tile, 16-byte word of a row).  Same
// arithmetic and order as the narrow kernel (w0 x_t first, then the older inputs), so both give
// identical bits.  The carried state is not written here (launch_conv_state_update does).
template <typename Tin, int W>
__global__ void __launch_bounds__(kWideThreads)
causal_conv_wide_kernel(ConvJobs jobs, int64_t B, int64_t T, int64_t ntiles) {
    constexpr int V = 16 / (int)sizeof(Tin);
    // select by comparisons: a computed index into the parameter arrays would copy them to local memory
    const int job = blockIdx.y;
    auto pick = [&](auto a0, auto a1, auto a2) { return job == 0 ? a0 : (job == 1 ? a1 : a2); };
    const Tin *__restrict__ x = static_cast<const Tin *>(pick(jobs.x[0], jobs.x[1], jobs.x[2]));
    Tin *__restrict__ y = static_cast<Tin *>(pick(jobs.y[0], jobs.y[1], jobs.y[2]));
    const float *__restrict__ w = pick(jobs.w[0], jobs.w[1], jobs.w[2]);
    const float *__restrict__ s_in = pick(jobs.s_in[0], jobs.s_in[1], jobs.s_in[2]);
    const int64_t C = pick(jobs.C[0], jobs.C[1], jobs.C[2]), nvec = C / V, per_row = ntiles * nvec;
    const int64_t gid = (int64_t)blockIdx.x * kWideThreads + threadIdx.x;
    if (gid >= B * per_row) return;
    const int64_t b = gid / per_row, rem = gid % per_row, tile = rem / nvec, c0 = (rem % nvec) * V;
    const int64_t t0 = tile * kWideTile, t1 = (t0 + kWideTile < T) ? t0 + kWideTile : T;
    float wc[W][V];
#pragma unroll
    for (int i = 0; i < V; ++i)
#pragma unroll
        for (int j = 0; j < W; ++j) wc[j][i] = w[(c0 + i) * W + j];
    // window h[j] = x_{t-1-j} for the token t about to be produced
    float h[W > 1 ? W - 1 : 1][V];
#pragma unroll
    for (int j = 0; j < W - 1; ++j) {
        const int64_t tt = t0 - 1 - j;
        if (tt >= 0) {
            unpack16(*reinterpret_cast<const uint4 *>(x + (b * T + tt) * C + c0), h[j], x);
        } else {
#pragma unroll
            for (int i = 0; i < V; ++i) h[j][i] = s_in ? s_in[(b * (W - 1) + (W - 1 + tt)) * C + c0 + i] : 0.f;
        }
    }
    for (int64_t tb = t0; tb < t1; tb += kWideUnroll) {
        uint4 raw[kWideUnroll];
#pragma unroll
        for (int u = 0; u < kWideUnroll; ++u)
            if (tb + u < t1) raw[u] = *reinterpret_cast<const uint4 *>(x + (b * T + tb + u) * C + c0);
#pragma unroll
        for (int u = 0; u < kWideUnroll; ++u) {
            if (tb + u < t1) {
                float xv[V], out[V];
                unpack16(raw[u], xv, x);
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    float acc = wc[0][i] * xv[i];
#pragma unroll
                    for (int j = 1; j < W; ++j) acc = fmaf(wc[j][i], h[j - 1][i], acc);
                    out[i] = acc;
                }
                *reinterpret_cast<uint4 *>(y + (b * T + tb + u) * C + c0) = pack16(out, x);
#pragma unroll
                for (int i = 0; i < V; ++i) {
#pragma unroll
                    for (int j = W - 2; j >= 1; --j) h[j][i] = h[j - 1][i];
                    if (W > 1) h[0][i] = xv[i];
                }
            }
        }
    }
}

template <typename Tin, int W>
cudaError_t launch_wide_w(const ConvJobs &jobs, int njobs, int64_t B, int64_t T, int64_t maxC, cudaStream_t stream) {
    constexpr int V = 16 / (int)sizeof(Tin);
    const int64_t ntiles = (T + kWideTile - 1) / kWideTile;
    const int64_t blocks = (B * ntiles * (maxC / V) + kWideThreads - 1) / kWideThreads;
    if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
    TimedLaunch tl_(GDN_KERNEL_INPUT, stream);
    causal_conv_wide_kernel<Tin, W><<<dim3((unsigned)blocks, (unsigned)njobs), kWideThreads, 0, stream>>>(jobs, B, T,
                                                                                                       ntiles);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_wide(const ConvJobs &jobs, int njobs, int64_t B, int64_t T, int64_t maxC, int W,
                        cudaStream_t stream) {
    switch (W) {
        case 1: return launch_wide_w<Tin, 1>(jobs, njobs, B, T, maxC, stream);
        case 2: return launch_wide_w<Tin, 2>(jobs, njobs, B, T, maxC, stream);
        case 3: return launch_wide_w<Tin, 3>(jobs, njobs, B, T, maxC, stream);
        case 4: return launch_wide_w<Tin, 4>(jobs, njobs, B, T, maxC, stream);
        default: return cudaErrorInvalidValue;
    }
}

bool wide_ok(const void *x, const void *y, int64_t C, int dtype) {
    const int64_t V = (dtype == GDN_F32) ? 4 : 8;
    return C % V == 0 && ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) & 15) == 0;
}

// The carried state after a call of T tokens: the last W - 1 inputs, oldest first, from x or (when
// T < W - 1) the state before the call.  One thread per (b, channel); slots in increasing order, so that
// state_out == state_in works in place (slot j reads slot j + T >= j of the old state).
template <typename Tin>
__global__ void __launch_bounds__(kConvThreads)
conv_state_kernel(const Tin *__restrict__ x, const float *state_in, float *state_out, int64_t B, int64_t T,
                  int64_t C, int W) {
    const int64_t gid = (int64_t)blockIdx.x * kConvThreads + threadIdx.x;
    if (gid >= B * C) return;
    const int64_t b = gid / C, c = gid % C;
    for (int j = 0; j < W - 1; ++j) {
        const int64_t tt = T - (W - 1) + j;
        float val = 0.f;
        if (tt >= 0) val = ld1(x + (b * T + tt) * C + c);
        else if (state_in) val = state_in[(b * (W - 1) + (W - 1 + tt)) * C + c];
        state_out[(b * (W - 1) + j) * C + c] = val;
    }
}

}  // namespace

cudaError_t launch_conv_state_update(const void *x, const float *state_in, float *state_out, int64_t B, int64_t T,
                                     int64_t C, int W, int dtype, cudaStream_t stream) {
    if (B * C == 0 || W <= 1 || !state_out) return cudaSuccess;
    const int64_t blocks = (B * C + kConvThreads - 1) / kConvThreads;
    TimedLaunch tl_(GDN_KERNEL_INPUT, stream);
    if (dtype == GDN_F32)
        conv_state_kernel<float><<<(unsigned)blocks, kConvThreads, 0, stream>>>(static_cast<const float *>(x), state_in,
                                                                                state_out, B, T, C, W);
    else
        conv_state_kernel<__nv_bfloat16><<<(unsigned)blocks, kConvThreads, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(x), state_in, state_out, B, T, C, W);
    return cudaGetLastError();
}

cudaError_t launch_causal_conv(const void *x, const float *w, const float *state_in, void *y, float *state_out,
                               int64_t B, int64_t T, int64_t C, int W, int dtype, cudaStream_t stream) {
    if (B * C == 0) return cudaSuccess;
    if (T > 0 && wide_ok(x, y, C, dtype)) {
        const void *xs[3] = {x, nullptr, nullptr};
        const float *ws[3] = {w, nullptr, nullptr}, *ss[3] = {state_in, nullptr, nullptr};
        void *ys[3] = {y, nullptr, nullptr};
        const int64_t Cs[3] = {C, 0, 0};
        cudaError_t e = launch_causal_conv3(xs, ws, ss, ys, Cs, 1, B, T, W, dtype, stream);
        if (e == cudaSuccess && state_out) e = launch_conv_state_update(x, state_in, state_out, B, T, C, W, dtype, stream);
        return e;
    }
    if (dtype == GDN_F32) return launch_t<float>(x, w, state_in, y, state_out, B, T, C, W, stream);
    return launch_t<__nv_bfloat16>(x, w, state_in, y, state_out, B, T, C, W, stream);
}

cudaError_t launch_causal_conv3(const void *const x[3], const float *const w[3], const float *const state_in[3],
                                void *const y[3], const int64_t C[3], int njobs, int64_t B, int64_t T, int W, int dtype,
                                cudaStream_t stream) {
    if (njobs < 1 || njobs > 3 || W < 1 || W > 4) return cudaErrorInvalidValue;
    ConvJobs jobs = {};
    int64_t maxC = 0;
    bool wide = true;
    for (int i = 0; i < njobs; ++i) {
        jobs.x[i] = x[i];
        jobs.w[i] = w[i];
        jobs.s_in[i] = state_in[i];
        jobs.y[i] = y[i];
        jobs.C[i] = C[i];
        maxC = C[i] > maxC ? C[i] : maxC;
        wide = wide && wide_ok(x[i], y[i], C[i], dtype);
    }
    if (B * maxC == 0 || T == 0) return cudaSuccess;
    if (wide)
        return dtype == GDN_F32 ? launch_wide<float>(jobs, njobs, B, T, maxC, W, stream)
                                : launch_wide<__nv_bfloat16>(jobs, njobs, B, T, maxC, W, stream);
    for (int i = 0; i < njobs; ++i) {
        cudaError_t e = dtype == GDN_F32 ? launch_t<float>(x[i], w[i], state_in[i], y[i], nullptr, B, T, C[i], W, stream)
                                         : launch_t<__nv_bfloat16>(x[i], w[i], state_in[i], y[i], nullptr, B, T, C[i],
                                                                   W, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace gdn
