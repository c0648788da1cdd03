// decode.cu -- single-token gated-delta step, state updated in place.
//
// Operation ("ATMA: Long-Context Language Modeling via Polar Attention and
// Gated-Delta Compression Memory", Sec. 3.3, gated-delta memory equation),
// per (b, h) and per row r of the d_v x d_k state:
//     a_r = S_r . k,  b_r = S_r . q
//     u_r = beta (v_r - alpha a_r)
//     S_r <- alpha S_r + u_r k^T
//     o_r = S'_r . q = alpha b_r + u_r (k . q)
// which is the equation's S (I - beta k k^T) alpha + beta v k^T written row by
// row.  The step is bound by HBM: each state row (dk float32) is read once
// with 128-bit loads and written once; everything else is a few bytes.
//
// Mapping: a row is held by DK/4 consecutive lanes, four columns per lane
// (one float4).  A warp covers 32/(DK/4) rows per step and each thread keeps
// kUnroll rows in flight, so a CTA of 4 warps owns 4 * (32/(DK/4)) * kUnroll
// rows of one head (32 rows at dk = 128).  Grid: (B*H) x ceil(dv / rows).
//
// With the input stage fused (RAW), q and k arrive unnormalised and the gates
// as logits: the kernel scales its q, k registers by 1 / sqrt(|.|^2 + eps)
// (the squared norms come from the same lane-group sums as k . q) and maps
// log alpha = -softplus(x_alpha), beta = sigmoid(x_beta); nothing extra is
// read or written.
#include "common.cuh"
#include "gdn.h"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kDecodeThreads = 128;
constexpr int kUnroll = 8;

template <int DK>
constexpr int decode_rows_per_cta() {
    return (kDecodeThreads / 32) * (32 / (DK / 4)) * kUnroll;
}

template <typename Tin, int DK, bool RAW>
__global__ void __launch_bounds__(kDecodeThreads)
decode_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
              const float *__restrict__ log_alpha, const float *__restrict__ beta,
              float *__restrict__ S, Tin *__restrict__ out, int dv) {
    constexpr int LPR = DK / 4;          // lanes per row
    constexpr int RPW = 32 / LPR;        // rows per warp per step
    constexpr int STRIDE = (kDecodeThreads / 32) * RPW;
    const int64_t head = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int grp = lane / LPR, gl = lane % LPR;
    const int row_base = blockIdx.y * decode_rows_per_cta<DK>() + warp * RPW + grp;

    float4 kf = load4(k + head * DK + 4 * gl);
    float4 qf = load4(q + head * DK + 4 * gl);
    float alpha, bt;
    if (RAW) {
        const float rk = rsqrtf(group_sum<LPR>(dot4(kf, kf)) + kNormEps);
        const float rq = rsqrtf(group_sum<LPR>(dot4(qf, qf)) + kNormEps);
        kf = make_float4(kf.x * rk, kf.y * rk, kf.z * rk, kf.w * rk);
        qf = make_float4(qf.x * rq, qf.y * rq, qf.z * rq, qf.w * rq);
        const float xa = log_alpha[head], xb = beta[head];
        alpha = expf(-(fmaxf(xa, 0.f) + log1pf(expf(-fabsf(xa)))));
        bt = 1.f / (1.f + expf(-xb));
    } else {
        alpha = expf(log_alpha[head]);
        bt = beta[head];
    }
    const float kq = group_sum<LPR>(dot4(kf, qf));

    float *Sh = S + head * (int64_t)dv * DK;
    float4 s[kUnroll];
    float vr[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int r = row_base + u * STRIDE;
        if (r < dv) {
            s[u] = *reinterpret_cast<const float4 *>(Sh + (int64_t)r * DK + 4 * gl);
            vr[u] = to_f32(v[head * dv + r]);
        } else {
            s[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            vr[u] = 0.f;
        }
    }
    float a[kUnroll], b[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        a[u] = dot4(s[u], kf);
        b[u] = dot4(s[u], qf);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        a[u] = group_sum<LPR>(a[u]);
        b[u] = group_sum<LPR>(b[u]);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int r = row_base + u * STRIDE;
        if (r < dv) {
            const float ur = bt * (vr[u] - alpha * a[u]);
            float4 n;
            n.x = fmaf(alpha, s[u].x, ur * kf.x);
            n.y = fmaf(alpha, s[u].y, ur * kf.y);
            n.z = fmaf(alpha, s[u].z, ur * kf.z);
            n.w = fmaf(alpha, s[u].w, ur * kf.w);
            *reinterpret_cast<float4 *>(Sh + (int64_t)r * DK + 4 * gl) = n;
            if (gl == 0) out[head * dv + r] = from_f32<Tin>(fmaf(alpha, b[u], ur * kq));
        }
    }
}

// Grouped heads: the memory of key-value head hk (its k, v, gates and state) is
// updated once, then read by its `group` query heads hk * group .. hk * group +
// group - 1: o_{r,g} = S'_r . q_g, from the updated rows still in registers.
template <typename Tin, int DK>
__global__ void __launch_bounds__(kDecodeThreads)
decode_grouped_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                      const float *__restrict__ log_alpha, const float *__restrict__ beta, float *__restrict__ S,
                      Tin *__restrict__ out, int dv, int group) {
    constexpr int LPR = DK / 4;
    constexpr int RPW = 32 / LPR;
    constexpr int STRIDE = (kDecodeThreads / 32) * RPW;
    const int64_t head = blockIdx.x;  // b * Hkv + hk
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int grp = lane / LPR, gl = lane % LPR;
    const int row_base = blockIdx.y * decode_rows_per_cta<DK>() + warp * RPW + grp;

    const float4 kf = load4(k + head * DK + 4 * gl);
    const float alpha = expf(log_alpha[head]);
    const float bt = beta[head];
    float *Sh = S + head * (int64_t)dv * DK;
    float4 s[kUnroll];
    float vr[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int r = row_base + u * STRIDE;
        if (r < dv) {
            s[u] = *reinterpret_cast<const float4 *>(Sh + (int64_t)r * DK + 4 * gl);
            vr[u] = to_f32(v[head * dv + r]);
        } else {
            s[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            vr[u] = 0.f;
        }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const float a = group_sum<LPR>(dot4(s[u], kf));
        const float ur = bt * (vr[u] - alpha * a);
        s[u] = make_float4(fmaf(alpha, s[u].x, ur * kf.x), fmaf(alpha, s[u].y, ur * kf.y),
                           fmaf(alpha, s[u].z, ur * kf.z), fmaf(alpha, s[u].w, ur * kf.w));
        const int r = row_base + u * STRIDE;
        if (r < dv) *reinterpret_cast<float4 *>(Sh + (int64_t)r * DK + 4 * gl) = s[u];
    }
    for (int g = 0; g < group; ++g) {
        const int64_t qh = head * group + g;  // (b * Hkv + hk) * group + g = b * Hq + hk * group + g
        const float4 qf = load4(q + qh * DK + 4 * gl);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const float o = group_sum<LPR>(dot4(s[u], qf));
            const int r = row_base + u * STRIDE;
            if (r < dv && gl == 0) out[qh * dv + r] = from_f32<Tin>(o);
        }
    }
}

template <typename Tin, int DK>
cudaError_t launch_decode_t(const DecodeProblem &p, cudaStream_t stream) {
    const int rows = decode_rows_per_cta<DK>();
    if (p.group > 1) {
        dim3 grid((unsigned)(p.B * (p.H / p.group)), (unsigned)((p.dv + rows - 1) / rows));
        TimedLaunch tl_(GDN_KERNEL_DECODE, stream);
        decode_grouped_kernel<Tin, DK><<<grid, kDecodeThreads, 0, stream>>>(
            static_cast<const Tin *>(p.q), static_cast<const Tin *>(p.k), static_cast<const Tin *>(p.v),
            p.log_alpha, p.beta, p.S, static_cast<Tin *>(p.out), (int)p.dv, p.group);
        return cudaGetLastError();
    }
    dim3 grid((unsigned)(p.B * p.H), (unsigned)((p.dv + rows - 1) / rows));
    {
        TimedLaunch tl_(GDN_KERNEL_DECODE, stream);
        auto kern = p.raw_inputs ? decode_kernel<Tin, DK, true> : decode_kernel<Tin, DK, false>;
        kern<<<grid, kDecodeThreads, 0, stream>>>(static_cast<const Tin *>(p.q), static_cast<const Tin *>(p.k),
                                                  static_cast<const Tin *>(p.v), p.log_alpha, p.beta, p.S,
                                                  static_cast<Tin *>(p.out), (int)p.dv);
    }
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_decode_dtype(const DecodeProblem &p, cudaStream_t stream) {
    switch (p.dk) {
        case 16: return launch_decode_t<Tin, 16>(p, stream);
        case 32: return launch_decode_t<Tin, 32>(p, stream);
        case 64: return launch_decode_t<Tin, 64>(p, stream);
        case 128: return launch_decode_t<Tin, 128>(p, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_decode(const DecodeProblem &p, cudaStream_t stream) {
    if (p.B * p.H == 0) return cudaSuccess;
    if (p.dtype == 0) return launch_decode_dtype<float>(p, stream);
    return launch_decode_dtype<__nv_bfloat16>(p, stream);
}

}  // namespace gdn
