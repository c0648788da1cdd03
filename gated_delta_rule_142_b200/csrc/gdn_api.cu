// gdn_api.cu -- the C ABI declared in include/gdn.h: argument validation,
// host-buffer staging and dispatch to the kernels.  No arithmetic of the
// recurrence happens here; every step of it runs in the CUDA kernels.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>

#include "gdn.h"
#include "gdn_internal.h"

namespace {

using gdn::DecodeProblem;
using gdn::FwdProblem;

// ---------------------------------------------------------------- device info
struct DeviceInfo {
    int sm_count = 0;
    int major = 0;
};

// Immutable per-device properties, filled on first use (benign race: every
// writer stores the same values).
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
std::atomic<int> g_major[kMaxDevices];

int device_info(DeviceInfo *info) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
        cudaGetLastError();
        return GDN_ERR_DEVICE;
    }
    if (dev < kMaxDevices && g_sm_count[dev].load(std::memory_order_relaxed) > 0) {
        info->sm_count = g_sm_count[dev].load(std::memory_order_relaxed);
        info->major = g_major[dev].load(std::memory_order_relaxed);
    } else {
        int sms = 0, major = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
            cudaGetLastError();
            return GDN_ERR_DEVICE;
        }
        info->sm_count = sms;
        info->major = major;
        if (dev < kMaxDevices) {
            g_major[dev].store(major, std::memory_order_relaxed);
            g_sm_count[dev].store(sms, std::memory_order_relaxed);
        }
    }
    // The kernels are built for sm_100a only.
    if (info->major != 10) return GDN_ERR_DEVICE;
    return GDN_OK;
}

// ---------------------------------------------------------------- validation
bool supported_dim(int64_t d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool supported_chunk(int64_t c) { return c == 16 || c == 32 || c == 64; }
bool aligned16(const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool mul2ok(int64_t a, int64_t b) {
    int64_t t;
    return !__builtin_mul_overflow(a, b, &t);
}

bool mul3(int64_t a, int64_t b, int64_t c, int64_t *r) {
    int64_t t;
    return !__builtin_mul_overflow(a, b, &t) && !__builtin_mul_overflow(t, c, r);
}

struct Span {
    uintptr_t lo = 0, hi = 0;  // [lo, hi); empty when lo == hi
    Span() = default;
    Span(const void *p, int64_t bytes) {
        if (p && bytes > 0) {
            lo = reinterpret_cast<uintptr_t>(p);
            hi = lo + (uintptr_t)bytes;
        }
    }
    bool empty() const { return lo == hi; }
};
bool overlaps(const Span &a, const Span &b) { return !a.empty() && !b.empty() && a.lo < b.hi && b.lo < a.hi; }

// ---------------------------------------------------------------- scratch pool
// Scratch (the per-chunk workspace, segment transfers, host staging) comes
// from a library-private stream-ordered pool per device whose release
// threshold keeps freed memory mapped: a repeated call of the same size takes
// its scratch back from the pool instead of mapping new memory.
// gdn_scratch_release() returns what is not in use to the driver.
std::atomic<cudaMemPool_t> g_pool[kMaxDevices];

cudaMemPool_t scratch_pool(int dev) {
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    cudaMemPool_t pool = g_pool[dev].load(std::memory_order_acquire);
    if (pool) return pool;
    cudaMemPoolProps props;
    memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    uint64_t keep = UINT64_MAX;
    cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    cudaMemPool_t expected = nullptr;
    if (!g_pool[dev].compare_exchange_strong(expected, pool)) {
        cudaMemPoolDestroy(pool);  // another thread created this device's pool first
        pool = expected;
    }
    return pool;
}

// GDN_TEST_FAIL_ALLOC=1 makes every scratch allocation fail: a test hook for the allocation-failure
// paths (fallbacks and GDN_ERR_ALLOC); no kernel is involved.
bool alloc_fails_for_test() {
    const char *e = getenv("GDN_TEST_FAIL_ALLOC");
    return e && strcmp(e, "1") == 0;
}

cudaError_t scratch_alloc(void **p, size_t bytes, cudaStream_t stream) {
    if (alloc_fails_for_test()) return cudaErrorMemoryAllocation;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    cudaMemPool_t pool = scratch_pool(dev);
    if (!pool) return cudaErrorMemoryAllocation;
    return cudaMallocFromPoolAsync(p, bytes, pool, stream);
}

// ---------------------------------------------------------------- staging
bool is_device_pointer(const void *p) {
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged;
}

// Stream-ordered device copies of host buffers, released on the same stream.
struct Stager {
    cudaStream_t stream;
    void *bufs[16];
    int n = 0;
    explicit Stager(cudaStream_t s) : stream(s) {}
    ~Stager() {
        for (int i = 0; i < n; ++i) cudaFreeAsync(bufs[i], stream);
    }
    // Returns a device pointer for p (p itself when it is device memory).
    int in(const void *p, int64_t bytes, bool copy, const void **dev) {
        if (p == nullptr || bytes <= 0 || is_device_pointer(p)) {
            *dev = p;
            return GDN_OK;
        }
        void *d = nullptr;
        if (scratch_alloc(&d, (size_t)bytes, stream) != cudaSuccess) {
            cudaGetLastError();
            return GDN_ERR_ALLOC;
        }
        bufs[n++] = d;
        if (copy && cudaMemcpyAsync(d, p, (size_t)bytes, cudaMemcpyDefault, stream) != cudaSuccess) {
            cudaGetLastError();
            return GDN_ERR_LAUNCH;
        }
        *dev = d;
        return GDN_OK;
    }
    int out_back(void *host, const void *dev, int64_t bytes) {
        if (host == nullptr || host == dev || bytes <= 0) return GDN_OK;
        if (cudaMemcpyAsync(host, dev, (size_t)bytes, cudaMemcpyDefault, stream) != cudaSuccess) {
            cudaGetLastError();
            return GDN_ERR_LAUNCH;
        }
        return GDN_OK;
    }
};

// GDN_FORWARD_PATH=simt forces the float32 CUDA-core forward, =fused the
// single-kernel tensor-core forward; otherwise the two-kernel tensor-core
// forward serves every shape it supports.
enum class FwdPath { Auto, Simt, Fused };

FwdPath forced_path() {
    const char *e = getenv("GDN_FORWARD_PATH");
    if (e && strcmp(e, "simt") == 0) return FwdPath::Simt;
    if (e && strcmp(e, "fused") == 0) return FwdPath::Fused;
    return FwdPath::Auto;
}

int64_t round256(int64_t x) { return (x + 255) & ~int64_t(255); }

// For the forwards that read normalised inputs: runs the input stage over the `rows` (token,
// head) rows of p into scratch taken on `stream` and points p at the results.  *scratch
// receives the allocation (released by the caller once the forward is enqueued).
int stage_inputs(FwdProblem &p, int64_t rows, void **scratch, cudaStream_t stream) {
    const int64_t es = (p.dtype == GDN_F32) ? 4 : 2;
    const int64_t nqk = round256(rows * p.dk * es), ng = round256(rows * 4);
    if (scratch_alloc(scratch, (size_t)(2 * nqk + 2 * ng), stream) != cudaSuccess) {
        cudaGetLastError();
        *scratch = nullptr;
        return GDN_ERR_ALLOC;
    }
    uint8_t *base = static_cast<uint8_t *>(*scratch);
    float *la = reinterpret_cast<float *>(base + 2 * nqk), *be = reinterpret_cast<float *>(base + 2 * nqk + ng);
    if (gdn::launch_input_stage(p.q, p.k, p.log_alpha, p.beta, base, base + nqk, la, be, rows, p.dk, p.dtype,
                                stream) != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_LAUNCH;
    }
    p.q = base;
    p.k = base + nqk;
    p.log_alpha = la;
    p.beta = be;
    p.raw_inputs = 0;
    return GDN_OK;
}

int forward_impl(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                 const float *S0, void *out, float *S_final, int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                 int64_t chunk, void *stream_, int dtype, bool raw);
int varlen_impl(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                const int64_t *cu_seqlens, int64_t N, const float *S0, void *out, float *S_final, int64_t T_total,
                int64_t H, int64_t dk, int64_t dv, int64_t chunk, void *stream_, int dtype, bool raw);
int decode_impl(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta, float *S,
                void *out, int64_t B, int64_t H, int64_t dk, int64_t dv, void *stream_, int dtype, bool raw);

}  // namespace

extern "C" {

int gdn_scratch_release(void) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
        cudaGetLastError();
        return GDN_ERR_DEVICE;
    }
    cudaMemPool_t pool = dev < kMaxDevices ? g_pool[dev].load(std::memory_order_acquire) : nullptr;
    if (pool && cudaMemPoolTrimTo(pool, 0) != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_DEVICE;
    }
    return GDN_OK;
}

const char *gdn_status_string(int status) {
    switch (status) {
        case GDN_OK: return "ok";
        case GDN_ERR_NULL_PTR: return "a required pointer is NULL";
        case GDN_ERR_INVALID_SIZE: return "invalid size (negative, or the element count overflows int64)";
        case GDN_ERR_UNSUPPORTED: return "unsupported dk/dv (16, 32, 64, 128), chunk (16, 32, 64) or dtype";
        case GDN_ERR_MISALIGNED: return "a pointer is misaligned (16 bytes; 4 bytes for log_alpha and beta)";
        case GDN_ERR_ALLOC: return "stream-ordered device allocation failed";
        case GDN_ERR_LAUNCH: return "kernel launch or enqueued copy failed";
        case GDN_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait gave up";
        case GDN_ERR_ALIAS: return "an output buffer overlaps an input it must not overlap";
        case GDN_ERR_DEVICE: return "no usable sm_100 CUDA device is current";
        case GDN_ERR_SCRATCH_LIMIT: return "problem needs more scratch than GDN_NOALLOC_SCRATCH_BYTES (no-allocation entry point)";
        default: return "unknown gdn status";
    }
}

int gdn_version(void) { return 100; }  // 0.1.0

int gdn_forward(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                const float *S0, void *out, float *S_final, int64_t B, int64_t T, int64_t H, int64_t dk,
                int64_t dv, int64_t chunk, void *stream, int dtype) {
    return forward_impl(q, k, v, log_alpha, beta, S0, out, S_final, B, T, H, dk, dv, chunk, stream, dtype, false);
}

int gdn_forward_raw(const void *q, const void *k, const void *v, const float *x_alpha, const float *x_beta,
                    const float *S0, void *out, float *S_final, int64_t B, int64_t T, int64_t H, int64_t dk,
                    int64_t dv, int64_t chunk, void *stream, int dtype) {
    return forward_impl(q, k, v, x_alpha, x_beta, S0, out, S_final, B, T, H, dk, dv, chunk, stream, dtype, true);
}

int gdn_forward_varlen(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                       const int64_t *cu_seqlens, int64_t N, const float *S0, void *out, float *S_final,
                       int64_t T_total, int64_t H, int64_t dk, int64_t dv, int64_t chunk, void *stream, int dtype) {
    return varlen_impl(q, k, v, log_alpha, beta, cu_seqlens, N, S0, out, S_final, T_total, H, dk, dv, chunk, stream,
                       dtype, false);
}

int gdn_forward_varlen_raw(const void *q, const void *k, const void *v, const float *x_alpha, const float *x_beta,
                           const int64_t *cu_seqlens, int64_t N, const float *S0, void *out, float *S_final,
                           int64_t T_total, int64_t H, int64_t dk, int64_t dv, int64_t chunk, void *stream,
                           int dtype) {
    return varlen_impl(q, k, v, x_alpha, x_beta, cu_seqlens, N, S0, out, S_final, T_total, H, dk, dv, chunk, stream,
                       dtype, true);
}

int gdn_decode_step(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                    float *S, void *out, int64_t B, int64_t H, int64_t dk, int64_t dv, void *stream, int dtype) {
    return decode_impl(q, k, v, log_alpha, beta, S, out, B, H, dk, dv, stream, dtype, false);
}

int gdn_decode_step_raw(const void *q, const void *k, const void *v, const float *x_alpha, const float *x_beta,
                        float *S, void *out, int64_t B, int64_t H, int64_t dk, int64_t dv, void *stream, int dtype) {
    return decode_impl(q, k, v, x_alpha, x_beta, S, out, B, H, dk, dv, stream, dtype, true);
}

}  // extern "C"

namespace {

// One forward on device buffers (T > 0): the two-kernel tensor-core forward where it applies and its
// workspace can be had, else the single-kernel tensor-core forward, else the CUDA-core forward.
int run_device(FwdProblem p, const DeviceInfo &info, bool raw, cudaStream_t stream) {
    const int64_t ntok = p.B * p.T * p.H;
    int st = GDN_OK;
    cudaError_t e = cudaSuccess;
    const FwdPath path = forced_path();
    bool done = false;
    if (path == FwdPath::Auto && gdn::fwd_split_supported(p)) {
        const int nseg = gdn::fwd_tc_segments(p, info.sm_count, true);
        void *ws = nullptr;
        if (scratch_alloc(&ws, gdn::fwd_split_workspace_bytes(p, nseg), stream) == cudaSuccess) {
            p.raw_inputs = raw ? 1 : 0;  // the prep kernel runs the input stage on its own loads
            e = gdn::launch_fwd_split(p, nseg, info.sm_count, ws, stream);
            cudaFreeAsync(ws, stream);
            done = true;
        } else {
            // too little device memory for the per-chunk workspace: the single-kernel path below
            cudaGetLastError();
        }
    }
    void *staged = nullptr;
    if (!done && raw) {
        if ((st = stage_inputs(p, ntok, &staged, stream))) {
            if (staged) cudaFreeAsync(staged, stream);
            return st;
        }
    }
    if (!done && path != FwdPath::Simt && p.group == 1 && gdn::fwd_tc_supported(p)) {
        const int nseg = gdn::fwd_tc_segments(p, info.sm_count, false);
        const size_t ws_bytes = gdn::fwd_tc_workspace_bytes(p, nseg);
        void *ws = nullptr;
        if (ws_bytes > 0 && scratch_alloc(&ws, ws_bytes, stream) != cudaSuccess) {
            cudaGetLastError();
            if (staged) cudaFreeAsync(staged, stream);
            return GDN_ERR_ALLOC;
        }
        e = gdn::launch_fwd_tc(p, nseg, ws, stream);
        if (ws) cudaFreeAsync(ws, stream);
    } else if (!done) {
        e = gdn::launch_fwd_simt(p, info.sm_count, stream);
    }
    if (staged) cudaFreeAsync(staged, stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_LAUNCH;
    }
    return GDN_OK;
}

// ---------------------------------------------------------------- host pipeline
bool is_pinned_host(const void *p) {
    cudaPointerAttributes attr;
    if (!p || cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return attr.type == cudaMemoryTypeHost;
}

// B rows of `width` bytes between buffers with row pitches dpitch and spitch: one strided copy
// where the pitches allow it, else one copy per row.
bool copy_rows(void *dst, int64_t dpitch, const void *src, int64_t spitch, int64_t width, int64_t B,
               cudaMemcpyKind kind, cudaStream_t s) {
    if (B == 1) return cudaMemcpyAsync(dst, src, (size_t)width, kind, s) == cudaSuccess;
    if (dpitch < ((int64_t)1 << 31) && spitch < ((int64_t)1 << 31))
        return cudaMemcpy2DAsync(dst, (size_t)dpitch, src, (size_t)spitch, (size_t)width, (size_t)B, kind, s) ==
               cudaSuccess;
    for (int64_t b = 0; b < B; ++b)
        if (cudaMemcpyAsync(static_cast<uint8_t *>(dst) + b * dpitch, static_cast<const uint8_t *>(src) + b * spitch,
                            (size_t)width, kind, s) != cudaSuccess)
            return false;
    return true;
}

// Two library-owned copy streams per device (host-to-device, device-to-host), created on first use.
std::atomic<cudaStream_t> g_copy_streams[kMaxDevices][2];

cudaStream_t copy_stream(int dev, int which) {
    cudaStream_t s = g_copy_streams[dev][which].load(std::memory_order_acquire);
    if (s) return s;
    if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    cudaStream_t expected = nullptr;
    if (!g_copy_streams[dev][which].compare_exchange_strong(expected, s)) {
        cudaStreamDestroy(s);
        s = expected;
    }
    return s;
}

// gdn_forward with q, k, v, gates and out in pinned host memory, cut along T into pieces of whole
// chunks: while piece p runs on the caller's stream, piece p + 1 is copied in on one copy stream
// and piece p - 1 copied out on the other, so that the two directions of the host link and the
// kernels overlap.  The state passes from piece to piece on the device in float32 (the forward
// over T1 then T2 tokens from the state at T1 is the forward over T1 + T2 tokens).  Device
// buffers: two piece slots and two states.  Returns GDN_OK, or a status when nothing could be
// set up (the caller then takes the staged path), or GDN_ERR_LAUNCH after a failed enqueue.
int forward_pipelined(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                      const float *S0, void *out, float *S_final, int64_t B, int64_t T, int64_t H, int64_t dk,
                      int64_t dv, int64_t chunk, int dtype, bool raw, int npieces, const DeviceInfo &info,
                      cudaStream_t cs) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return GDN_ERR_DEVICE;
    }
    cudaStream_t hs = copy_stream(dev, 0), ds = copy_stream(dev, 1);
    if (!hs || !ds) return GDN_ERR_ALLOC;
    const int64_t es = (dtype == GDN_F32) ? 4 : 2;
    const int64_t L = ((T + npieces - 1) / npieces + chunk - 1) / chunk * chunk;  // tokens per piece
    const int64_t P = (T + L - 1) / L;
    const int64_t nstate = B * H * dv * dk * 4;
    // slot layout: q, k, v, out, log_alpha, beta of one piece, [B, L, H, .] each
    const int64_t bq = B * L * H * dk * es, bv = B * L * H * dv * es, bg = B * L * H * 4;
    const int64_t slot = 2 * bq + 2 * bv + 2 * bg;
    void *mem = nullptr;
    if (scratch_alloc(&mem, (size_t)(2 * slot + 3 * nstate), cs) != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_ALLOC;
    }
    uint8_t *base = static_cast<uint8_t *>(mem);
    float *st[2] = {reinterpret_cast<float *>(base + 2 * slot), reinterpret_cast<float *>(base + 2 * slot + nstate)};
    float *s0dev = reinterpret_cast<float *>(base + 2 * slot + 2 * nstate);
    cudaEvent_t ev[7] = {};
    bool ok = true;
    for (cudaEvent_t &x : ev) ok = ok && cudaEventCreateWithFlags(&x, cudaEventDisableTiming) == cudaSuccess;
    // ev[0]: the allocation (and S0) on the caller's stream; ev[1 + s]: inputs of slot s landed;
    // ev[3 + s]: slot s computed; ev[5 + s]: outputs of slot s copied out
    const float *s_in = nullptr;
    if (ok && S0) {
        ok = cudaMemcpyAsync(s0dev, S0, (size_t)nstate, cudaMemcpyDefault, cs) == cudaSuccess;
        s_in = s0dev;
    }
    ok = ok && cudaEventRecord(ev[0], cs) == cudaSuccess && cudaStreamWaitEvent(hs, ev[0], 0) == cudaSuccess &&
         cudaStreamWaitEvent(ds, ev[0], 0) == cudaSuccess;
    int st_status = GDN_OK;
    for (int64_t pc = 0; pc < P && ok; ++pc) {
        const int sl = (int)(pc & 1);
        const int64_t t0 = pc * L, len = (T - t0 < L) ? (T - t0) : L;
        uint8_t *sb = base + sl * slot;
        uint8_t *dq = sb, *dkk = sb + bq, *dvv = sb + 2 * bq, *dout = sb + 2 * bq + bv;
        float *dla = reinterpret_cast<float *>(sb + 2 * bq + 2 * bv), *dbe = reinterpret_cast<float *>(sb + 2 * bq + 2 * bv + bg);
        // inputs of this piece: one strided copy per tensor (B rows of len * H * d elements)
        if (pc >= 2) ok = ok && cudaStreamWaitEvent(hs, ev[3 + sl], 0) == cudaSuccess;
        auto in2d = [&](void *dst, const void *src, int64_t tok_bytes) {
            return copy_rows(dst, len * tok_bytes, static_cast<const uint8_t *>(src) + t0 * tok_bytes, T * tok_bytes,
                             len * tok_bytes, B, cudaMemcpyHostToDevice, hs);
        };
        ok = ok && in2d(dq, q, H * dk * es) && in2d(dkk, k, H * dk * es) && in2d(dvv, v, H * dv * es) &&
             in2d(dla, log_alpha, H * 4) && in2d(dbe, beta, H * 4);
        ok = ok && cudaEventRecord(ev[1 + sl], hs) == cudaSuccess;
        // the piece's forward on the caller's stream
        ok = ok && cudaStreamWaitEvent(cs, ev[1 + sl], 0) == cudaSuccess;
        if (pc >= 2) ok = ok && cudaStreamWaitEvent(cs, ev[5 + sl], 0) == cudaSuccess;
        if (!ok) break;
        FwdProblem p;
        p.q = dq; p.k = dkk; p.v = dvv; p.log_alpha = dla; p.beta = dbe;
        p.S0 = s_in;
        p.out = dout;
        p.S_final = st[sl];
        p.B = B; p.T = len; p.H = H; p.dk = dk; p.dv = dv; p.chunk = chunk; p.dtype = dtype;
        if ((st_status = run_device(p, info, raw, cs))) {
            ok = false;
            break;
        }
        s_in = st[sl];
        ok = ok && cudaEventRecord(ev[3 + sl], cs) == cudaSuccess;
        // outputs of this piece
        ok = ok && cudaStreamWaitEvent(ds, ev[3 + sl], 0) == cudaSuccess &&
             copy_rows(static_cast<uint8_t *>(out) + t0 * H * dv * es, T * H * dv * es, dout, len * H * dv * es,
                       len * H * dv * es, B, cudaMemcpyDeviceToHost, ds) &&
             cudaEventRecord(ev[5 + sl], ds) == cudaSuccess;
    }
    // the caller's stream orders after everything enqueued on the copy streams (also after a
    // failure part-way); then the final state and the frees
    ok = cudaEventRecord(ev[1], hs) == cudaSuccess && cudaEventRecord(ev[5], ds) == cudaSuccess &&
         cudaStreamWaitEvent(cs, ev[1], 0) == cudaSuccess && cudaStreamWaitEvent(cs, ev[5], 0) == cudaSuccess && ok;
    if (ok && S_final && s_in) ok = cudaMemcpyAsync(S_final, s_in, (size_t)nstate, cudaMemcpyDefault, cs) == cudaSuccess;
    for (cudaEvent_t &x : ev)
        if (x) cudaEventDestroy(x);
    cudaFreeAsync(mem, cs);
    if (!ok) {
        cudaGetLastError();
        return st_status ? st_status : GDN_ERR_LAUNCH;
    }
    return GDN_OK;
}

int forward_impl(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                 const float *S0, void *out, float *S_final, int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                 int64_t chunk, void *stream_, int dtype, bool raw) {
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if (B < 0 || T < 0 || H < 0 || dk < 0 || dv < 0 || chunk < 0) return GDN_ERR_INVALID_SIZE;
    if (!supported_dim(dk) || !supported_dim(dv) || !supported_chunk(chunk)) return GDN_ERR_UNSUPPORTED;
    const int64_t es = (dtype == GDN_F32) ? 4 : 2;
    int64_t ntok, nqk, nv, nstate;
    if (!mul3(B, T, H, &ntok) || !mul3(ntok, dk, es, &nqk) || !mul3(ntok, dv, es, &nv) ||
        !mul2ok(B, H) || !mul3(B * H, dv, dk * 4, &nstate) || ntok > (INT64_MAX / 8))
        return GDN_ERR_INVALID_SIZE;
    if (B * H == 0) return GDN_OK;
    if (ntok > 0 && (!q || !k || !v || !log_alpha || !beta || !out)) return GDN_ERR_NULL_PTR;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned4(log_alpha) || !aligned4(beta) ||
        !aligned16(S0) || !aligned16(out) || !aligned16(S_final))
        return GDN_ERR_MISALIGNED;
    const Span sq(q, nqk), sk(k, nqk), sv(v, nv), sla(log_alpha, ntok * 4), sbe(beta, ntok * 4);
    const Span s0(S0, nstate), sf(S_final, nstate), so(out, nv);
    const Span inputs[] = {sq, sk, sv, sla, sbe, s0, sf};
    for (const Span &x : inputs)
        if (overlaps(so, x)) return GDN_ERR_ALIAS;
    if (overlaps(sf, s0) && !(sf.lo == s0.lo)) return GDN_ERR_ALIAS;
    for (const Span &x : {sq, sk, sv, sla, sbe})
        if (overlaps(sf, x)) return GDN_ERR_ALIAS;

    DeviceInfo info;
    if (int st = device_info(&info)) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);

    // Large problems whose token-major tensors are all in pinned host memory: pipelined over
    // pieces of T (copies in both directions overlap the kernels), unless GDN_HOST_PIPELINE=0.
    const int64_t host_bytes = 2 * nqk + 2 * nv + 2 * ntok * 4;
    const char *pipe_env = getenv("GDN_HOST_PIPELINE");
    if (T >= 2 * chunk && host_bytes >= ((int64_t)64 << 20) && !(pipe_env && strcmp(pipe_env, "0") == 0) &&
        is_pinned_host(q) && is_pinned_host(k) && is_pinned_host(v) && is_pinned_host(log_alpha) &&
        is_pinned_host(beta) && is_pinned_host(out)) {
        int64_t pieces = host_bytes / ((int64_t)64 << 20);
        pieces = pieces < 2 ? 2 : (pieces > 16 ? 16 : pieces);
        if (pieces > T / chunk) pieces = T / chunk;
        const int st = forward_pipelined(q, k, v, log_alpha, beta, S0, out, S_final, B, T, H, dk, dv, chunk,
                                         dtype, raw, (int)pieces, info, stream);
        if (st != GDN_ERR_ALLOC && st != GDN_ERR_DEVICE) return st;
        // no room for the pipeline's buffers: the staged path below
    }

    Stager stg(stream);
    FwdProblem p;
    int st = GDN_OK;
    const void *dS0 = nullptr;
    if ((st = stg.in(q, nqk, true, &p.q)) || (st = stg.in(k, nqk, true, &p.k)) || (st = stg.in(v, nv, true, &p.v)) ||
        (st = stg.in(log_alpha, ntok * 4, true, reinterpret_cast<const void **>(&p.log_alpha))) ||
        (st = stg.in(beta, ntok * 4, true, reinterpret_cast<const void **>(&p.beta))) ||
        (st = stg.in(S0, nstate, true, &dS0)))
        return st;
    p.S0 = static_cast<const float *>(dS0);
    const void *dout = nullptr, *dSf = nullptr;
    if ((st = stg.in(out, nv, false, &dout))) return st;
    if (S_final && S_final == S0) {
        dSf = dS0;
    } else if ((st = stg.in(S_final, nstate, false, &dSf))) {
        return st;
    }
    p.out = const_cast<void *>(dout);
    p.S_final = static_cast<float *>(const_cast<void *>(dSf));
    p.B = B; p.T = T; p.H = H; p.dk = dk; p.dv = dv; p.chunk = chunk; p.dtype = dtype;

    cudaError_t e = cudaSuccess;
    if (T == 0) {
        if (p.S_final && p.S_final != p.S0) {
            e = p.S0 ? cudaMemcpyAsync(p.S_final, p.S0, (size_t)nstate, cudaMemcpyDeviceToDevice, stream)
                     : cudaMemsetAsync(p.S_final, 0, (size_t)nstate, stream);
        }
    } else if ((st = run_device(p, info, raw, stream))) {
        return st;
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_LAUNCH;
    }
    if ((st = stg.out_back(out, p.out, nv))) return st;
    if ((st = stg.out_back(S_final, p.S_final, nstate))) return st;
    return GDN_OK;
}

int varlen_impl(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                const int64_t *cu_seqlens, int64_t N, const float *S0, void *out, float *S_final, int64_t T_total,
                int64_t H, int64_t dk, int64_t dv, int64_t chunk, void *stream_, int dtype, bool raw) {
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if (N < 0 || T_total < 0 || H < 0 || dk < 0 || dv < 0 || chunk < 0) return GDN_ERR_INVALID_SIZE;
    if (!supported_dim(dk) || !supported_dim(dv) || !supported_chunk(chunk)) return GDN_ERR_UNSUPPORTED;
    if (N > 0 && !cu_seqlens) return GDN_ERR_INVALID_SIZE;
    if (N > 0) {
        if (cu_seqlens[0] != 0 || cu_seqlens[N] != T_total) return GDN_ERR_INVALID_SIZE;
        for (int64_t i = 0; i < N; ++i)
            if (cu_seqlens[i + 1] < cu_seqlens[i]) return GDN_ERR_INVALID_SIZE;
    } else if (T_total != 0) {
        return GDN_ERR_INVALID_SIZE;
    }
    const int64_t es = (dtype == GDN_F32) ? 4 : 2;
    if (N > (int64_t)INT32_MAX / (H > 0 ? H : 1) || T_total > (int64_t)INT32_MAX / 2) return GDN_ERR_INVALID_SIZE;
    int64_t ntok, nqk, nv, nstate;
    if (!mul3(1, T_total, H, &ntok) || !mul3(ntok, dk, es, &nqk) || !mul3(ntok, dv, es, &nv) ||
        !mul2ok(N, H) || !mul3(N * H, dv, dk * 4, &nstate) || ntok > (INT64_MAX / 8))
        return GDN_ERR_INVALID_SIZE;
    if (N * H == 0) return GDN_OK;
    if (ntok > 0 && (!q || !k || !v || !log_alpha || !beta || !out)) return GDN_ERR_NULL_PTR;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned4(log_alpha) || !aligned4(beta) ||
        !aligned16(S0) || !aligned16(out) || !aligned16(S_final))
        return GDN_ERR_MISALIGNED;
    const Span sq(q, nqk), sk(k, nqk), sv(v, nv), sla(log_alpha, ntok * 4), sbe(beta, ntok * 4);
    const Span s0(S0, nstate), sf(S_final, nstate), so(out, nv);
    const Span inputs[] = {sq, sk, sv, sla, sbe, s0, sf};
    for (const Span &x : inputs)
        if (overlaps(so, x)) return GDN_ERR_ALIAS;
    if (overlaps(sf, s0) && !(sf.lo == s0.lo)) return GDN_ERR_ALIAS;
    for (const Span &x : {sq, sk, sv, sla, sbe})
        if (overlaps(sf, x)) return GDN_ERR_ALIAS;

    DeviceInfo info;
    if (int st = device_info(&info)) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    Stager stg(stream);
    FwdProblem p;
    int st = GDN_OK;
    const void *dS0 = nullptr;
    if ((st = stg.in(q, nqk, true, &p.q)) || (st = stg.in(k, nqk, true, &p.k)) || (st = stg.in(v, nv, true, &p.v)) ||
        (st = stg.in(log_alpha, ntok * 4, true, reinterpret_cast<const void **>(&p.log_alpha))) ||
        (st = stg.in(beta, ntok * 4, true, reinterpret_cast<const void **>(&p.beta))) ||
        (st = stg.in(S0, nstate, true, &dS0)))
        return st;
    p.S0 = static_cast<const float *>(dS0);
    const void *dout = nullptr, *dSf = nullptr;
    if ((st = stg.in(out, nv, false, &dout))) return st;
    if (S_final && S_final == S0) {
        dSf = dS0;
    } else if ((st = stg.in(S_final, nstate, false, &dSf))) {
        return st;
    }
    p.out = const_cast<void *>(dout);
    p.S_final = static_cast<float *>(const_cast<void *>(dSf));
    p.B = 1; p.T = T_total; p.H = H; p.dk = dk; p.dv = dv; p.chunk = chunk; p.dtype = dtype;

    cudaError_t e = cudaSuccess;
    const FwdPath path = forced_path();
    bool done = false;
    if (T_total == 0) {  // every sequence is empty: S_final receives S0 (or zeros)
        if (p.S_final && p.S_final != p.S0)
            e = p.S0 ? cudaMemcpyAsync(p.S_final, p.S0, (size_t)nstate, cudaMemcpyDeviceToDevice, stream)
                     : cudaMemsetAsync(p.S_final, 0, (size_t)nstate, stream);
        done = true;
    }
    gdn::PackedPlan plan;
    if (!done && path == FwdPath::Auto && gdn::fwd_tc_supported(p) &&
        gdn::plan_packed(cu_seqlens, N, H, info.sm_count, &plan)) {
        // every sequence at once on the two-kernel tensor-core forward
        void *ws = nullptr;
        if (scratch_alloc(&ws, gdn::packed_workspace_bytes(plan), stream) == cudaSuccess) {
            p.raw_inputs = raw ? 1 : 0;  // the prep kernel runs the input stage on its own loads
            e = gdn::launch_fwd_split_packed(p, plan, ws, stream);
            cudaFreeAsync(ws, stream);
            done = true;
        } else {
            cudaGetLastError();
        }
    }
    // otherwise one fixed-length launch per sequence: the single-kernel tensor-core forward (no
    // segments, so no scratch) or the CUDA-core forward
    void *staged = nullptr;
    if (!done && raw) {
        if ((st = stage_inputs(p, ntok, &staged, stream))) {
            if (staged) cudaFreeAsync(staged, stream);
            return st;
        }
    }
    const int64_t state = H * dv * dk;
    for (int64_t i = 0; i < N && !done && e == cudaSuccess; ++i) {
        const int64_t t0 = cu_seqlens[i], len = cu_seqlens[i + 1] - t0;
        FwdProblem pi = p;
        pi.q = static_cast<const uint8_t *>(p.q) + t0 * H * dk * es;
        pi.k = static_cast<const uint8_t *>(p.k) + t0 * H * dk * es;
        pi.v = static_cast<const uint8_t *>(p.v) + t0 * H * dv * es;
        pi.log_alpha = p.log_alpha + t0 * H;
        pi.beta = p.beta + t0 * H;
        pi.out = static_cast<uint8_t *>(p.out) + t0 * H * dv * es;
        pi.S0 = p.S0 ? p.S0 + i * state : nullptr;
        pi.S_final = p.S_final ? p.S_final + i * state : nullptr;
        pi.T = len;
        if (len == 0) {
            if (pi.S_final && pi.S_final != pi.S0)
                e = pi.S0 ? cudaMemcpyAsync(pi.S_final, pi.S0, (size_t)(state * 4), cudaMemcpyDeviceToDevice, stream)
                          : cudaMemsetAsync(pi.S_final, 0, (size_t)(state * 4), stream);
        } else if (path != FwdPath::Simt && gdn::fwd_tc_supported(pi)) {
            e = gdn::launch_fwd_tc(pi, 1, nullptr, stream);
        } else {
            e = gdn::launch_fwd_simt(pi, info.sm_count, stream);
        }
    }
    if (staged) cudaFreeAsync(staged, stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_LAUNCH;
    }
    if ((st = stg.out_back(out, p.out, nv))) return st;
    if ((st = stg.out_back(S_final, p.S_final, nstate))) return st;
    return GDN_OK;
}

}  // namespace

extern "C" {

int gdn_forward_plan(int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv, int64_t chunk, int dtype,
                     int64_t *scratch_bytes, int *launches) {
    if (scratch_bytes) *scratch_bytes = 0;
    if (launches) *launches = 0;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if (B < 0 || T < 0 || H < 0 || dk < 0 || dv < 0 || chunk < 0) return GDN_ERR_INVALID_SIZE;
    if (!supported_dim(dk) || !supported_dim(dv) || !supported_chunk(chunk)) return GDN_ERR_UNSUPPORTED;
    int64_t ntok;
    if (!mul3(B, T, H, &ntok)) return GDN_ERR_INVALID_SIZE;
    if (B * H == 0 || T == 0) return GDN_OK;
    DeviceInfo info;
    if (int st = device_info(&info)) return st;
    FwdProblem p;
    p.q = p.k = p.v = nullptr;
    p.log_alpha = p.beta = p.S0 = nullptr;
    p.out = nullptr;
    p.S_final = nullptr;
    p.B = B; p.T = T; p.H = H; p.dk = dk; p.dv = dv; p.chunk = chunk; p.dtype = dtype;
    const FwdPath path = forced_path();
    if (path == FwdPath::Auto && gdn::fwd_split_supported(p)) {
        const int nseg = gdn::fwd_tc_segments(p, info.sm_count, true);
        if (scratch_bytes) *scratch_bytes = (int64_t)gdn::fwd_split_workspace_bytes(p, nseg);
        if (launches) *launches = nseg > 1 ? 4 : 2;
    } else if (path != FwdPath::Simt && gdn::fwd_tc_supported(p)) {
        const int nseg = gdn::fwd_tc_segments(p, info.sm_count, false);
        if (scratch_bytes) *scratch_bytes = (int64_t)gdn::fwd_tc_workspace_bytes(p, nseg);
        if (launches) *launches = nseg > 1 ? 3 : 1;
    } else if (launches) {
        *launches = 1;
    }
    return GDN_OK;
}

}  // extern "C"

namespace {

int decode_impl(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta, float *S,
                void *out, int64_t B, int64_t H, int64_t dk, int64_t dv, void *stream_, int dtype, bool raw) {
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if (B < 0 || H < 0 || dk < 0 || dv < 0) return GDN_ERR_INVALID_SIZE;
    if (!supported_dim(dk) || !supported_dim(dv)) return GDN_ERR_UNSUPPORTED;
    const int64_t es = (dtype == GDN_F32) ? 4 : 2;
    int64_t nh, nqk, nv, nstate;
    if (__builtin_mul_overflow(B, H, &nh) || !mul3(nh, dk, es, &nqk) || !mul3(nh, dv, es, &nv) ||
        !mul3(nh, dv, dk * 4, &nstate) || nh > (int64_t)INT32_MAX)
        return GDN_ERR_INVALID_SIZE;
    if (nh == 0) return GDN_OK;
    if (!q || !k || !v || !log_alpha || !beta || !S || !out) return GDN_ERR_NULL_PTR;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned4(log_alpha) || !aligned4(beta) ||
        !aligned16(S) || !aligned16(out))
        return GDN_ERR_MISALIGNED;
    const Span sq(q, nqk), sk(k, nqk), sv(v, nv), sla(log_alpha, nh * 4), sbe(beta, nh * 4);
    const Span ss(S, nstate), so(out, nv);
    for (const Span &x : {sq, sk, sv, sla, sbe, ss})
        if (overlaps(so, x)) return GDN_ERR_ALIAS;
    for (const Span &x : {sq, sk, sv, sla, sbe})
        if (overlaps(ss, x)) return GDN_ERR_ALIAS;

    DeviceInfo info;
    if (int st = device_info(&info)) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    Stager stg(stream);
    DecodeProblem p;
    int st = GDN_OK;
    const void *dS = nullptr, *dout = nullptr;
    if ((st = stg.in(q, nqk, true, &p.q)) || (st = stg.in(k, nqk, true, &p.k)) || (st = stg.in(v, nv, true, &p.v)) ||
        (st = stg.in(log_alpha, nh * 4, true, reinterpret_cast<const void **>(&p.log_alpha))) ||
        (st = stg.in(beta, nh * 4, true, reinterpret_cast<const void **>(&p.beta))) ||
        (st = stg.in(S, nstate, true, &dS)) || (st = stg.in(out, nv, false, &dout)))
        return st;
    p.S = static_cast<float *>(const_cast<void *>(dS));
    p.out = const_cast<void *>(dout);
    p.B = B; p.H = H; p.dk = dk; p.dv = dv; p.dtype = dtype;
    p.raw_inputs = raw ? 1 : 0;
    if (gdn::launch_decode(p, stream) != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_LAUNCH;
    }
    if ((st = stg.out_back(out, p.out, nv))) return st;
    if ((st = stg.out_back(S, p.S, nstate))) return st;
    return GDN_OK;
}

}  // namespace

extern "C" int gdn_backward(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                            const float *S0, const void *grad_out, const float *grad_S_final, void *grad_q,
                            void *grad_k, void *grad_v, float *grad_log_alpha, float *grad_beta, float *grad_S0,
                            int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv, int64_t chunk, void *stream_,
                            int dtype) {
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if (B < 0 || T < 0 || H < 0 || dk < 0 || dv < 0 || chunk < 0) return GDN_ERR_INVALID_SIZE;
    if (!supported_dim(dk) || !supported_dim(dv) || !supported_chunk(chunk)) return GDN_ERR_UNSUPPORTED;
    const int64_t es = (dtype == GDN_F32) ? 4 : 2;
    int64_t ntok, nqk, nv, nstate;
    if (!mul3(B, T, H, &ntok) || !mul3(ntok, dk, es, &nqk) || !mul3(ntok, dv, es, &nv) ||
        !mul2ok(B, H) || !mul3(B * H, dv, dk * 4, &nstate) || ntok > (INT64_MAX / 8))
        return GDN_ERR_INVALID_SIZE;
    if (B * H == 0) return GDN_OK;
    if (ntok > 0 && (!q || !k || !v || !log_alpha || !beta || !grad_out || !grad_q || !grad_k || !grad_v ||
                     !grad_log_alpha || !grad_beta))
        return GDN_ERR_NULL_PTR;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned4(log_alpha) || !aligned4(beta) ||
        !aligned16(S0) || !aligned16(grad_out) || !aligned16(grad_S_final) || !aligned16(grad_q) ||
        !aligned16(grad_k) || !aligned16(grad_v) || !aligned4(grad_log_alpha) || !aligned4(grad_beta) ||
        !aligned16(grad_S0))
        return GDN_ERR_MISALIGNED;
    const Span inputs[] = {Span(q, nqk), Span(k, nqk), Span(v, nv), Span(log_alpha, ntok * 4), Span(beta, ntok * 4),
                           Span(S0, nstate), Span(grad_out, nv), Span(grad_S_final, nstate)};
    const Span outputs[] = {Span(grad_q, nqk), Span(grad_k, nqk), Span(grad_v, nv), Span(grad_log_alpha, ntok * 4),
                            Span(grad_beta, ntok * 4), Span(grad_S0, nstate)};
    for (const Span &o : outputs) {
        for (const Span &x : inputs)
            if (overlaps(o, x)) return GDN_ERR_ALIAS;
        for (const Span &x : outputs)
            if (&x != &o && overlaps(o, x)) return GDN_ERR_ALIAS;
    }

    DeviceInfo info;
    if (int st = device_info(&info)) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    Stager stg(stream);
    gdn::BwdProblem p;
    int st = GDN_OK;
    const void *dS0in = nullptr, *dgo = nullptr, *dgSf = nullptr;
    if ((st = stg.in(q, nqk, true, &p.f.q)) || (st = stg.in(k, nqk, true, &p.f.k)) ||
        (st = stg.in(v, nv, true, &p.f.v)) ||
        (st = stg.in(log_alpha, ntok * 4, true, reinterpret_cast<const void **>(&p.f.log_alpha))) ||
        (st = stg.in(beta, ntok * 4, true, reinterpret_cast<const void **>(&p.f.beta))) ||
        (st = stg.in(S0, nstate, true, &dS0in)) || (st = stg.in(grad_out, nv, true, &dgo)) ||
        (st = stg.in(grad_S_final, nstate, true, &dgSf)))
        return st;
    p.f.S0 = static_cast<const float *>(dS0in);
    p.d_out = dgo;
    p.dS_final = static_cast<const float *>(dgSf);
    const void *oq = nullptr, *ok = nullptr, *ov = nullptr, *ola = nullptr, *obe = nullptr, *oS0 = nullptr;
    if ((st = stg.in(grad_q, nqk, false, &oq)) || (st = stg.in(grad_k, nqk, false, &ok)) ||
        (st = stg.in(grad_v, nv, false, &ov)) || (st = stg.in(grad_log_alpha, ntok * 4, false, &ola)) ||
        (st = stg.in(grad_beta, ntok * 4, false, &obe)) || (st = stg.in(grad_S0, nstate, false, &oS0)))
        return st;
    p.dq = const_cast<void *>(oq);
    p.dk = const_cast<void *>(ok);
    p.dv = const_cast<void *>(ov);
    p.dlog_alpha = static_cast<float *>(const_cast<void *>(ola));
    p.dbeta = static_cast<float *>(const_cast<void *>(obe));
    p.dS0 = static_cast<float *>(const_cast<void *>(oS0));
    p.f.out = nullptr;
    p.f.S_final = nullptr;
    p.f.B = B; p.f.T = T; p.f.H = H; p.f.dk = dk; p.f.dv = dv; p.f.chunk = chunk; p.f.dtype = dtype;

    cudaError_t e = cudaSuccess;
    if (T == 0) {  // nothing flows but dS_final -> dS0
        if (p.dS0)
            e = p.dS_final ? cudaMemcpyAsync(p.dS0, p.dS_final, (size_t)nstate, cudaMemcpyDeviceToDevice, stream)
                           : cudaMemsetAsync(p.dS0, 0, (size_t)nstate, stream);
    } else {
        void *ws = nullptr;
        bool done = false;
        if (gdn::bwd_tc_supported(p)) {
            // the tensor-core reverse mode; without room for its workspace, the CUDA-core one below
            if (scratch_alloc(&ws, gdn::bwd_tc_workspace_bytes(p, info.sm_count), stream) == cudaSuccess) {
                e = gdn::launch_bwd_tc(p, info.sm_count, ws, stream);
                cudaFreeAsync(ws, stream);
                done = true;
            } else {
                cudaGetLastError();
            }
        }
        if (!done) {
            if (scratch_alloc(&ws, gdn::bwd_simt_workspace_bytes(p, info.sm_count), stream) != cudaSuccess) {
                cudaGetLastError();
                return GDN_ERR_ALLOC;
            }
            e = gdn::launch_bwd_simt(p, info.sm_count, ws, stream);
            cudaFreeAsync(ws, stream);
        }
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_LAUNCH;
    }
    if ((st = stg.out_back(grad_q, p.dq, nqk)) || (st = stg.out_back(grad_k, p.dk, nqk)) ||
        (st = stg.out_back(grad_v, p.dv, nv)) || (st = stg.out_back(grad_log_alpha, p.dlog_alpha, ntok * 4)) ||
        (st = stg.out_back(grad_beta, p.dbeta, ntok * 4)) || (st = stg.out_back(grad_S0, p.dS0, nstate)))
        return st;
    return GDN_OK;
}

extern "C" int gdn_forward_grouped(const void *q, const void *k, const void *v, const float *log_alpha,
                                   const float *beta, const float *S0, void *out, float *S_final, int64_t B,
                                   int64_t T, int64_t Hq, int64_t Hkv, int64_t dk, int64_t dv, int64_t chunk,
                                   void *stream_, int dtype) {
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if (B < 0 || T < 0 || Hq < 0 || Hkv < 0 || dk < 0 || dv < 0 || chunk < 0) return GDN_ERR_INVALID_SIZE;
    if (!supported_dim(dk) || !supported_dim(dv) || !supported_chunk(chunk)) return GDN_ERR_UNSUPPORTED;
    if ((Hq > 0) != (Hkv > 0) || (Hkv > 0 && (Hq % Hkv != 0 || Hq / Hkv > INT32_MAX))) return GDN_ERR_INVALID_SIZE;
    const int64_t es = (dtype == GDN_F32) ? 4 : 2;
    int64_t nq, nkv, nqk, nk, nv, nout, nstate, nxstate;
    if (!mul3(B, T, Hq, &nq) || !mul3(B, T, Hkv, &nkv) || !mul3(nq, dk, es, &nqk) || !mul3(nkv, dk, es, &nk) ||
        !mul3(nkv, dv, es, &nv) || !mul3(nq, dv, es, &nout) || !mul3(B * Hkv, dv, dk * 4, &nstate) ||
        !mul2ok(B, Hq) || !mul3(B * Hq, dv, dk * 4, &nxstate) || nq > (INT64_MAX / 8))
        return GDN_ERR_INVALID_SIZE;
    if (B * Hq == 0) return GDN_OK;
    if (nq > 0 && (!q || !k || !v || !log_alpha || !beta || !out)) return GDN_ERR_NULL_PTR;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned4(log_alpha) || !aligned4(beta) ||
        !aligned16(S0) || !aligned16(out) || !aligned16(S_final))
        return GDN_ERR_MISALIGNED;
    const Span sq(q, nqk), sk(k, nk), sv(v, nv), sla(log_alpha, nkv * 4), sbe(beta, nkv * 4);
    const Span s0(S0, nstate), sf(S_final, nstate), so(out, nout);
    for (const Span &x : {sq, sk, sv, sla, sbe, s0, sf})
        if (overlaps(so, x)) return GDN_ERR_ALIAS;
    if (overlaps(sf, s0) && !(sf.lo == s0.lo)) return GDN_ERR_ALIAS;
    for (const Span &x : {sq, sk, sv, sla, sbe})
        if (overlaps(sf, x)) return GDN_ERR_ALIAS;
    const int group = (int)(Hq / Hkv);
    if (group == 1)
        return gdn_forward(q, k, v, log_alpha, beta, S0, out, S_final, B, T, Hq, dk, dv, chunk, stream_, dtype);

    DeviceInfo info;
    if (int st = device_info(&info)) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    Stager stg(stream);
    FwdProblem p;
    int st = GDN_OK;
    const void *dS0 = nullptr, *dout = nullptr, *dSf = nullptr;
    if ((st = stg.in(q, nqk, true, &p.q)) || (st = stg.in(k, nk, true, &p.k)) || (st = stg.in(v, nv, true, &p.v)) ||
        (st = stg.in(log_alpha, nkv * 4, true, reinterpret_cast<const void **>(&p.log_alpha))) ||
        (st = stg.in(beta, nkv * 4, true, reinterpret_cast<const void **>(&p.beta))) ||
        (st = stg.in(S0, nstate, true, &dS0)) || (st = stg.in(out, nout, false, &dout)))
        return st;
    if (S_final && S_final == S0) {
        dSf = dS0;
    } else if ((st = stg.in(S_final, nstate, false, &dSf))) {
        return st;
    }
    p.out = const_cast<void *>(dout);
    p.B = B; p.T = T; p.H = Hq; p.dk = dk; p.dv = dv; p.chunk = chunk; p.dtype = dtype;
    p.group = group;
    if (T > 0 && forced_path() == FwdPath::Auto && gdn::fwd_split_supported(p)) {
        // one memory per key-value head: the two-kernel forward in lead mode (prep over every query
        // head, transfers, prefix and chain over the key-value heads, checkpoints and U^T kept), then
        // the other query heads' outputs from them
        FwdProblem pl = p;
        pl.lead = group;
        pl.S0 = static_cast<const float *>(dS0);
        pl.S_final = static_cast<float *>(const_cast<void *>(dSf));
        pl.ckpt_bf16 = 1;
        FwdProblem plan = pl;  // the planner counts memories
        plan.H = Hkv;
        plan.group = 1;
        plan.lead = 1;
        const int nseg = gdn::fwd_tc_segments(plan, info.sm_count, true);
        const int64_t nch = (T + 63) / 64, mems = B * Hkv * nch;
        auto round256 = [](size_t x) { return (x + 255) & ~(size_t)255; };
        const size_t wsb = round256(gdn::fwd_split_workspace_bytes(pl, nseg)), ckb = (size_t)mems * 128 * 128 * 2,
                     ub = (size_t)mems * 128 * 64 * 2;
        void *ws = nullptr;
        if (scratch_alloc(&ws, wsb + ckb + ub, stream) == cudaSuccess) {
            uint8_t *w8 = static_cast<uint8_t *>(ws);
            pl.ckpt = reinterpret_cast<float *>(w8 + wsb);
            pl.u_out = w8 + wsb + ckb;
            cudaError_t e = gdn::launch_fwd_split(pl, nseg, info.sm_count, ws, stream);
            if (e == cudaSuccess) {
                void *pt = nullptr, *tbt = nullptr;
                gdn::fwd_split_ws_tiles(ws, B * Hq * nch, &pt, &tbt);
                e = gdn::launch_grouped_outputs(pl, pl.ckpt, pl.u_out, pt, gdn::fwd_split_ws_gates(ws, B * Hq * nch),
                                                info.sm_count, stream);
            }
            cudaFreeAsync(ws, stream);
            if (e != cudaSuccess) {
                cudaGetLastError();
                return GDN_ERR_LAUNCH;
            }
            if ((st = stg.out_back(out, dout, nout))) return st;
            if ((st = stg.out_back(S_final, dSf, nstate))) return st;
            return GDN_OK;
        }
        cudaGetLastError();
    }
    // per-query-head copies of the states (each query head of a group recomputes its memory)
    void *xs = nullptr;
    if (scratch_alloc(&xs, (size_t)(2 * nxstate), stream) != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_ALLOC;
    }
    float *S0x = static_cast<float *>(xs), *Sfx = S0x + nxstate / 4;
    cudaError_t e = cudaSuccess;
    if (dS0) e = gdn::launch_expand_states(static_cast<const float *>(dS0), S0x, B, Hq, group, dv * dk, stream);
    p.S0 = dS0 ? S0x : nullptr;
    p.out = const_cast<void *>(dout);
    p.S_final = dSf ? Sfx : nullptr;
    p.B = B; p.T = T; p.H = Hq; p.dk = dk; p.dv = dv; p.chunk = chunk; p.dtype = dtype;
    p.group = group;
    if (e == cudaSuccess) {
        if (T == 0) {
            if (p.S_final)
                e = p.S0 ? cudaMemcpyAsync(Sfx, S0x, (size_t)nxstate, cudaMemcpyDeviceToDevice, stream)
                         : cudaMemsetAsync(Sfx, 0, (size_t)nxstate, stream);
        } else if ((st = run_device(p, info, false, stream))) {
            cudaFreeAsync(xs, stream);
            return st;
        }
    }
    if (e == cudaSuccess && dSf)
        e = gdn::launch_pick_states(Sfx, static_cast<float *>(const_cast<void *>(dSf)), B, Hq, group, dv * dk,
                                    stream);
    cudaFreeAsync(xs, stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_LAUNCH;
    }
    if ((st = stg.out_back(out, dout, nout))) return st;
    if ((st = stg.out_back(S_final, dSf, nstate))) return st;
    return GDN_OK;
}

extern "C" int gdn_decode_step_grouped(const void *q, const void *k, const void *v, const float *log_alpha,
                                       const float *beta, float *S, void *out, int64_t B, int64_t Hq, int64_t Hkv,
                                       int64_t dk, int64_t dv, void *stream_, int dtype) {
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if (B < 0 || Hq < 0 || Hkv < 0 || dk < 0 || dv < 0) return GDN_ERR_INVALID_SIZE;
    if (!supported_dim(dk) || !supported_dim(dv)) return GDN_ERR_UNSUPPORTED;
    if ((Hq > 0) != (Hkv > 0) || (Hkv > 0 && (Hq % Hkv != 0 || Hq / Hkv > 64))) return GDN_ERR_INVALID_SIZE;
    const int64_t es = (dtype == GDN_F32) ? 4 : 2;
    int64_t nhq, nhk, nq, nk, nv, nout, nstate;
    if (__builtin_mul_overflow(B, Hq, &nhq) || __builtin_mul_overflow(B, Hkv, &nhk) || !mul3(nhq, dk, es, &nq) ||
        !mul3(nhk, dk, es, &nk) || !mul3(nhk, dv, es, &nv) || !mul3(nhq, dv, es, &nout) ||
        !mul3(nhk, dv, dk * 4, &nstate) || nhq > (int64_t)INT32_MAX)
        return GDN_ERR_INVALID_SIZE;
    if (nhq == 0) return GDN_OK;
    if (!q || !k || !v || !log_alpha || !beta || !S || !out) return GDN_ERR_NULL_PTR;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned4(log_alpha) || !aligned4(beta) ||
        !aligned16(S) || !aligned16(out))
        return GDN_ERR_MISALIGNED;
    const Span sq(q, nq), sk(k, nk), sv(v, nv), sla(log_alpha, nhk * 4), sbe(beta, nhk * 4);
    const Span ss(S, nstate), so(out, nout);
    for (const Span &x : {sq, sk, sv, sla, sbe, ss})
        if (overlaps(so, x)) return GDN_ERR_ALIAS;
    for (const Span &x : {sq, sk, sv, sla, sbe})
        if (overlaps(ss, x)) return GDN_ERR_ALIAS;

    DeviceInfo info;
    if (int st = device_info(&info)) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    Stager stg(stream);
    DecodeProblem p;
    int st = GDN_OK;
    const void *dS = nullptr, *dout = nullptr;
    if ((st = stg.in(q, nq, true, &p.q)) || (st = stg.in(k, nk, true, &p.k)) || (st = stg.in(v, nv, true, &p.v)) ||
        (st = stg.in(log_alpha, nhk * 4, true, reinterpret_cast<const void **>(&p.log_alpha))) ||
        (st = stg.in(beta, nhk * 4, true, reinterpret_cast<const void **>(&p.beta))) ||
        (st = stg.in(S, nstate, true, &dS)) || (st = stg.in(out, nout, false, &dout)))
        return st;
    p.S = static_cast<float *>(const_cast<void *>(dS));
    p.out = const_cast<void *>(dout);
    p.B = B; p.H = Hq; p.dk = dk; p.dv = dv; p.dtype = dtype;
    p.group = (int)(Hq / Hkv);
    if (gdn::launch_decode(p, stream) != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_LAUNCH;
    }
    if ((st = stg.out_back(out, p.out, nout))) return st;
    if ((st = stg.out_back(S, p.S, nstate))) return st;
    return GDN_OK;
}

extern "C" int gdn_causal_conv(const void *x, const float *weight, const float *state_in, void *y,
                               float *state_out, int64_t B, int64_t T, int64_t C, int64_t W, void *stream_,
                               int dtype) {
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if (B < 0 || T < 0 || C < 0) return GDN_ERR_INVALID_SIZE;
    if (W < 1 || W > 4) return GDN_ERR_UNSUPPORTED;
    const int64_t es = (dtype == GDN_F32) ? 4 : 2;
    int64_t nx, nst;
    if (!mul3(B, T, C * es, &nx) || !mul3(B, W - 1, C * 4, &nst) || C > (INT64_MAX / 16)) return GDN_ERR_INVALID_SIZE;
    if (B * C == 0) return GDN_OK;
    if ((T > 0 && (!x || !y)) || !weight) return GDN_ERR_NULL_PTR;
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) & (uintptr_t)(es - 1)) return GDN_ERR_MISALIGNED;
    if (!aligned4(weight) || !aligned4(state_in) || !aligned4(state_out)) return GDN_ERR_MISALIGNED;
    const Span sx(x, nx), sy(y, nx), sw(weight, C * W * 4), si(state_in, nst), so(state_out, nst);
    for (const Span &o : {sy, so})
        for (const Span &i : {sx, sw})
            if (overlaps(o, i)) return GDN_ERR_ALIAS;
    if (overlaps(sy, si) || overlaps(sy, so)) return GDN_ERR_ALIAS;
    if (overlaps(si, so) && si.lo != so.lo) return GDN_ERR_ALIAS;

    DeviceInfo info;
    if (int st = device_info(&info)) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    Stager stg(stream);
    int st = GDN_OK;
    const void *dx = nullptr, *dw = nullptr, *dsi = nullptr, *dy = nullptr, *dso = nullptr;
    if ((st = stg.in(x, nx, true, &dx)) || (st = stg.in(weight, C * W * 4, true, &dw)) ||
        (st = stg.in(state_in, nst, true, &dsi)) || (st = stg.in(y, nx, false, &dy)))
        return st;
    if (state_out && state_out == state_in) {
        dso = dsi;
    } else if ((st = stg.in(state_out, nst, false, &dso))) {
        return st;
    }
    // an in-place state update with several token tiles reads the old state from a copy
    void *copy = nullptr;
    cudaError_t e = cudaSuccess;
    if (dso && dso == dsi && T > 128 && nst > 0) {
        if (scratch_alloc(&copy, (size_t)nst, stream) != cudaSuccess) {
            cudaGetLastError();
            return GDN_ERR_ALLOC;
        }
        e = cudaMemcpyAsync(copy, dsi, (size_t)nst, cudaMemcpyDeviceToDevice, stream);
        dsi = copy;
    }
    if (e == cudaSuccess)
        e = gdn::launch_causal_conv(dx, static_cast<const float *>(dw), static_cast<const float *>(dsi),
                                    const_cast<void *>(dy), static_cast<float *>(const_cast<void *>(dso)), B, T, C,
                                    (int)W, dtype, stream);
    if (copy) cudaFreeAsync(copy, stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_LAUNCH;
    }
    if ((st = stg.out_back(y, dy, nx))) return st;
    if ((st = stg.out_back(state_out, dso, nst))) return st;
    return GDN_OK;
}

extern "C" int gdn_device_status(void *stream_) {
    DeviceInfo info;
    if (int st = device_info(&info)) return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream_)) != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_LAUNCH;
    }
    // take every word (each read clears it), then report
    const bool a = gdn::take_split_timeout(), b = gdn::take_tc_timeout(), c = gdn::take_selftest_timeout(),
               d = gdn::take_bwd_timeout(), g = gdn::take_grouped_timeout();
    return (a || b || c || d || g) ? GDN_ERR_DEVICE_TIMEOUT : GDN_OK;
}

extern "C" int gdn_selftest_device_timeout(void *stream_) {
    DeviceInfo info;
    if (int st = device_info(&info)) return st;
    if (gdn::launch_selftest_timeout(static_cast<cudaStream_t>(stream_)) != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_LAUNCH;
    }
    return GDN_OK;
}

// ---------------------------------------------------------------- forward with the short convolution
extern "C" int gdn_forward_conv(const void *q, const void *k, const void *v, const float *x_alpha, const float *x_beta,
                                const float *conv_weight, const float *conv_state, float *conv_state_out,
                                const float *S0, void *out, float *S_final, int64_t B, int64_t T, int64_t H,
                                int64_t dk, int64_t dv, int64_t W, int64_t chunk, void *stream_, int dtype) {
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if (B < 0 || T < 0 || H < 0 || dk < 0 || dv < 0 || chunk < 0 || W < 0) return GDN_ERR_INVALID_SIZE;
    if (!supported_dim(dk) || !supported_dim(dv) || !supported_chunk(chunk) || W < 1 || W > 4)
        return GDN_ERR_UNSUPPORTED;
    const int64_t es = (dtype == GDN_F32) ? 4 : 2;
    int64_t ntok, nqk, nv, nstate, cq = 0, cv = 0, nw = 0, ncs = 0;
    if (!mul3(B, T, H, &ntok) || !mul3(ntok, dk, es, &nqk) || !mul3(ntok, dv, es, &nv) || !mul2ok(B, H) ||
        !mul3(B * H, dv, dk * 4, &nstate) || ntok > (INT64_MAX / 8) || __builtin_mul_overflow(H, dk, &cq) ||
        __builtin_mul_overflow(H, dv, &cv) || !mul3(2 * cq + cv, W, 4, &nw) || !mul3(B, (W - 1) * 4, 2 * cq + cv, &ncs))
        return GDN_ERR_INVALID_SIZE;
    if (B * H == 0) return GDN_OK;
    if (ntok > 0 && (!q || !k || !v || !x_alpha || !x_beta || !out || !conv_weight)) return GDN_ERR_NULL_PTR;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned4(x_alpha) || !aligned4(x_beta) ||
        !aligned16(S0) || !aligned16(out) || !aligned16(S_final) || !aligned4(conv_weight) || !aligned4(conv_state) ||
        !aligned4(conv_state_out))
        return GDN_ERR_MISALIGNED;
    const Span sq(q, nqk), sk(k, nqk), sv(v, nv), sla(x_alpha, ntok * 4), sbe(x_beta, ntok * 4);
    const Span s0(S0, nstate), sf(S_final, nstate), so(out, nv), swt(conv_weight, nw), scs(conv_state, ncs),
        sco(conv_state_out, ncs);
    for (const Span &x : {sq, sk, sv, sla, sbe, s0, sf, swt, scs, sco})
        if (overlaps(so, x)) return GDN_ERR_ALIAS;
    if (overlaps(sf, s0) && !(sf.lo == s0.lo)) return GDN_ERR_ALIAS;
    for (const Span &x : {sq, sk, sv, sla, sbe, swt, scs, sco})
        if (overlaps(sf, x)) return GDN_ERR_ALIAS;
    if (overlaps(sco, scs) && !(sco.lo == scs.lo)) return GDN_ERR_ALIAS;
    for (const Span &x : {sq, sk, sv, sla, sbe, swt, s0})
        if (overlaps(sco, x)) return GDN_ERR_ALIAS;
    DeviceInfo info;
    if (int st = device_info(&info)) return st;
    // device memory only
    const void *ptrs[] = {q, k, v, x_alpha, x_beta, conv_weight, conv_state, conv_state_out, S0, out, S_final};
    for (const void *ptr : ptrs)
        if (ptr && !is_device_pointer(ptr)) return GDN_ERR_UNSUPPORTED;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const float *st_q = conv_state, *st_k = conv_state ? conv_state + B * (W - 1) * cq : nullptr,
                *st_v = conv_state ? conv_state + 2 * B * (W - 1) * cq : nullptr;
    cudaError_t e = cudaSuccess;
    int st = GDN_OK;
    if (T == 0) {
        if (S_final && S_final != S0)
            e = S0 ? cudaMemcpyAsync(S_final, S0, (size_t)nstate, cudaMemcpyDeviceToDevice, stream)
                   : cudaMemsetAsync(S_final, 0, (size_t)nstate, stream);
    } else {
        // the convolution of q, k and v into scratch (one launch), then the raw forward on its outputs
        void *y = nullptr;
        if (scratch_alloc(&y, (size_t)(2 * nqk + nv), stream) != cudaSuccess) {
            cudaGetLastError();
            return GDN_ERR_ALLOC;
        }
        uint8_t *yb = static_cast<uint8_t *>(y);
        const void *xs[3] = {q, k, v};
        const float *wts[3] = {conv_weight, conv_weight + cq * W, conv_weight + 2 * cq * W};
        const float *sts[3] = {st_q, st_k, st_v};
        void *ys[3] = {yb, yb + nqk, yb + 2 * nqk};
        const int64_t Cs[3] = {cq, cq, cv};
        e = gdn::launch_causal_conv3(xs, wts, sts, ys, Cs, 3, B, T, (int)W, dtype, stream);
        if (e == cudaSuccess)
            st = forward_impl(yb, yb + nqk, yb + 2 * nqk, x_alpha, x_beta, S0, out, S_final, B, T, H, dk, dv, chunk,
                              stream_, dtype, true);
        cudaFreeAsync(y, stream);
        if (st) return st;
    }
    // the carried state after the call (after every read of the old one on this stream)
    if (e == cudaSuccess && conv_state_out) {
        float *o = conv_state_out;
        e = gdn::launch_conv_state_update(q, st_q, o, B, T, cq, (int)W, dtype, stream);
        if (e == cudaSuccess)
            e = gdn::launch_conv_state_update(k, st_k, o + B * (W - 1) * cq, B, T, cq, (int)W, dtype, stream);
        if (e == cudaSuccess)
            e = gdn::launch_conv_state_update(v, st_v, o + 2 * B * (W - 1) * cq, B, T, cv, (int)W, dtype, stream);
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_LAUNCH;
    }
    return GDN_OK;
}
