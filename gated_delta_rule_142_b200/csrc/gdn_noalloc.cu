// gdn_noalloc.cu -- gdn_forward_noalloc: the forward without any device
// allocation.
//
// Some callers cannot allocate device memory during a call. Examples:
// - a framework whose caching allocator already owns the whole device heap;
// - a serving loop that must never enter the driver's allocator on its hot
//   path, because of its latency or its failure modes;
// - code that has no permission to grow the process's device footprint.
// gdn_forward takes stream-ordered scratch for long sequences with few heads
// (the segment transfers, the prefix entry states) and staging buffers for host
// pointers. This entry point does neither. Its scratch is one file-scope device
// array of GDN_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds
// until the process exits, and it accepts device memory only.
//
// The array's device address comes from cudaGetSymbolAddress, called once per
// device with that device current during the first call on it (host code may
// not use the symbol itself as a device address). That first call on a device
// should therefore come before any stream capture. Every call shares the array
// and leaves its last contents there. Nothing in it needs to start at zero,
// because each launch writes every scratch element before reading it (the
// test runs an unrelated problem between two checked calls to show it). Calls
// whose executions overlap on the GPU (different streams, no ordering) race
// on the array.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include <atomic>

#include "gdn.h"
#include "gdn_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[GDN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::atomic<uintptr_t> g_scratch_addr[kMaxDevices];
std::atomic<int> g_sm_count[kMaxDevices];

// Device address of the scratch array on the current device (set up on first use).
int scratch_address(int dev, void **addr) {
    if (dev < 0 || dev >= kMaxDevices) return GDN_ERR_DEVICE;
    uintptr_t a = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (a == 0) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return GDN_ERR_DEVICE;
        }
        a = reinterpret_cast<uintptr_t>(p);
        g_scratch_addr[dev].store(a, std::memory_order_release);
    }
    *addr = reinterpret_cast<void *>(a);
    return GDN_OK;
}

bool is_device(const void *p) {
    if (p == nullptr) return true;
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged;
}

bool dim_ok(int64_t d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool al(const void *p, uintptr_t m) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & m) == 0; }
bool overlap(const void *a, int64_t na, const void *b, int64_t nb) {
    if (!a || !b || na <= 0 || nb <= 0) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + (uintptr_t)nb && y < x + (uintptr_t)na;
}

}  // namespace

extern "C" int gdn_forward_noalloc(const void *q, const void *k, const void *v, const float *log_alpha,
                                   const float *beta, const float *S0, void *out, float *S_final, int64_t B,
                                   int64_t T, int64_t H, int64_t dk, int64_t dv, int64_t chunk, void *stream_,
                                   int dtype) {
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;
    if (B < 0 || T < 0 || H < 0 || dk < 0 || dv < 0 || chunk < 0) return GDN_ERR_INVALID_SIZE;
    if (!dim_ok(dk) || !dim_ok(dv) || !(chunk == 16 || chunk == 32 || chunk == 64)) return GDN_ERR_UNSUPPORTED;
    const int64_t es = (dtype == GDN_F32) ? 4 : 2;
    // the same size checks as gdn_forward: B * H first, since with T == 0 the token count says nothing
    int64_t nh, ntok, nqk, nv, nst;
    if (__builtin_mul_overflow(B, H, &nh) || __builtin_mul_overflow(nh, T, &ntok) ||
        __builtin_mul_overflow(ntok, dk * es, &nqk) || __builtin_mul_overflow(ntok, dv * es, &nv) ||
        __builtin_mul_overflow(nh, dv * dk * 4, &nst) || ntok > (INT64_MAX / 8))
        return GDN_ERR_INVALID_SIZE;
    if (nh == 0) return GDN_OK;
    if (ntok > 0 && (!q || !k || !v || !log_alpha || !beta || !out)) return GDN_ERR_NULL_PTR;
    if (!al(q, 15) || !al(k, 15) || !al(v, 15) || !al(log_alpha, 3) || !al(beta, 3) || !al(S0, 15) ||
        !al(out, 15) || !al(S_final, 15))
        return GDN_ERR_MISALIGNED;
    const void *ins[] = {q, k, v, log_alpha, beta, S0, S_final};
    const int64_t lens[] = {nqk, nqk, nv, ntok * 4, ntok * 4, nst, nst};
    for (int i = 0; i < 7; ++i)
        if (overlap(out, nv, ins[i], lens[i])) return GDN_ERR_ALIAS;
    for (int i = 0; i < 5; ++i)
        if (overlap(S_final, nst, ins[i], lens[i])) return GDN_ERR_ALIAS;
    if (S0 && S_final && S0 != S_final && overlap(S0, nst, S_final, nst)) return GDN_ERR_ALIAS;

    int dev = -1, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10) {
        cudaGetLastError();
        return GDN_ERR_DEVICE;
    }
    // device memory only: host buffers would need staging allocations
    if (!is_device(q) || !is_device(k) || !is_device(v) || !is_device(log_alpha) || !is_device(beta) ||
        !is_device(S0) || !is_device(out) || !is_device(S_final))
        return GDN_ERR_UNSUPPORTED;
    int sms = g_sm_count[dev].load(std::memory_order_relaxed);
    if (sms <= 0) {
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return GDN_ERR_DEVICE;
        }
        g_sm_count[dev].store(sms, std::memory_order_relaxed);
    }
    void *scratch = nullptr;
    if (int st = scratch_address(dev, &scratch)) return st;

    gdn::FwdProblem p;
    p.q = q; p.k = k; p.v = v; p.log_alpha = log_alpha; p.beta = beta; p.S0 = S0; p.out = out;
    p.S_final = S_final; p.B = B; p.T = T; p.H = H; p.dk = dk; p.dv = dv; p.chunk = chunk; p.dtype = dtype;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    cudaError_t e = cudaSuccess;
    if (T == 0) {
        if (S_final && S_final != S0)
            e = S0 ? cudaMemcpyAsync(S_final, S0, (size_t)nst, cudaMemcpyDeviceToDevice, stream)
                   : cudaMemsetAsync(S_final, 0, (size_t)nst, stream);
    } else if (gdn::fwd_tc_supported(p)) {
        // the two-kernel forward when its per-chunk workspace fits the array, else the
        // single-kernel forward, which needs scratch only for segments
        const int nseg_split = gdn::fwd_tc_segments(p, sms, true);
        if (gdn::fwd_split_supported(p) &&
            gdn::fwd_split_workspace_bytes(p, nseg_split) <= (size_t)GDN_NOALLOC_SCRATCH_BYTES) {
            e = gdn::launch_fwd_split(p, nseg_split, sms, scratch, stream);
        } else {
            int nseg = gdn::fwd_tc_segments(p, sms, false);
            if (gdn::fwd_tc_workspace_bytes(p, nseg) > (size_t)GDN_NOALLOC_SCRATCH_BYTES) {
                // a segment count the caller forced through GDN_SEGMENTS is honoured or refused;
                // otherwise the forward runs with the most segments whose scratch fits (one
                // segment needs none), trading chunk-level parallelism for the fixed array
                const char *env = getenv("GDN_SEGMENTS");
                if (env && atoi(env) >= 1) return GDN_ERR_SCRATCH_LIMIT;
                while (nseg > 1 && gdn::fwd_tc_workspace_bytes(p, nseg) > (size_t)GDN_NOALLOC_SCRATCH_BYTES) --nseg;
            }
            const size_t need = gdn::fwd_tc_workspace_bytes(p, nseg);
            e = gdn::launch_fwd_tc(p, nseg, need ? scratch : nullptr, stream);
        }
    } else {
        e = gdn::launch_fwd_simt(p, sms, stream);  // needs no scratch
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_LAUNCH;
    }
    return GDN_OK;
}
