// gdn_timing.cu -- per-kernel device times for benchmarking (gdn_timing_start
// / gdn_timing_stop in include/gdn.h).  While recording is on, every kernel
// the library launches is bracketed by a pair of CUDA events recorded on its
// own stream; gdn_timing_stop waits for the last of them and sums the
// elapsed times per kernel kind.  Recording only adds event records on the
// host side of each launch; the kernels and their order are unchanged.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <vector>

#include "gdn.h"
#include "gdn_internal.h"

namespace gdn {
namespace {

struct Pair {
    int kind;
    cudaEvent_t begin, end;
};

std::mutex g_mu;
bool g_on = false;
std::vector<Pair> g_pairs;
std::vector<cudaEvent_t> g_free;  // events kept for reuse
constexpr size_t kMaxPairs = 1 << 16;

cudaEvent_t take_event() {
    if (!g_free.empty()) {
        cudaEvent_t e = g_free.back();
        g_free.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return e;
}

}  // namespace

TimedLaunch::TimedLaunch(int kind, cudaStream_t stream) : kind_(kind), stream_(stream) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_on || g_pairs.size() >= kMaxPairs) return;
    begin_ = take_event();
    end_ = take_event();
    if (!begin_ || !end_ || cudaEventRecord(begin_, stream_) != cudaSuccess) {
        cudaGetLastError();
        if (begin_) g_free.push_back(begin_);
        if (end_) g_free.push_back(end_);
        begin_ = end_ = nullptr;
    }
}

TimedLaunch::~TimedLaunch() {
    if (!begin_) return;
    std::lock_guard<std::mutex> lk(g_mu);
    if (cudaEventRecord(end_, stream_) != cudaSuccess) {
        cudaGetLastError();
        g_free.push_back(begin_);
        g_free.push_back(end_);
        return;
    }
    g_pairs.push_back({kind_, begin_, end_});
}

}  // namespace gdn

extern "C" int gdn_timing_start(void) {
    std::lock_guard<std::mutex> lk(gdn::g_mu);
    for (const gdn::Pair &p : gdn::g_pairs) {
        gdn::g_free.push_back(p.begin);
        gdn::g_free.push_back(p.end);
    }
    gdn::g_pairs.clear();
    gdn::g_on = true;
    return GDN_OK;
}

extern "C" int gdn_timing_stop(double *ms, int64_t *launches) {
    std::lock_guard<std::mutex> lk(gdn::g_mu);
    gdn::g_on = false;
    for (int i = 0; i < GDN_KERNEL_KINDS; ++i) {
        if (ms) ms[i] = 0.0;
        if (launches) launches[i] = 0;
    }
    int status = GDN_OK;
    for (const gdn::Pair &p : gdn::g_pairs) {
        float t = 0.f;
        if (cudaEventSynchronize(p.end) != cudaSuccess || cudaEventElapsedTime(&t, p.begin, p.end) != cudaSuccess) {
            cudaGetLastError();
            status = GDN_ERR_LAUNCH;
        } else if (p.kind >= 0 && p.kind < GDN_KERNEL_KINDS) {
            if (ms) ms[p.kind] += t;
            if (launches) launches[p.kind] += 1;
        }
        gdn::g_free.push_back(p.begin);
        gdn::g_free.push_back(p.end);
    }
    gdn::g_pairs.clear();
    return status;
}
