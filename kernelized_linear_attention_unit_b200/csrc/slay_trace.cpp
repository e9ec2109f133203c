// slay_trace.cpp -- optional per-launch timing of libslay.so's kernels.
//
// While enabled (slay_trace_enable(1)), every kernel launch inside the library is
// bracketed by a pair of CUDA events recorded on the launch's stream; slay_trace_read
// waits for them and returns (kernel name, milliseconds) records.  Disabled, the cost is
// one relaxed atomic load per launch.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "slay.h"
#include "slay_internal.h"

namespace slay {
namespace {

struct Rec {
    const char* name;
    cudaEvent_t a, b;
};

std::atomic<int> g_on{0};
std::mutex g_mu;
std::vector<Rec>& recs() { static auto* v = new std::vector<Rec>(); return *v; }
std::vector<cudaEvent_t>& pool() { static auto* v = new std::vector<cudaEvent_t>(); return *v; }
thread_local int t_open = -1;

cudaEvent_t take()
{
    if (!pool().empty()) {
        cudaEvent_t e = pool().back();
        pool().pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

}  // namespace

TraceScope::TraceScope(const char* name, cudaStream_t st) : st_(st), idx_(-1)
{
    if (!g_on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lock(g_mu);
    Rec r{name, take(), take()};
    if (!r.a || !r.b) return;
    cudaEventRecord(r.a, st);
    recs().push_back(r);
    idx_ = static_cast<int>(recs().size()) - 1;
}

TraceScope::~TraceScope()
{
    if (idx_ < 0) return;
    std::lock_guard<std::mutex> lock(g_mu);
    if (idx_ < static_cast<int>(recs().size())) cudaEventRecord(recs()[idx_].b, st_);
}

}  // namespace slay

using namespace slay;

extern "C" {

slay_status slay_trace_enable(int on)
{
    g_on.store(on ? 1 : 0);
    return SLAY_OK;
}

int slay_trace_read(const char** names, float* ms, int cap)
{
    std::lock_guard<std::mutex> lock(g_mu);
    int n = 0;
    for (const Rec& r : recs()) {
        if (n < cap) {
            float t = -1.0f;
            if (cudaEventSynchronize(r.b) == cudaSuccess) cudaEventElapsedTime(&t, r.a, r.b);
            if (names) names[n] = r.name;
            if (ms) ms[n] = t;
        }
        ++n;
        pool().push_back(r.a);
        pool().push_back(r.b);
    }
    recs().clear();
    return n;
}

}  // extern "C"
