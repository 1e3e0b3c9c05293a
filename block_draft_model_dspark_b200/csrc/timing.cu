// Launch counting and optional per-kernel-class device timing.
//
// Every kernel launch of the library increments a process-wide counter.
// While timing is enabled, the launches of each kernel class are bracketed by
// CUDA events on their own stream, together with the algorithmic bytes and
// flops of the launch; dspark_timer_read() waits for those events and sums
// them per class.
#include <atomic>
#include <mutex>
#include <vector>

#include "internal.h"

namespace dspark {
namespace {

struct Rec { int kind; cudaEvent_t a, b; double bytes, flops; };

std::atomic<uint64_t> g_launches{0};
std::atomic<bool> g_timing{false};
std::mutex g_mu;
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t get_event() {
    if (!g_pool.empty()) { cudaEvent_t e = g_pool.back(); g_pool.pop_back(); return e; }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

}  // namespace

void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

KernelTimer::KernelTimer(int kind, cudaStream_t s, double bytes, double flops)
    : kind_(kind), s_(s), bytes_(bytes), flops_(flops) {
    if (!g_timing.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_mu);
    a_ = get_event();
    b_ = get_event();
    if (a_) cudaEventRecord(a_, s_);
}

KernelTimer::~KernelTimer() {
    if (!a_ || !b_) return;
    cudaEventRecord(b_, s_);
    std::lock_guard<std::mutex> lk(g_mu);
    g_recs.push_back({kind_, a_, b_, bytes_, flops_});
}

}  // namespace dspark

using namespace dspark;

extern "C" {

uint64_t dspark_kernel_launches(void) { return g_launches.load(); }

int dspark_timer_enable(int enable) {
    g_timing.store(enable != 0);
    return DSPARK_OK;
}

int dspark_timer_read(int kind, double* total_ms, int64_t* launches, double* bytes, double* flops) {
    if (kind < 0 || kind >= DSPARK_TIMER_KINDS || !total_ms || !launches)
        DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "timer kind out of range or NULL output");
    std::lock_guard<std::mutex> lk(g_mu);
    double ms = 0.0, by = 0.0, fl = 0.0;
    int64_t n = 0;
    std::vector<Rec> keep;
    for (const Rec& r : g_recs) {
        if (r.kind != kind) { keep.push_back(r); continue; }
        cudaError_t e = cudaEventSynchronize(r.b);
        float t = 0.f;
        if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.a, r.b);
        if (e != cudaSuccess) DSPARK_FAIL(DSPARK_ERR_CUDA, std::string("timer events: ") + cudaGetErrorString(e));
        ms += t; by += r.bytes; fl += r.flops; ++n;
        g_pool.push_back(r.a);
        g_pool.push_back(r.b);
    }
    g_recs.swap(keep);
    *total_ms = ms; *launches = n;
    if (bytes) *bytes = by;
    if (flops) *flops = fl;
    return DSPARK_OK;
}

}  // extern "C"
