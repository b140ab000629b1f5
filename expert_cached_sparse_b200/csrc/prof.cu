// Launch counters and optional per-step device timing.  Counters are always
// on (one relaxed atomic add per launch).  With timing enabled, each step's
// launches are bracketed by a pair of CUDA events on the stream they run on;
// moe_profile_read waits for the pending events and sums their durations.
#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"

namespace moe {
namespace {

struct Pending {
    int kind;
    cudaEvent_t a, b;
};

std::atomic<uint64_t> g_launches[MOE_PROF_COUNT];
std::atomic<int> g_timing{0};
std::mutex g_mu;
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_free;
double g_ms[MOE_PROF_COUNT];
uint64_t g_timed[MOE_PROF_COUNT];

cudaEvent_t get_event()
{
    if (!g_free.empty()) {
        cudaEvent_t e = g_free.back();
        g_free.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

}  // namespace

void prof_count(int kind, int launches) { g_launches[kind].fetch_add((uint64_t)launches, std::memory_order_relaxed); }

ProfScope::ProfScope(int kind, cudaStream_t st) : kind_(kind), st_(st), a_(nullptr)
{
    if (!g_timing.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_mu);
    a_ = get_event();
    if (a_ && cudaEventRecord(a_, st_) != cudaSuccess) {
        g_free.push_back(a_);
        a_ = nullptr;
    }
}

ProfScope::~ProfScope()
{
    if (!a_) return;
    std::lock_guard<std::mutex> lk(g_mu);
    cudaEvent_t b = get_event();
    if (!b || cudaEventRecord(b, st_) != cudaSuccess) {
        g_free.push_back(a_);
        if (b) g_free.push_back(b);
        return;
    }
    g_pending.push_back({kind_, a_, b});
}

}  // namespace moe

extern "C" int moe_profile_enable(int timing)
{
    moe::g_timing.store(timing ? 1 : 0);
    return MOE_OK;
}

extern "C" int moe_profile_read(moe_prof_entry* out, int count, int reset)
{
    if (!out || count < 0) return MOE_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(moe::g_mu);
    int rc = MOE_OK;
    for (auto& p : moe::g_pending) {
        float ms = 0.0f;
        if (cudaEventSynchronize(p.b) != cudaSuccess || cudaEventElapsedTime(&ms, p.a, p.b) != cudaSuccess)
            rc = MOE_ERR_CUDA;
        moe::g_ms[p.kind] += ms;
        moe::g_timed[p.kind] += 1;
        moe::g_free.push_back(p.a);
        moe::g_free.push_back(p.b);
    }
    moe::g_pending.clear();
    for (int i = 0; i < count && i < MOE_PROF_COUNT; i++) {
        out[i].launches = moe::g_launches[i].load();
        out[i].timed = moe::g_timed[i];
        out[i].ms = moe::g_ms[i];
    }
    if (reset) {
        for (int i = 0; i < MOE_PROF_COUNT; i++) {
            moe::g_launches[i].store(0);
            moe::g_timed[i] = 0;
            moe::g_ms[i] = 0.0;
        }
    }
    return rc;
}
