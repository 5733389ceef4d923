// Launch accounting and optional CUDA-event timing of each kernel (diagnostics only).
#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "internal.h"

namespace kda {
namespace {
std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_profile{0};
std::atomic<int> g_drop_handoff{0};
std::mutex g_mu;
std::map<std::string, std::vector<std::pair<cudaEvent_t, cudaEvent_t>>> g_events;
}  // namespace

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
int debug_drop_handoff() { return g_drop_handoff.load(std::memory_order_relaxed); }

ProfileScope::ProfileScope(const char* name, cudaStream_t s) : name_(name), s_(s)
{
    if (!g_profile.load(std::memory_order_relaxed)) return;
    if (cudaEventCreate(&a_) != cudaSuccess || cudaEventCreate(&b_) != cudaSuccess) {
        a_ = b_ = nullptr;
        return;
    }
    cudaEventRecord(a_, s_);
}

ProfileScope::~ProfileScope()
{
    if (!a_) return;
    cudaEventRecord(b_, s_);
    std::lock_guard<std::mutex> lk(g_mu);
    g_events[name_].push_back({a_, b_});
}

}  // namespace kda

extern "C" {

void kda_debug_drop_handoff(int on) { kda::g_drop_handoff.store(on ? 1 : 0, std::memory_order_relaxed); }

uint64_t kda_kernel_launches(void) { return kda::g_launches.load(); }

void kda_profile_enable(int on) { kda::g_profile.store(on ? 1 : 0); }

int kda_profile_collect(const char* name, double* total_ms, int* launches)
{
    std::vector<std::pair<cudaEvent_t, cudaEvent_t>> ev;
    {
        std::lock_guard<std::mutex> lk(kda::g_mu);
        auto it = kda::g_events.find(name ? name : "");
        if (it == kda::g_events.end()) return -1;
        ev.swap(it->second);
        kda::g_events.erase(it);
    }
    double sum = 0.0;
    for (auto& p : ev) {
        cudaEventSynchronize(p.second);
        float ms = 0.f;
        cudaEventElapsedTime(&ms, p.first, p.second);
        sum += ms;
        cudaEventDestroy(p.first);
        cudaEventDestroy(p.second);
    }
    if (total_ms) *total_ms = sum;
    if (launches) *launches = (int)ev.size();
    return 0;
}

}  // extern "C"
