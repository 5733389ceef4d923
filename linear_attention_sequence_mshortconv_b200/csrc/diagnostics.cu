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

// fp32 FMA throughput probe: 8 independent FMA chains per thread, enough blocks to fill
// every SM several times; the result is stored only if it is a sentinel no input hits,
// so the compiler cannot drop the chains.
__global__ void __launch_bounds__(512) fma_probe_kernel(float a, float b, int iters, float* sink)
{
    float x[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = a + i * 1e-3f + threadIdx.x * 1e-6f;
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = fmaf(x[i], b, a);
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) s += x[i];
    if (s == -12345.678f) *sink = s;
}

}  // namespace kda

extern "C" {

int kda_fma_probe(double* fma_per_s)
{
    if (!fma_per_s) return -1;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return -1;
    float* sink = nullptr;
    if (cudaMalloc(&sink, sizeof(float)) != cudaSuccess) return -1;
    const int blocks = sms * 8, threads = 512, iters = 4096;
    cudaEvent_t e0, e1;
    cudaEventCreate(&e0);
    cudaEventCreate(&e1);
    kda::fma_probe_kernel<<<blocks, threads>>>(0.5f, 0.999f, iters, sink);   // warm-up
    cudaEventRecord(e0);
    kda::fma_probe_kernel<<<blocks, threads>>>(0.5f, 0.999f, iters, sink);
    cudaEventRecord(e1);
    const cudaError_t err = cudaEventSynchronize(e1);
    float ms = 0.f;
    cudaEventElapsedTime(&ms, e0, e1);
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    cudaFree(sink);
    if (err != cudaSuccess || ms <= 0.f) return -1;
    *fma_per_s = (double)blocks * threads * iters * 8 / (ms * 1e-3);
    return 0;
}


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
