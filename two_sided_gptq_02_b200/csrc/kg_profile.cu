// kg_profile.cu -- launch counters and optional event timing (see kg_profile.cuh).
#include <atomic>
#include <mutex>
#include <vector>

#include "kg_common.cuh"
#include "kg_profile.cuh"

namespace kg {

namespace {
struct Pending {
    int kind;
    cudaEvent_t a, b;
};
std::atomic<int64_t> g_launches[PK_COUNT];
std::atomic<int> g_enabled{0};
std::mutex g_mu;
std::vector<cudaEvent_t> g_pool;
std::vector<Pending> g_pending;
thread_local cudaEvent_t t_open = nullptr;
double g_ms[PK_COUNT];

cudaEvent_t take_event() {
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}
}  // namespace

void prof_before(int kind, cudaStream_t st) {
    g_launches[kind].fetch_add(1, std::memory_order_relaxed);
    if (!g_enabled.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_mu);
    t_open = take_event();
    if (t_open) cudaEventRecord(t_open, st);
}

void prof_after(int kind, cudaStream_t st) {
    if (!g_enabled.load(std::memory_order_relaxed) || !t_open) return;
    std::lock_guard<std::mutex> lk(g_mu);
    cudaEvent_t b = take_event();
    if (!b) return;
    cudaEventRecord(b, st);
    g_pending.push_back(Pending{kind, t_open, b});
    t_open = nullptr;
}

bool prof_timing() { return g_enabled.load(std::memory_order_relaxed) != 0; }

void prof_counts(int64_t out[PK_COUNT]) {
    for (int k = 0; k < PK_COUNT; ++k) out[k] = g_launches[k].load(std::memory_order_relaxed);
}

void prof_add(const int64_t add[PK_COUNT]) {
    for (int k = 0; k < PK_COUNT; ++k) g_launches[k].fetch_add(add[k], std::memory_order_relaxed);
}

}  // namespace kg

using namespace kg;

extern "C" void kron_gptq_profile_enable(int enable) { g_enabled.store(enable ? 1 : 0); }

extern "C" int kron_gptq_profile_read(int64_t* launches, double* ms, int nkinds, int reset) {
    if (nkinds < 0) return KG_ERR_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    for (const Pending& p : g_pending) {
        float t = 0.f;
        if (cudaEventSynchronize(p.b) != cudaSuccess) return KG_ERR_CUDA;
        if (cudaEventElapsedTime(&t, p.a, p.b) == cudaSuccess) g_ms[p.kind] += t;
        g_pool.push_back(p.a);
        g_pool.push_back(p.b);
    }
    g_pending.clear();
    for (int k = 0; k < nkinds && k < PK_COUNT; ++k) {
        if (launches) launches[k] = g_launches[k].load();
        if (ms) ms[k] = g_ms[k];
    }
    if (reset) {
        for (int k = 0; k < PK_COUNT; ++k) {
            g_launches[k].store(0);
            g_ms[k] = 0.0;
        }
    }
    return KG_OK;
}
