// Measurement hooks: a count of kernel launches and optional CUDA-event
// timing around each launch, read back per kernel name. They observe the
// kernels; they take no part in what the kernels compute.
#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"

namespace qnf4 {
namespace {
std::atomic<unsigned long long> g_launches{0};
std::atomic<int> g_profiling{0};
std::mutex g_mu;
struct Rec {
    const char *name;
    cudaEvent_t a, b;
};
struct Token {
    const char *name;
    cudaEvent_t a;
};
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}
}  // namespace

void note_launch_begin(const char *name, cudaStream_t st, void **token) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    *token = nullptr;
    if (!g_profiling.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lock(g_mu);
    cudaEvent_t a = take_event();
    cudaEventRecord(a, st);
    *token = new Token{name, a};
}

bool profiling_launches() { return g_profiling.load(std::memory_order_relaxed) != 0; }

void note_launch_end(void *token, cudaStream_t st) {
    if (!token) return;
    Token *t = static_cast<Token *>(token);
    std::lock_guard<std::mutex> lock(g_mu);
    cudaEvent_t b = take_event();
    cudaEventRecord(b, st);
    g_recs.push_back(Rec{t->name, t->a, b});
    delete t;
}

}  // namespace qnf4

using namespace qnf4;

extern "C" {

void qlora_profile_enable(int on) { g_profiling.store(on ? 1 : 0); }

unsigned long long qlora_launch_count(void) { return g_launches.load(); }

int qlora_profile_read(const char *kernel, double *total_ms, int *launches) {
    double tot = 0.0;
    int cnt = 0;
    std::lock_guard<std::mutex> lock(g_mu);
    std::vector<Rec> keep;
    for (const Rec &r : g_recs) {
        if (kernel && std::strcmp(kernel, r.name) != 0) {
            keep.push_back(r);
            continue;
        }
        float ms = 0.0f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
            return (int)QLORA_ERR_CUDA;
        tot += ms;
        ++cnt;
        g_pool.push_back(r.a);
        g_pool.push_back(r.b);
    }
    g_recs.swap(keep);
    if (total_ms) *total_ms = tot;
    if (launches) *launches = cnt;
    return (int)QLORA_OK;
}

}  // extern "C"
