// Diagnostics: launch counter and per-stage event timing (see runtime.cuh).
#include <atomic>
#include <mutex>
#include <string.h>
#include <vector>

#include "common.cuh"
#include "runtime.cuh"

namespace path {

namespace {
std::atomic<unsigned long long> g_launches{0};
std::atomic<int> g_profile{0};
std::atomic<int> g_withhold{0};
struct Rec {
    const char *name;
    cudaEvent_t e0, e1;
};
std::mutex g_mu;
std::vector<Rec> g_recs;
}  // namespace

void count_launches(int n) { g_launches.fetch_add((unsigned long long)n); }

int withhold_kv_load() { return g_withhold.load(); }

int sm_count()
{
    static std::atomic<int> cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cache[dev].load();
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            return 148;
        cache[dev].store(n);
    }
    return n;
}

Stage::Stage(const char *name, cudaStream_t st) : name_(name), st_(st)
{
    if (!g_profile.load()) return;
    if (cudaEventCreate(&e0_) != cudaSuccess) {
        e0_ = nullptr;
        return;
    }
    cudaEventRecord(e0_, st_);
}

Stage::~Stage()
{
    if (!e0_) return;
    cudaEvent_t e1;
    if (cudaEventCreate(&e1) != cudaSuccess) {
        cudaEventDestroy(e0_);
        return;
    }
    cudaEventRecord(e1, st_);
    std::lock_guard<std::mutex> lk(g_mu);
    g_recs.push_back({name_, e0_, e1});
}

}  // namespace path

extern "C" {

unsigned long long path_kernel_launch_count(void) { return path::g_launches.load(); }

int path_profile_enable(int on)
{
    const int prev = path::g_profile.exchange(on ? 1 : 0);
    return prev;
}

int path_profile_read(path_stage_time *out, int max_entries)
{
    using namespace path;
    std::vector<Rec> recs;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        recs.swap(g_recs);
    }
    int n = 0;
    for (const Rec &r : recs) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.e1) == cudaSuccess) cudaEventElapsedTime(&ms, r.e0, r.e1);
        cudaEventDestroy(r.e0);
        cudaEventDestroy(r.e1);
        int slot = -1;
        for (int i = 0; i < n; ++i)
            if (strcmp(out[i].name, r.name) == 0) slot = i;
        if (slot < 0) {
            if (n >= max_entries) continue;
            slot = n++;
            memset(&out[slot], 0, sizeof(out[slot]));
            strncpy(out[slot].name, r.name, sizeof(out[slot].name) - 1);
        }
        out[slot].total_ms += ms;
        out[slot].count += 1;
    }
    return n;
}

}  // extern "C"

extern "C" path_status path_test_withhold_kv_load(int on)
{
    if (on != 0 && on != 1) return PATH_ERR_INVALID_ARG;
    path::g_withhold.store(on);
    return PATH_OK;
}
