// Stage timing with CUDA events recorded on the caller's stream between the
// kernels of one operator call (moe_profile_enable / moe_profile_read).
#include <string.h>

#include <mutex>

#include "common.cuh"

namespace moe {

namespace {
constexpr int kMaxEvents = 4096;
struct Rec {
    cudaEvent_t ev;
    const char* name;  // null = start of a call
    int launches;      // kernels launched since the previous record
};
bool g_enabled = false;
int g_count = 0;
Rec g_recs[kMaxEvents];
cudaEvent_t g_pool[kMaxEvents];
int g_pool_n = 0;
std::mutex g_mu;

void record(cudaStream_t s, const char* name, int launches) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_enabled || g_count >= kMaxEvents) return;
    if (g_count >= g_pool_n) {
        if (cudaEventCreate(&g_pool[g_pool_n]) != cudaSuccess) return;
        ++g_pool_n;
    }
    cudaEvent_t e = g_pool[g_count];
    if (cudaEventRecord(e, s) != cudaSuccess) return;
    g_recs[g_count++] = Rec{e, name, launches};
}
}  // namespace

void prof_begin(cudaStream_t s) { if (g_enabled) record(s, nullptr, 0); }
void prof_mark(cudaStream_t s, const char* stage, int launches) { if (g_enabled) record(s, stage, launches); }

}  // namespace moe

using namespace moe;

extern "C" {

void moe_profile_enable(int enable) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_enabled = enable != 0;
    if (g_enabled) g_count = 0;
}

int moe_profile_read(const char** names, int* launches, double* total_ms, int max_stages) {
    std::lock_guard<std::mutex> lk(g_mu);
    int n = 0;
    for (int i = 1; i < g_count; ++i) {
        if (!g_recs[i].name || !g_recs[i - 1].ev) continue;
        if (cudaEventSynchronize(g_recs[i].ev) != cudaSuccess) return MOE_ERR_CUDA;
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, g_recs[i - 1].ev, g_recs[i].ev) != cudaSuccess) return MOE_ERR_CUDA;
        int j = 0;
        while (j < n && strcmp(names[j], g_recs[i].name) != 0) ++j;
        if (j == n) {
            if (n == max_stages) continue;
            names[n] = g_recs[i].name;
            launches[n] = 0;
            total_ms[n] = 0.0;
            ++n;
        }
        launches[j] += g_recs[i].launches;
        total_ms[j] += ms;
    }
    return n;
}

}  // extern "C"
