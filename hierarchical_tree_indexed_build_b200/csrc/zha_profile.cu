// zha_profile.cu - CUDA-event intervals around libzha kernel launches, summed per kernel.
#include <string.h>

#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "zha.h"
#include "zha_profile.h"

namespace zha {

namespace {

struct Interval {
    const char* name;
    cudaEvent_t a, b;
};

std::mutex g_mu;
bool g_on = false;
std::vector<Interval> g_done;
std::vector<cudaEvent_t> g_pool;
thread_local Interval t_open = {nullptr, nullptr, nullptr};

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

bool prof_on() { return g_on; }

void prof_begin(const char* name, cudaStream_t st) {
    std::lock_guard<std::mutex> lk(g_mu);
    t_open.name = name;
    t_open.a = take_event();
    t_open.b = take_event();
    cudaEventRecord(t_open.a, st);
}

void prof_end(cudaStream_t st) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!t_open.name) return;
    cudaEventRecord(t_open.b, st);
    g_done.push_back(t_open);
    t_open.name = nullptr;
}

}  // namespace zha

using namespace zha;

extern "C" zha_status zha_profile_enable(int32_t on) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_on = on != 0;
    return ZHA_OK;
}

extern "C" zha_status zha_profile_reset(void) {
    cudaDeviceSynchronize();
    std::lock_guard<std::mutex> lk(g_mu);
    for (auto& iv : g_done) {
        g_pool.push_back(iv.a);
        g_pool.push_back(iv.b);
    }
    g_done.clear();
    return ZHA_OK;
}

extern "C" int32_t zha_profile_read(char* names, int32_t name_len, int64_t* launches, double* total_ms,
                                    int32_t max_kernels) {
    cudaDeviceSynchronize();
    std::lock_guard<std::mutex> lk(g_mu);
    std::map<std::string, std::pair<int64_t, double>> agg;
    for (auto& iv : g_done) {
        float ms = 0.0f;
        if (cudaEventElapsedTime(&ms, iv.a, iv.b) != cudaSuccess) ms = 0.0f;
        auto& e = agg[iv.name];
        e.first += 1;
        e.second += ms;
    }
    int32_t k = 0;
    for (auto& kv : agg) {
        if (k < max_kernels) {
            if (names && name_len > 0) {
                strncpy(names + (size_t)k * name_len, kv.first.c_str(), (size_t)name_len - 1);
                names[(size_t)k * name_len + name_len - 1] = 0;
            }
            if (launches) launches[k] = kv.second.first;
            if (total_ms) total_ms[k] = kv.second.second;
        }
        ++k;
    }
    return k;
}
