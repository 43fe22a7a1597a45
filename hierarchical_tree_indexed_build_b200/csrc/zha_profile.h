// zha_profile.h - optional device-time profile of libzha's own kernel launches.
#pragma once

#include <cuda_runtime.h>

namespace zha {

bool prof_on();
void prof_begin(const char* name, cudaStream_t st);
void prof_end(cudaStream_t st);

// Brackets one kernel launch with CUDA events on its stream while profiling is enabled.
struct ProfScope {
    bool on;
    cudaStream_t st;
    ProfScope(const char* name, cudaStream_t s) : on(prof_on()), st(s) {
        if (on) prof_begin(name, st);
    }
    ~ProfScope() {
        if (on) prof_end(st);
    }
};

}  // namespace zha
