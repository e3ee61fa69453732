// Host-side diagnostics of the library: a process-wide count of kernel
// launches and optional per-stage timing with CUDA events on the stage's own
// stream (used by the benchmark to time one stage inside a full step).
#pragma once
#include <cuda_runtime.h>

namespace path {

void count_launches(int n = 1);

// path_test_withhold_kv_load's setting (0 or 1).
int withhold_kv_load();

// Streaming multiprocessors of the current device (cached per device; 148 if
// the query fails).
int sm_count();

// Brackets one stage of an entry point with events when profiling is on.
class Stage {
  public:
    Stage(const char *name, cudaStream_t st);
    ~Stage();
    Stage(const Stage &) = delete;
    Stage &operator=(const Stage &) = delete;

  private:
    const char *name_;
    cudaStream_t st_;
    cudaEvent_t e0_ = nullptr;
};

}  // namespace path
