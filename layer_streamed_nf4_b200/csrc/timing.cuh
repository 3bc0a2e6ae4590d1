// Scope that brackets one kernel launch with timing events when per-launch
// timing is enabled (lsn_timing_enable); a no-op otherwise.
#pragma once

#include <cuda_runtime.h>

namespace lsn {

class TimingScope {
  public:
    TimingScope(int kind, double work, cudaStream_t st, int kernels = 1);
    ~TimingScope();
    TimingScope(const TimingScope&) = delete;
    TimingScope& operator=(const TimingScope&) = delete;

  private:
    cudaStream_t st_;
    long idx_;
};

}  // namespace lsn
