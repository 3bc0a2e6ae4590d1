// Optional per-launch device timing of the library's kernels (CUDA events on
// the launch stream), summed per kernel kind with each launch's algorithmic
// work.  Used by the benchmark to report the dominant kernel's achieved rate
// over the timed region.
#include <mutex>
#include <vector>

#include "common.cuh"
#include "timing.cuh"

namespace lsn {

namespace {

constexpr size_t kMaxRecords = 65536;

struct Record {
    cudaEvent_t a = nullptr, b = nullptr;
    int kind = 0;
    int kernels = 1;
    double work = 0.0;
};

struct TimingState {
    std::mutex mu;
    bool on = false;
    std::vector<Record> recs;     // events are kept for reuse across reads
    size_t used = 0;
    lsn_kernel_timing untimed = {};
};

TimingState& state() {
    static TimingState s;
    return s;
}

}  // namespace

TimingScope::TimingScope(int kind, double work, cudaStream_t st, int kernels) : st_(st), idx_(-1) {
    TimingState& s = state();
    std::lock_guard<std::mutex> lk(s.mu);
    if (!s.on) return;
    if (s.used >= kMaxRecords) {
        s.untimed.launches[kind] += 1;
        s.untimed.kernels[kind] += (uint64_t)kernels;
        s.untimed.work[kind] += work;
        return;
    }
    if (s.used == s.recs.size()) {
        Record r;
        if (cudaEventCreate(&r.a) != cudaSuccess || cudaEventCreate(&r.b) != cudaSuccess) return;
        s.recs.push_back(r);
    }
    Record& r = s.recs[s.used];
    r.kind = kind;
    r.kernels = kernels;
    r.work = work;
    if (cudaEventRecord(r.a, st) != cudaSuccess) return;
    idx_ = (long)s.used++;
}

TimingScope::~TimingScope() {
    if (idx_ < 0) return;
    TimingState& s = state();
    std::lock_guard<std::mutex> lk(s.mu);
    cudaEventRecord(s.recs[(size_t)idx_].b, st_);
}

}  // namespace lsn

extern "C" {

lsn_status lsn_timing_enable(int on) {
    lsn::TimingState& s = lsn::state();
    std::lock_guard<std::mutex> lk(s.mu);
    s.on = on != 0;
    if (s.on) {
        s.used = 0;
        s.untimed = lsn_kernel_timing();
    }
    return LSN_OK;
}

lsn_status lsn_timing_read(lsn_kernel_timing* out) {
    LSN_CHECK_ARG(out != nullptr, "lsn_timing_read: out is NULL");
    lsn::TimingState& s = lsn::state();
    std::lock_guard<std::mutex> lk(s.mu);
    lsn_kernel_timing t = s.untimed;
    for (size_t i = 0; i < s.used; ++i) {
        lsn::Record& r = s.recs[i];
        LSN_CUDA_TRY(cudaEventSynchronize(r.b));
        float ms = 0.0f;
        LSN_CUDA_TRY(cudaEventElapsedTime(&ms, r.a, r.b));
        t.launches[r.kind] += 1;
        t.kernels[r.kind] += (uint64_t)r.kernels;
        t.ms[r.kind] += ms;
        t.work[r.kind] += r.work;
    }
    s.used = 0;
    s.untimed = lsn_kernel_timing();
    *out = t;
    return LSN_OK;
}

}  // extern "C"
