// The VRAM layer pool: a fixed set of pre-allocated device slots that the
// frozen base streams through from pinned host RAM.
//
// "Can You Fine-Tune a 27B Model on a Laptop? (I Did the Math)", 7:11-7:42:
// the frozen base sits in system RAM, one decoder layer at a time is copied
// into a small buffer on the card on a separate stream so that it lands while
// the previous layer still computes, and each layer is read twice per step
// (forward, and again when backward recomputes it).  The sourcefeed article
// "An 8B Fine-Tune Now Fits in 4 GB of VRAM" (section "The trick is that
// frozen weights are just data") adds that the buffers are pre-allocated.
// The abstract of "Exact Layer Streaming" reports the failure mode this
// design rules out: gradients silently wrong through aliasing.  Here a slot
// is only ever overwritten after every holder has released it: each release
// records an event of its own on the releasing stream, and the copy stream
// waits on all the events recorded since the slot's last fill before the
// copy (a layer acquired on two streams is safe from the reader that releases
// first).
#include <chrono>
#include <mutex>
#include <thread>
#include <unordered_map>
#include <vector>

#include "common.cuh"

namespace {

constexpr int kTimingRing = 64;

struct Slot {
    int layer = -1;          // layer held (or being copied), -1 if none
    int refs = 0;            // acquire count not yet released
    bool pending = false;    // prefetched, not yet acquired: not evictable
    int n_rel = 0;           // release events recorded since the slot's last fill
    uint64_t last_release = 0;
    uint64_t last_fill = 0;
};

}  // namespace

struct lsn_pool {
    int device = 0;
    int n_slots = 0;
    size_t slot_bytes = 0, slot_stride = 0;
    uint8_t* dev = nullptr;
    cudaStream_t copy = nullptr;
    std::vector<cudaEvent_t> ready;
    // Per slot, one event per release since the slot's last fill (the vector
    // grows to the largest number of holders a slot has had at once).
    std::vector<std::vector<cudaEvent_t>> released;
    std::vector<Slot> slots;
    std::unordered_map<int, std::pair<const void*, size_t>> blobs;
    cudaEvent_t t0[kTimingRing] = {}, t1[kTimingRing] = {};
    int timing_next = 0, timing_live = 0;
    uint64_t tick = 0;
    lsn_pool_stats stats = {};
    int fault = LSN_POOL_FAULT_NONE;
    int debug = 0;                                    // LSN_POOL_DEBUG_* flags
    std::unordered_map<int, std::vector<int>> held;   // layer -> slots acquired for it
    std::mutex mu;
};

namespace {

struct DeviceGuard {
    int prev = -1;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        if (prev != dev) cudaSetDevice(dev);
    }
    ~DeviceGuard() {
        int cur;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

// Add the device time of finished copies to the counters (oldest first).
void harvest_timing(lsn_pool* p, bool block) {
    while (p->timing_live > 0) {
        const int idx = (p->timing_next - p->timing_live + kTimingRing) % kTimingRing;
        if (block) cudaEventSynchronize(p->t1[idx]);
        else if (cudaEventQuery(p->t1[idx]) != cudaSuccess) break;
        float ms = 0.0f;
        if (cudaEventElapsedTime(&ms, p->t0[idx], p->t1[idx]) == cudaSuccess) p->stats.copy_ms += ms;
        --p->timing_live;
    }
}

int find_slot(lsn_pool* p, int layer) {
    for (int s = 0; s < p->n_slots; ++s)
        if (p->slots[s].layer == layer) return s;
    return -1;
}

lsn_status start_copy(lsn_pool* p, int layer, int* slot_out) {
    lsn::NvtxRange nvtx("layer_pool copy");
    auto it = p->blobs.find(layer);
    if (it == p->blobs.end()) return lsn::fail(LSN_ERR_INVALID_ARG, "layer " + std::to_string(layer) + " is not registered");
    int best = -1;
    for (int s = 0; s < p->n_slots; ++s) {
        const Slot& sl = p->slots[s];
        if (sl.refs > 0 || sl.pending) continue;
        if (best < 0 || sl.last_release < p->slots[best].last_release ||
            (sl.last_release == p->slots[best].last_release && sl.layer < 0 && p->slots[best].layer >= 0))
            best = s;
    }
    if (best < 0) return lsn::fail(LSN_ERR_STATE, "layer pool: every slot is acquired or holds a prefetched layer");
    if (p->fault == LSN_POOL_FAULT_COPY_ERROR) {
        p->fault = LSN_POOL_FAULT_NONE;
        return lsn::fail(LSN_ERR_CUDA, "layer pool: injected copy failure");
    }
    Slot& sl = p->slots[best];
    uint8_t* dst = p->dev + (size_t)best * p->slot_stride;
    for (int i = 0; i < sl.n_rel; ++i) LSN_CUDA_TRY(cudaStreamWaitEvent(p->copy, p->released[best][i], 0));
    sl.n_rel = 0;
    if (p->timing_live == kTimingRing) harvest_timing(p, true);
    const int ti = p->timing_next;
    LSN_CUDA_TRY(cudaEventRecord(p->t0[ti], p->copy));
    // Debugging aid: the slot holds a sentinel from its release until the copy lands.
    if (p->debug & LSN_POOL_DEBUG_POISON) LSN_CUDA_TRY(cudaMemsetAsync(dst, 0xFF, p->slot_bytes, p->copy));
    // Planted defect (test hook): a reused slot is relabelled without its copy.
    const bool stale = p->fault == LSN_POOL_FAULT_STALE_SLOT && sl.layer >= 0;
    if (!stale)
        LSN_CUDA_TRY(cudaMemcpyAsync(dst, it->second.first, it->second.second, cudaMemcpyHostToDevice, p->copy));
    LSN_CUDA_TRY(cudaEventRecord(p->ready[best], p->copy));
    LSN_CUDA_TRY(cudaEventRecord(p->t1[ti], p->copy));
    p->timing_next = (ti + 1) % kTimingRing;
    ++p->timing_live;
    sl.layer = layer;
    sl.pending = true;
    sl.last_fill = ++p->tick;
    p->stats.copies += 1;
    p->stats.bytes_copied += it->second.second;
    *slot_out = best;
    return LSN_OK;
}

void destroy_resources(lsn_pool* p) {
    if (p->copy) cudaStreamSynchronize(p->copy);
    for (auto e : p->ready) if (e) cudaEventDestroy(e);
    for (auto& v : p->released)
        for (auto e : v) if (e) cudaEventDestroy(e);
    for (int i = 0; i < kTimingRing; ++i) {
        if (p->t0[i]) cudaEventDestroy(p->t0[i]);
        if (p->t1[i]) cudaEventDestroy(p->t1[i]);
    }
    if (p->copy) cudaStreamDestroy(p->copy);
    if (p->dev) cudaFree(p->dev);
}

}  // namespace

extern "C" {

lsn_status layer_pool_create(int n_slots, size_t slot_bytes, int device, lsn_pool** out) {
    LSN_CHECK_ARG(out != nullptr, "layer_pool_create: out is NULL");
    *out = nullptr;
    LSN_CHECK_ARG(n_slots >= 1 && n_slots <= 64, "layer_pool_create: n_slots must be in [1, 64]");
    LSN_CHECK_ARG(slot_bytes > 0, "layer_pool_create: slot_bytes must be > 0");
    int ndev = 0;
    LSN_CUDA_TRY(cudaGetDeviceCount(&ndev));
    LSN_CHECK_ARG(device >= 0 && device < ndev, "layer_pool_create: no such device");
    DeviceGuard g(device);
    lsn_pool* p = new lsn_pool();
    p->device = device;
    p->n_slots = n_slots;
    p->slot_bytes = slot_bytes;
    p->slot_stride = lsn::round_up(slot_bytes, 1024);
    cudaError_t e = cudaMalloc(&p->dev, p->slot_stride * (size_t)n_slots);
    if (e != cudaSuccess) {
        p->dev = nullptr;
        destroy_resources(p);
        delete p;
        cudaGetLastError();
        return lsn::fail(LSN_ERR_NO_MEMORY, "layer_pool_create: cannot allocate the slots");
    }
    bool ok = cudaStreamCreateWithFlags(&p->copy, cudaStreamNonBlocking) == cudaSuccess;
    p->ready.assign(n_slots, nullptr);
    p->released.assign(n_slots, {});
    for (int s = 0; ok && s < n_slots; ++s) {
        p->released[s].push_back(nullptr);
        ok = cudaEventCreateWithFlags(&p->ready[s], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&p->released[s][0], cudaEventDisableTiming) == cudaSuccess;
    }
    for (int i = 0; ok && i < kTimingRing; ++i)
        ok = cudaEventCreate(&p->t0[i]) == cudaSuccess && cudaEventCreate(&p->t1[i]) == cudaSuccess;
    if (!ok) {
        destroy_resources(p);
        delete p;
        return lsn::fail(LSN_ERR_CUDA, "layer_pool_create: stream/event creation failed");
    }
    p->slots.assign(n_slots, Slot());
    *out = p;
    return LSN_OK;
}

lsn_status layer_pool_register(lsn_pool* p, int layer, const void* host, size_t bytes) {
    LSN_CHECK_ARG(p != nullptr, "layer_pool_register: pool is NULL");
    LSN_CHECK_ARG(layer >= 0 && layer < 65536, "layer_pool_register: layer out of range");
    LSN_CHECK_ARG(host != nullptr && bytes > 0, "layer_pool_register: empty blob");
    LSN_CHECK_ARG(bytes <= p->slot_bytes, "layer_pool_register: blob larger than a slot");
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, host) != cudaSuccess || attr.type != cudaMemoryTypeHost) {
        cudaGetLastError();
        return lsn::fail(LSN_ERR_INVALID_ARG, "layer_pool_register: host blob is not page-locked (pinned) memory");
    }
    std::lock_guard<std::mutex> lk(p->mu);
    const int s = find_slot(p, layer);
    if (s >= 0) {
        if (p->slots[s].refs > 0) return lsn::fail(LSN_ERR_STATE, "layer_pool_register: layer is acquired");
        p->slots[s].layer = -1;
        p->slots[s].pending = false;
    }
    p->blobs[layer] = {host, bytes};
    return LSN_OK;
}

lsn_status layer_pool_prefetch(lsn_pool* p, int layer) {
    LSN_CHECK_ARG(p != nullptr, "layer_pool_prefetch: pool is NULL");
    std::lock_guard<std::mutex> lk(p->mu);
    const int s = find_slot(p, layer);
    if (s >= 0) {                        // resident: keep it there until it is acquired
        p->stats.hits += 1;
        if (p->slots[s].refs == 0) p->slots[s].pending = true;
        return LSN_OK;
    }
    DeviceGuard g(p->device);
    int slot;
    return start_copy(p, layer, &slot);
}

lsn_status layer_pool_acquire(lsn_pool* p, int layer, lsn_stream_t compute, void** dev_ptr) {
    LSN_CHECK_ARG(p != nullptr && dev_ptr != nullptr, "layer_pool_acquire: NULL argument");
    std::lock_guard<std::mutex> lk(p->mu);
    DeviceGuard g(p->device);
    int s = find_slot(p, layer);
    if (s < 0) {
        if (p->blobs.find(layer) == p->blobs.end())
            return lsn::fail(LSN_ERR_INVALID_ARG, "layer_pool_acquire: layer " + std::to_string(layer) + " is not registered");
        lsn_status st = start_copy(p, layer, &s);
        if (st != LSN_OK) return st;
        p->stats.misses += 1;
    } else {
        p->stats.hits += 1;
    }
    Slot& sl = p->slots[s];
    LSN_CUDA_TRY(cudaStreamWaitEvent(reinterpret_cast<cudaStream_t>(compute), p->ready[s], 0));
    sl.pending = false;
    sl.refs += 1;
    p->held[layer].push_back(s);
    *dev_ptr = p->dev + (size_t)s * p->slot_stride;
    return LSN_OK;
}

lsn_status layer_pool_release(lsn_pool* p, int layer, lsn_stream_t compute) {
    LSN_CHECK_ARG(p != nullptr, "layer_pool_release: pool is NULL");
    std::lock_guard<std::mutex> lk(p->mu);
    auto it = p->held.find(layer);
    if (it == p->held.end() || it->second.empty())
        return lsn::fail(LSN_ERR_STATE, "layer_pool_release: layer " + std::to_string(layer) + " is not acquired");
    const int s = it->second.back();
    DeviceGuard g(p->device);
    Slot& sl = p->slots[s];
    std::vector<cudaEvent_t>& ev = p->released[s];
    if (sl.n_rel == (int)ev.size()) {               // more holders than ever before: one more event
        cudaEvent_t e = nullptr;
        LSN_CUDA_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
        ev.push_back(e);
    }
    LSN_CUDA_TRY(cudaEventRecord(ev[sl.n_rel], reinterpret_cast<cudaStream_t>(compute)));
    it->second.pop_back();
    sl.n_rel += 1;
    sl.refs -= 1;
    sl.last_release = ++p->tick;
    return LSN_OK;
}

lsn_status layer_pool_wait_idle(lsn_pool* p, int timeout_ms) {
    LSN_CHECK_ARG(p != nullptr, "layer_pool_wait_idle: pool is NULL");
    DeviceGuard g(p->device);
    const auto t_end = std::chrono::steady_clock::now() + std::chrono::milliseconds(timeout_ms < 0 ? 0 : timeout_ms);
    while (true) {
        cudaError_t e = cudaStreamQuery(p->copy);
        if (e == cudaSuccess) return LSN_OK;
        if (e != cudaErrorNotReady) return lsn::fail_cuda(e, "layer_pool_wait_idle");
        if (std::chrono::steady_clock::now() >= t_end)
            return lsn::fail(LSN_ERR_TIMEOUT, "layer_pool_wait_idle: copies still running after the time limit");
        std::this_thread::sleep_for(std::chrono::microseconds(50));
    }
}

lsn_status layer_pool_stats(lsn_pool* p, lsn_pool_stats* out) {
    LSN_CHECK_ARG(p != nullptr && out != nullptr, "layer_pool_stats: NULL argument");
    std::lock_guard<std::mutex> lk(p->mu);
    DeviceGuard g(p->device);
    harvest_timing(p, false);
    *out = p->stats;
    return LSN_OK;
}

lsn_status layer_pool_reset(lsn_pool* p) {
    LSN_CHECK_ARG(p != nullptr, "layer_pool_reset: pool is NULL");
    lsn_status st = layer_pool_wait_idle(p, 10000);
    if (st != LSN_OK) return st;
    std::lock_guard<std::mutex> lk(p->mu);
    for (auto& sl : p->slots) {
        if (sl.refs > 0) return lsn::fail(LSN_ERR_STATE, "layer_pool_reset: a slot is still acquired");
    }
    DeviceGuard g(p->device);
    harvest_timing(p, true);
    for (auto& sl : p->slots) { sl.layer = -1; sl.pending = false; }
    p->stats = lsn_pool_stats();
    p->fault = LSN_POOL_FAULT_NONE;
    return LSN_OK;
}

lsn_status layer_pool_inject_fault(lsn_pool* p, int fault) {
    LSN_CHECK_ARG(p != nullptr, "layer_pool_inject_fault: pool is NULL");
    LSN_CHECK_ARG(fault >= LSN_POOL_FAULT_NONE && fault <= LSN_POOL_FAULT_COPY_ERROR, "layer_pool_inject_fault: unknown fault");
    std::lock_guard<std::mutex> lk(p->mu);
    p->fault = fault;
    return LSN_OK;
}

lsn_status layer_pool_set_debug(lsn_pool* p, int flags) {
    LSN_CHECK_ARG(p != nullptr, "layer_pool_set_debug: pool is NULL");
    LSN_CHECK_ARG((flags & ~LSN_POOL_DEBUG_POISON) == 0, "layer_pool_set_debug: unknown flag bits");
    std::lock_guard<std::mutex> lk(p->mu);
    p->debug = flags;
    return LSN_OK;
}

void layer_pool_destroy(lsn_pool* p) {
    if (!p) return;
    {
        DeviceGuard g(p->device);
        destroy_resources(p);
    }
    delete p;
}

}  // extern "C"
