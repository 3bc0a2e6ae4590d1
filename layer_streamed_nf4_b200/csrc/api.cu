// The C entry points of liblsnf4.so (declared in include/lsnf4.h): argument
// checks, workspace carving and the launch sequence of each call.
#include <cstring>
#include <atomic>
#include <mutex>
#include <string>

#include "common.cuh"
#include "launch.cuh"
#include "timing.cuh"

namespace lsn {


namespace {
thread_local std::string g_last_error = "no error";
std::atomic<int> g_fused_nf4{0};
std::atomic<int> g_layer_lanes{2};
std::atomic<int> g_pdl{1};
}

lsn_status fail(lsn_status st, const std::string& msg) {
    g_last_error = msg;
    return st;
}

lsn_status fail_cuda(cudaError_t e, const char* what) {
    g_last_error = std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
    return LSN_ERR_CUDA;
}

bool pdl_enabled() { return g_pdl.load() != 0; }

int sm_count() {
    int dev = 0;
    cudaGetDevice(&dev);
    static int cache[64] = {0};
    if (dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

bool device_is_sm100() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    return major == 10 && minor == 0;
}

}  // namespace lsn

using namespace lsn;

namespace lsn {

lsn_status check_device() {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
    if (!device_is_sm100()) return fail(LSN_ERR_UNSUPPORTED, "liblsnf4 is built for sm_100a (B200) only");
    return LSN_OK;
}

lsn_status check_nf4(const lsn_nf4_weight* w, const char* who) {
    const std::string f(who);
    LSN_CHECK_ARG(w != nullptr, f + ": weight is NULL");
    LSN_CHECK_ARG(w->rows >= 0 && w->cols >= 0, f + ": negative shape");
    LSN_CHECK_ARG(w->cols % 64 == 0, f + ": cols must be a multiple of 64");
    // rows * cols is formed only once it is known to fit (at most 2^46 elements).
    LSN_CHECK_ARG(w->cols == 0 || w->rows <= kMaxNf4Elems / w->cols, f + ": rows * cols too large");
    if (w->rows * w->cols == 0) return LSN_OK;
    LSN_CHECK_ARG(w->packed && w->absmax_q && w->absmax_s2 && w->offset, f + ": NULL array in the NF4 weight");
    LSN_CHECK_ARG(aligned16(w->packed), f + ": packed must be 16-byte aligned");
    LSN_CHECK_ARG((reinterpret_cast<uintptr_t>(w->absmax_s2) & 3) == 0 && (reinterpret_cast<uintptr_t>(w->offset) & 3) == 0,
                  f + ": absmax_s2/offset must be 4-byte aligned");
    return LSN_OK;
}

}  // namespace lsn

namespace {

// Workspace layout of the LoRA calls (each region 256-byte aligned):
//   [0, 256)  status word of the GEMM kernels
//   split     stream-K scratch of the GEMM (arrival counters, partial tiles)
//   u32  fp32 [T, r]     x A^T
//   g32  fp32 [T, r]     dY B
//   s16  bf16 [T, r]     bf16(s u) or bf16(s g)
//   w16  bf16 [N, K]     dequantised base (NF4 base only)
// The status word and the stream-K counters must be zero when the workspace
// is first used: fill the workspace with zeros once, when it is allocated.
struct LoraWs {
    int* err;
    GemmSplitWs split;
    float* u32;
    float* g32;
    uint16_t* s16;
    uint16_t* w16;
    size_t total;
};

LoraWs carve(void* ws, int64_t T, int64_t K, int64_t N, int r, int kind) {
    LoraWs w;
    size_t off = 0;
    char* b = reinterpret_cast<char*>(ws);
    auto take = [&](size_t bytes) { char* p = b ? b + off : nullptr; off += round_up(bytes, 256); return p; };
    w.err = reinterpret_cast<int*>(take(256));
    w.split = gemm_split_ws(take(gemm_split_ws_bytes()));
    w.u32 = reinterpret_cast<float*>(take((size_t)T * r * 4));
    w.g32 = reinterpret_cast<float*>(take((size_t)T * r * 4));
    w.s16 = reinterpret_cast<uint16_t*>(take((size_t)T * r * 2));
    w.w16 = reinterpret_cast<uint16_t*>(take(kind == LSN_BASE_NF4 ? (size_t)N * K * 2 : 0));
    w.total = off;
    return w;
}

lsn_status check_proj(const lsn_base* W, const uint16_t* x, int64_t T, const uint16_t* A, const uint16_t* B, int r,
                      const std::string& f, bool adapter_may_be_off = false) {
    LSN_CHECK_ARG(W != nullptr, f + ": base is NULL");
    LSN_CHECK_ARG(W->kind == LSN_BASE_NF4 || W->kind == LSN_BASE_BF16, f + ": unknown base kind");
    LSN_CHECK_ARG(T >= 0, f + ": T must be >= 0");
    LSN_CHECK_ARG(W->rows > 0 && W->cols > 0, f + ": empty base weight");
    LSN_CHECK_ARG(W->rows % 64 == 0 && W->cols % 64 == 0, f + ": N and K must be multiples of 64");
    LSN_CHECK_ARG(W->rows <= (int64_t)1 << 30 && W->cols <= (int64_t)1 << 30 && T <= (int64_t)1 << 30,
                  f + ": dimension too large");
    LSN_CHECK_ARG(r >= 8 && r <= 64 && r % 8 == 0, f + ": rank must be a multiple of 8 in [8, 64]");
    if (W->kind == LSN_BASE_NF4) {
        lsn_status s = check_nf4(&W->nf4, f.c_str());
        if (s != LSN_OK) return s;
        LSN_CHECK_ARG(W->nf4.rows == W->rows && W->nf4.cols == W->cols, f + ": NF4 weight shape differs from the base shape");
    } else {
        LSN_CHECK_ARG(W->bf16 != nullptr && aligned16(W->bf16), f + ": bf16 base must be a 16-byte aligned pointer");
    }
    const bool off = adapter_may_be_off && A == nullptr && B == nullptr;
    LSN_CHECK_ARG((x || T == 0) && ((A && B) || off), f + ": NULL tensor");
    LSN_CHECK_ARG(aligned16(x) && aligned16(A) && aligned16(B), f + ": tensors must be 16-byte aligned");
    return LSN_OK;
}

lsn_status check_lora(const lsn_base* W, const uint16_t* x, int64_t T, const uint16_t* A, const uint16_t* B, int r,
                      void* ws, size_t ws_bytes, const char* who) {
    const std::string f(who);
    lsn_status s = check_proj(W, x, T, A, B, r, f);
    if (s != LSN_OK) return s;
    LSN_CHECK_ARG(ws != nullptr && aligned16(ws), f + ": workspace must be a 16-byte aligned device pointer");
    const size_t need = carve(nullptr, T, W->cols, W->rows, r, W->kind).total;
    LSN_CHECK_ARG(ws_bytes >= need, f + ": workspace too small (need " + std::to_string(need) + " bytes)");
    return LSN_OK;
}

double dequant_bytes(int64_t N, int64_t K) {
    const double n = (double)N * (double)K;
    return n / 2.0 + n / 64.0 + 4.0 * (double)((N * K / 64 + 255) / 256) + 4.0 + 2.0 * n;
}

// Workspace of the layer calls: the status word, the stream-K scratch of the
// two lanes' GEMMs, then per projection i
//   s16 bf16 [T, r]  bf16(s u_i) (forward) or bf16(s g_i) (backward)
//   g32 fp32 [T, r]  dY_i B_i
//   u32 fp32 [T, r]  x_i A_i^T when the caller keeps no u
// then per group (led by its first member g):
//   la  bf16 [T, m r]        the members' bf16(s u) or bf16(s g), side by side
//   lb  bf16 [N_sum, m r]    forward: block-diagonal of the members' B
//       bf16 [m r, K]        backward: the members' A stacked
// and last, back to back in projection order (so a group's stack is one
// matrix):
//   w16 bf16 [N, K]  dequantised base (NF4 bases only)

// The groups of a layer call: group k spans projections first[k] ..
// first[k] + count[k] - 1 (ungrouped projections are groups of one).
struct Groups {
    int n = 0;
    int first[LSN_LAYER_MAX_PROJ];
    int count[LSN_LAYER_MAX_PROJ];
};

Groups find_groups(int n, const lsn_lora_proj* p) {
    Groups g;
    for (int i = 0; i < n;) {
        int j = i + 1;
        if (p[i].group > 0)
            while (j < n && p[j].group == p[i].group && j - i < kGemmMaxSeg) ++j;
        g.first[g.n] = i;
        g.count[g.n++] = j - i;
        i = j;
    }
    return g;
}

struct LayerWs {
    int* err;
    GemmSplitWs split[2];               // stream-K scratch of the GEMMs on the main and the side lane
    uint16_t* s16[LSN_LAYER_MAX_PROJ];
    float* g32[LSN_LAYER_MAX_PROJ];
    float* u32[LSN_LAYER_MAX_PROJ];
    uint16_t* w16[LSN_LAYER_MAX_PROJ];
    uint16_t* la[LSN_LAYER_MAX_PROJ];   // per group leader
    uint16_t* lb[LSN_LAYER_MAX_PROJ];   // per group leader
    size_t total;
};

LayerWs carve_layer(void* ws, int n, const lsn_lora_proj* p, int64_t T, int r) {
    LayerWs w{};
    size_t off = 0;
    char* b = reinterpret_cast<char*>(ws);
    auto take = [&](size_t bytes) { char* q = b ? b + off : nullptr; off += round_up(bytes, 256); return q; };
    w.err = reinterpret_cast<int*>(take(256));
    for (auto& sp : w.split) sp = gemm_split_ws(take(gemm_split_ws_bytes()));
    for (int i = 0; i < n; ++i) {
        w.s16[i] = reinterpret_cast<uint16_t*>(take((size_t)T * r * 2));
        w.g32[i] = reinterpret_cast<float*>(take((size_t)T * r * 4));
        w.u32[i] = reinterpret_cast<float*>(take((size_t)T * r * 4));
    }
    const Groups g = find_groups(n, p);
    for (int k = 0; k < g.n; ++k) {
        if (g.count[k] < 2) continue;
        const int i0 = g.first[k], m = g.count[k];
        int64_t nsum = 0;
        for (int j = 0; j < m; ++j) nsum += p[i0 + j].W.rows;
        const int64_t K = p[i0].W.cols;
        w.la[i0] = reinterpret_cast<uint16_t*>(take((size_t)T * m * r * 2));
        const int64_t lb_elems = nsum * m * r > (int64_t)m * r * K ? nsum * m * r : (int64_t)m * r * K;
        w.lb[i0] = reinterpret_cast<uint16_t*>(take((size_t)lb_elems * 2));
    }
    for (int i = 0; i < n; ++i) {
        const bool nf4 = p[i].W.kind == LSN_BASE_NF4;
        w.w16[i] = reinterpret_cast<uint16_t*>(take(nf4 ? (size_t)p[i].W.rows * p[i].W.cols * 2 : 0));
    }
    w.total = off;
    return w;
}

bool adapter_off(const lsn_lora_proj& q) { return q.A == nullptr && q.B == nullptr; }

lsn_status check_layer(int n, const lsn_lora_proj* p, int64_t T, int r, void* ws, size_t ws_bytes, bool bwd,
                       const char* who) {
    const std::string f(who);
    LSN_CHECK_ARG(n >= 1 && n <= LSN_LAYER_MAX_PROJ, f + ": n must be in [1, LSN_LAYER_MAX_PROJ]");
    LSN_CHECK_ARG(p != nullptr, f + ": projection array is NULL");
    for (int i = 0; i < n; ++i) {
        const std::string fi = f + ": projection " + std::to_string(i);
        lsn_status s = check_proj(&p[i].W, p[i].x, T, p[i].A, p[i].B, r, fi, true);
        if (s != LSN_OK) return s;
        LSN_CHECK_ARG(aligned16(p[i].u), fi + ": u must be 16-byte aligned");
        if (!bwd) {
            LSN_CHECK_ARG((p[i].y != nullptr || T == 0) && aligned16(p[i].y), fi + ": y must be a 16-byte aligned device pointer");
        } else {
            LSN_CHECK_ARG((p[i].dY != nullptr || T == 0) && aligned16(p[i].dY), fi + ": dY must be a 16-byte aligned device pointer");
            LSN_CHECK_ARG(adapter_off(p[i]) || (p[i].dA && p[i].dB && aligned16(p[i].dA) && aligned16(p[i].dB)),
                          fi + ": dA/dB must be 16-byte aligned device pointers");
            LSN_CHECK_ARG(aligned16(p[i].dX), fi + ": dX must be 16-byte aligned");
        }
    }
    const Groups g = find_groups(n, p);
    for (int k = 0; k < g.n; ++k) {
        const int i0 = g.first[k], m = g.count[k];
        if (m < 2) continue;
        const std::string fg = f + ": group of projections " + std::to_string(i0) + ".." + std::to_string(i0 + m - 1);
        LSN_CHECK_ARG(m * r <= 64, fg + ": group size x rank must be <= 64");
        for (int j = 1; j < m; ++j) {
            const lsn_lora_proj& a = p[i0 + j - 1];
            const lsn_lora_proj& q = p[i0 + j];
            LSN_CHECK_ARG(q.x == p[i0].x && q.W.cols == p[i0].W.cols && q.W.kind == p[i0].W.kind &&
                              adapter_off(q) == adapter_off(p[i0]),
                          fg + ": members must share x, K, base kind and adapter state");
            if (q.W.kind == LSN_BASE_BF16)
                LSN_CHECK_ARG(q.W.bf16 == a.W.bf16 + a.W.rows * a.W.cols,
                              fg + ": bf16 bases of a group must lie back to back");
            if (bwd) LSN_CHECK_ARG(q.dX == nullptr, fg + ": only the first member has a dX (the group's sum)");
        }
        for (int j = 0; j + 1 < m && bwd; ++j)
            LSN_CHECK_ARG(p[i0 + j].W.rows % 128 == 0, fg + ": N of all but the last member must be a multiple of 128");
    }
    LSN_CHECK_ARG(ws != nullptr && aligned16(ws), f + ": workspace must be a 16-byte aligned device pointer");
    const size_t need = carve_layer(nullptr, n, p, T, r).total;
    LSN_CHECK_ARG(ws_bytes >= need, f + ": workspace too small (need " + std::to_string(need) + " bytes)");
    return LSN_OK;
}

// NF4 conversion inside the GEMM (LSN_OPT_FUSED_NF4): 1 = converter warps
// writing the bf16 tile into shared memory (both directions, 2-SM shapes);
// 2 = converter warps writing W into tensor memory (forward only, shapes
// with at least a wave of 256 x 256 tiles).
bool fused_here(const lsn_base& W, int64_t M, int64_t N) {
    return W.kind == LSN_BASE_NF4 && g_fused_nf4.load() == 1 && gemm_use_pairs(M, N);
}
bool fused_tmem_fwd(const lsn_base& W, int64_t T) {
    return W.kind == LSN_BASE_NF4 && g_fused_nf4.load() == 2 && gemm_nf4t_supported(T, W.rows, W.cols);
}

// Dequantise the NF4 bases of the listed projections into their workspace copies, one launch.
lsn_status layer_dequant(int n, const lsn_lora_proj* p, const bool* want, const LayerWs& w, cudaStream_t st) {
    const lsn_nf4_weight* ws[LSN_LAYER_MAX_PROJ];
    uint16_t* outs[LSN_LAYER_MAX_PROJ];
    int m = 0;
    double bytes = 0.0;
    for (int i = 0; i < n; ++i) {
        if (!want[i]) continue;
        ws[m] = &p[i].W.nf4;
        outs[m++] = w.w16[i];
        bytes += dequant_bytes(p[i].W.rows, p[i].W.cols);
    }
    if (m == 0) return LSN_OK;
    TimingScope ts(LSN_K_DEQUANT, bytes, st);
    return launch_dequant_batch(m, ws, outs, st);
}

lsn_status timed_down_batch(int n, const DownSpec* d, bool w_rk, int r, cudaStream_t st) {
    if (n == 0) return LSN_OK;
    double bytes = 0.0;
    for (int i = 0; i < n; ++i)
        bytes += 2.0 * d[i].T * d[i].Kd + 2.0 * r * d[i].Kd + (d[i].u32 ? 4.0 * d[i].T * r : 0.0) +
                 (d[i].u16 ? 2.0 * d[i].T * r : 0.0);
    TimingScope ts(LSN_K_LORA_DOWN, bytes, st, 1);
    return launch_lora_down_batch(n, d, w_rk, r, st);
}

lsn_status timed_tgrad_batch(int n, const TgSpec* d, int r, cudaStream_t st) {
    if (n == 0) return LSN_OK;
    double bytes = 0.0;
    for (int i = 0; i < n; ++i)
        bytes += 2.0 * d[i].T * d[i].Kd + 4.0 * d[i].T * r + 4.0 * r * d[i].Kd * (d[i].accumulate ? 2.0 : 1.0);
    TimingScope ts(LSN_K_LORA_TGRAD, bytes, st, 1);
    return launch_lora_tgrad_batch(n, d, r, st);
}

// The second stream of the layer calls (one per device, created on first
// use).  A call forks it from the caller's stream with an event, enqueues
// independent work on both, and makes the caller's stream wait for it again
// before returning.  The enqueue sequence of a call runs under `mu`, so calls
// from several host threads cannot interleave their fork/join events.
struct SideLane {
    cudaStream_t side = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr, mark = nullptr;
};
std::mutex g_side_mu;
SideLane g_side[64];

class LaneScope {
  public:
    // Forks the side stream from `st` when two lanes are wanted; otherwise
    // (or if the stream cannot be made) side() is `st` itself.
    LaneScope(cudaStream_t st, bool want) : st_(st), lk_(g_side_mu) {
        int dev = 0;
        if (!want || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return;
        SideLane& L = g_side[dev];
        if (!L.side) {
            if (cudaStreamCreateWithFlags(&L.side, cudaStreamNonBlocking) != cudaSuccess ||
                cudaEventCreateWithFlags(&L.fork, cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&L.join, cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&L.mark, cudaEventDisableTiming) != cudaSuccess) {
                L = SideLane{};
                return;
            }
        }
        if (cudaEventRecord(L.fork, st) != cudaSuccess || cudaStreamWaitEvent(L.side, L.fork, 0) != cudaSuccess) return;
        lane_ = &L;
    }
    cudaStream_t main() const { return st_; }
    bool two() const { return lane_ != nullptr; }
    cudaStream_t side() const { return lane_ ? lane_->side : st_; }
    // Both lanes continue only after everything enqueued so far on either.
    lsn_status barrier() {
        if (!lane_) return LSN_OK;
        LSN_CUDA_TRY(cudaEventRecord(lane_->fork, st_));
        LSN_CUDA_TRY(cudaEventRecord(lane_->join, lane_->side));
        LSN_CUDA_TRY(cudaStreamWaitEvent(st_, lane_->join, 0));
        LSN_CUDA_TRY(cudaStreamWaitEvent(lane_->side, lane_->fork, 0));
        return LSN_OK;
    }
    // One-way orderings: one lane waits for what the other has enqueued so far.
    lsn_status main_waits_side() {
        if (!lane_) return LSN_OK;
        LSN_CUDA_TRY(cudaEventRecord(lane_->join, lane_->side));
        LSN_CUDA_TRY(cudaStreamWaitEvent(st_, lane_->join, 0));
        return LSN_OK;
    }
    // A point on the side lane that the main lane can wait for later.
    lsn_status mark_side() {
        if (!lane_) return LSN_OK;
        LSN_CUDA_TRY(cudaEventRecord(lane_->mark, lane_->side));
        return LSN_OK;
    }
    lsn_status main_waits_mark() {
        if (!lane_) return LSN_OK;
        LSN_CUDA_TRY(cudaStreamWaitEvent(st_, lane_->mark, 0));
        return LSN_OK;
    }
    lsn_status side_waits_main() {
        if (!lane_) return LSN_OK;
        LSN_CUDA_TRY(cudaEventRecord(lane_->fork, st_));
        LSN_CUDA_TRY(cudaStreamWaitEvent(lane_->side, lane_->fork, 0));
        return LSN_OK;
    }
    // Join: the caller's stream waits for everything enqueued on the side stream.
    lsn_status join() {
        if (!lane_) return LSN_OK;
        SideLane* L = lane_;
        lane_ = nullptr;
        LSN_CUDA_TRY(cudaEventRecord(L->join, L->side));
        LSN_CUDA_TRY(cudaStreamWaitEvent(st_, L->join, 0));
        return LSN_OK;
    }
    ~LaneScope() { join(); }

  private:
    cudaStream_t st_;
    std::lock_guard<std::mutex> lk_;
    SideLane* lane_ = nullptr;
};

lsn_status timed_dequant(const lsn_nf4_weight* w, uint16_t* out, cudaStream_t st) {
    TimingScope ts(LSN_K_DEQUANT, dequant_bytes(w->rows, w->cols), st);
    return launch_dequant(w, out, st);
}

lsn_status timed_down(const uint16_t* X, const uint16_t* W, bool w_rk, int64_t T, int64_t Kd, int r, float scale,
                      float* u32, uint16_t* u16, const LoraWs& w, cudaStream_t st) {
    const double bytes = 2.0 * T * Kd + 2.0 * r * Kd + (u32 ? 4.0 * T * r : 0.0) + (u16 ? 2.0 * T * r : 0.0);
    TimingScope ts(LSN_K_LORA_DOWN, bytes, st, 1);
    return launch_lora_down(X, W, w_rk, T, Kd, r, scale, u32, u16, st);
}

lsn_status timed_tgrad(const float* G, const uint16_t* X, bool out_rk, int64_t T, int64_t Kd, int r, float scale,
                       int accumulate, float* out, const LoraWs& w, cudaStream_t st) {
    const double bytes = 2.0 * T * Kd + 4.0 * T * r + 4.0 * r * Kd * (accumulate ? 2.0 : 1.0);
    TimingScope ts(LSN_K_LORA_TGRAD, bytes, st, 1);
    return launch_lora_tgrad(G, X, out_rk, T, Kd, r, scale, accumulate, out, st);
}

lsn_status timed_gemm(int kind, const uint16_t* A, int64_t lda, const uint16_t* B, int64_t ldb, bool b_mn,
                      const uint16_t* LA, const uint16_t* LB, int r, int64_t M, int64_t N, int64_t Kc, uint16_t* D,
                      int64_t ldd, int* err, cudaStream_t st, const GemmSplitWs* split) {
    TimingScope ts(kind, 2.0 * M * N * (double)(Kc + r), st);
    return launch_gemm(A, lda, B, ldb, b_mn, LA, LB, r, M, N, Kc, D, ldd, err, st, split);
}

}  // namespace

extern "C" {

const char* lsn_last_error(void) { return g_last_error.c_str(); }

int lsn_version(void) { return 100; }

void lsn_nf4_codebook(float out[16]) { std::memcpy(out, nf4_tables().level, sizeof(float) * 16); }

void lsn_dq_codebook(float out[256]) { std::memcpy(out, nf4_tables().dq, sizeof(float) * 256); }

size_t lsn_nf4_packed_bytes(int64_t rows, int64_t cols) { return (size_t)(rows * cols / 2); }
size_t lsn_nf4_absmax_bytes(int64_t rows, int64_t cols) { return (size_t)(rows * cols / 64); }
size_t lsn_nf4_s2_bytes(int64_t rows, int64_t cols) { return (size_t)((rows * cols / 64 + 255) / 256) * 4; }

void lsn_nf4_blob_layout(int64_t rows, int64_t cols, size_t out[4]) {
    size_t off = 0;
    out[0] = off;
    off += round_up(lsn_nf4_packed_bytes(rows, cols), 1024);
    out[1] = off;
    off += round_up(lsn_nf4_absmax_bytes(rows, cols), 1024);
    out[2] = off;
    off += round_up(lsn_nf4_s2_bytes(rows, cols), 1024);
    out[3] = off;
}

size_t lsn_nf4_blob_bytes(int64_t rows, int64_t cols) {
    size_t o[4];
    lsn_nf4_blob_layout(rows, cols, o);
    return o[3] + 1024;
}

size_t lsn_nf4_quantize_ws_bytes(int64_t rows, int64_t cols) { return quantize_ws_bytes(rows, cols); }

lsn_status nf4_quantize(const float* W, const lsn_nf4_weight* out, void* ws, size_t ws_bytes, lsn_stream_t stream) {
    NvtxRange nvtx("nf4_quantize");
    lsn_status s = check_nf4(out, "nf4_quantize");
    if (s != LSN_OK) return s;
    if (out->rows * out->cols == 0) return LSN_OK;
    LSN_CHECK_ARG(W != nullptr && aligned16(W), "nf4_quantize: W must be a 16-byte aligned device pointer");
    LSN_CHECK_ARG(ws != nullptr && aligned16(ws), "nf4_quantize: workspace must be 16-byte aligned");
    LSN_CHECK_ARG(ws_bytes >= quantize_ws_bytes(out->rows, out->cols), "nf4_quantize: workspace too small");
    if ((s = check_device()) != LSN_OK) return s;
    const double numel = (double)out->rows * (double)out->cols;
    TimingScope ts(LSN_K_QUANTIZE, numel * 4.0 + numel / 2.0 + numel / 64.0 * 6.0, reinterpret_cast<cudaStream_t>(stream),
                   4);
    return launch_quantize(W, out, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

lsn_status nf4_dequant(const lsn_nf4_weight* w, uint16_t* W_out, lsn_stream_t stream) {
    NvtxRange nvtx("nf4_dequant");
    lsn_status s = check_nf4(w, "nf4_dequant");
    if (s != LSN_OK) return s;
    if (w->rows * w->cols == 0) return LSN_OK;
    LSN_CHECK_ARG(W_out != nullptr && aligned16(W_out), "nf4_dequant: output must be a 16-byte aligned device pointer");
    if ((s = check_device()) != LSN_OK) return s;
    return timed_dequant(w, W_out, reinterpret_cast<cudaStream_t>(stream));
}

lsn_status nf4_dequant_batch(int n, const lsn_nf4_weight* w, uint16_t* const* W_out, int blocks_per_sm,
                             lsn_stream_t stream) {
    NvtxRange nvtx("nf4_dequant_batch");
    LSN_CHECK_ARG(n >= 0 && blocks_per_sm >= 0, "nf4_dequant_batch: n and blocks_per_sm must be >= 0");
    if (n == 0) return LSN_OK;
    LSN_CHECK_ARG(w != nullptr && W_out != nullptr, "nf4_dequant_batch: NULL array");
    const lsn_nf4_weight* ws[16];
    uint16_t* outs[16];
    double bytes = 0.0;
    for (int i = 0; i < n; ++i) {
        lsn_status s = check_nf4(&w[i], "nf4_dequant_batch");
        if (s != LSN_OK) return s;
        if (w[i].rows * w[i].cols != 0)
            LSN_CHECK_ARG(W_out[i] != nullptr && aligned16(W_out[i]),
                          "nf4_dequant_batch: outputs must be 16-byte aligned device pointers");
    }
    lsn_status s = check_device();
    if (s != LSN_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    for (int i0 = 0; i0 < n; i0 += 16) {
        const int m = n - i0 < 16 ? n - i0 : 16;
        bytes = 0.0;
        for (int j = 0; j < m; ++j) {
            ws[j] = &w[i0 + j];
            outs[j] = W_out[i0 + j];
            bytes += dequant_bytes(w[i0 + j].rows, w[i0 + j].cols);
        }
        TimingScope ts(LSN_K_DEQUANT, bytes, st);
        if ((s = launch_dequant_batch(m, ws, outs, st, blocks_per_sm)) != LSN_OK) return s;
    }
    return LSN_OK;
}

size_t lsn_lora_ws_bytes(int64_t T, int64_t K, int64_t N, int r, int kind) {
    return carve(nullptr, T, K, N, r, kind).total;
}

lsn_status lora_linear_fwd(const lsn_base* W, const uint16_t* x, int64_t T, const uint16_t* A, const uint16_t* B, int r,
                           float scale, uint16_t* y, void* ws, size_t ws_bytes, lsn_stream_t stream) {
    NvtxRange nvtx("lora_linear_fwd");
    lsn_status s = check_lora(W, x, T, A, B, r, ws, ws_bytes, "lora_linear_fwd");
    if (s != LSN_OK) return s;
    LSN_CHECK_ARG((y != nullptr || T == 0) && aligned16(y), "lora_linear_fwd: y must be a 16-byte aligned device pointer");
    if (T == 0) return LSN_OK;
    if ((s = check_device()) != LSN_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t N = W->rows, K = W->cols;
    LoraWs w = carve(ws, T, K, N, r, W->kind);
    if ((s = timed_down(x, A, true, T, K, r, scale, nullptr, w.s16, w, st)) != LSN_OK) return s;
    if (fused_tmem_fwd(*W, T)) {
        // NF4 converted straight into tensor memory (no bf16 copy of W).
        TimingScope ts(LSN_K_GEMM_FWD, 2.0 * T * N * (double)(K + r), st);
        return launch_gemm_nf4t(x, K, &W->nf4, w.s16, B, r, T, N, K, y, N, w.err, st);
    }
    if (fused_here(*W, T, N)) {
        // NF4 converted inside the GEMM (no bf16 copy of W).
        TimingScope ts(LSN_K_GEMM_FWD, 2.0 * T * N * (double)(K + r), st);
        return launch_gemm_nf4(x, K, &W->nf4, false, w.s16, B, r, T, N, K, y, N, w.err, st);
    }
    const uint16_t* Wb = W->bf16;
    if (W->kind == LSN_BASE_NF4) {
        if ((s = timed_dequant(&W->nf4, w.w16, st)) != LSN_OK) return s;
        Wb = w.w16;
    }
    return timed_gemm(LSN_K_GEMM_FWD, x, K, Wb, K, false, w.s16, B, r, T, N, K, y, N, w.err, st, &w.split);
}

lsn_status lora_linear_bwd(const lsn_base* W, const uint16_t* x, const uint16_t* dY, int64_t T, const uint16_t* A,
                           const uint16_t* B, int r, float scale, uint16_t* dX, float* dA, float* dB, int accumulate,
                           void* ws, size_t ws_bytes, lsn_stream_t stream) {
    NvtxRange nvtx("lora_linear_bwd");
    lsn_status s = check_lora(W, x, T, A, B, r, ws, ws_bytes, "lora_linear_bwd");
    if (s != LSN_OK) return s;
    LSN_CHECK_ARG((dY != nullptr || T == 0) && aligned16(dY), "lora_linear_bwd: dY must be a 16-byte aligned device pointer");
    LSN_CHECK_ARG(dA && dB && aligned16(dA) && aligned16(dB), "lora_linear_bwd: dA/dB must be 16-byte aligned device pointers");
    LSN_CHECK_ARG(dX == nullptr || aligned16(dX), "lora_linear_bwd: dX must be 16-byte aligned");
    if ((s = check_device()) != LSN_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t N = W->rows, K = W->cols;
    LoraWs w = carve(ws, T, K, N, r, W->kind);
    if (T > 0) {
        if ((s = timed_down(dY, B, false, T, N, r, scale, w.g32, w.s16, w, st)) != LSN_OK) return s;
        if ((s = timed_down(x, A, true, T, K, r, scale, w.u32, nullptr, w, st)) != LSN_OK) return s;
        if (dX && fused_here(*W, T, K)) {
            TimingScope ts(LSN_K_GEMM_BWD, 2.0 * T * K * (double)(N + r), st);
            if ((s = launch_gemm_nf4(dY, N, &W->nf4, true, w.s16, A, r, T, K, N, dX, K, w.err, st)) != LSN_OK) return s;
        } else if (dX) {
            const uint16_t* Wb = W->bf16;
            if (W->kind == LSN_BASE_NF4) {
                if ((s = timed_dequant(&W->nf4, w.w16, st)) != LSN_OK) return s;
                Wb = w.w16;
            }
            if ((s = timed_gemm(LSN_K_GEMM_BWD, dY, N, Wb, K, true, w.s16, A, r, T, K, N, dX, K, w.err, st, &w.split)) != LSN_OK)
                return s;
        }
    }
    // With T == 0 the reductions write zeros (or leave accumulators unchanged).
    if ((s = timed_tgrad(w.g32, x, true, T, K, r, scale, accumulate, dA, w, st)) != LSN_OK) return s;
    return timed_tgrad(w.u32, dY, false, T, N, r, scale, accumulate, dB, w, st);
}

size_t lsn_layer_ws_bytes(int n, const lsn_lora_proj* p, int64_t T, int r) {
    if (n < 1 || n > LSN_LAYER_MAX_PROJ || p == nullptr || T < 0 || r < 8 || r > 64 || r % 8 != 0) return 0;
    for (int i = 0; i < n; ++i)
        if (p[i].W.rows < 0 || p[i].W.cols < 0) return 0;
    return carve_layer(nullptr, n, p, T, r).total;
}

// The LoRA operand of a group's extra K-block, built on stream st:
// forward, the block-diagonal [N_sum, m r] of the members' B (member j's B in
// rows of its outputs, columns j r .. j r + r - 1, zeros elsewhere, so every
// output column gets exactly its own projection's s u B^T); backward, the
// members' A stacked into [m r, K].
lsn_status build_group_lb(const lsn_lora_proj* p, int i0, int m, int r, bool bwd, uint16_t* lb, cudaStream_t st) {
    const int64_t K = p[i0].W.cols;
    if (!bwd) {
        int64_t nsum = 0;
        for (int j = 0; j < m; ++j) nsum += p[i0 + j].W.rows;
        LSN_CUDA_TRY(cudaMemsetAsync(lb, 0, (size_t)nsum * m * r * 2, st));
        int64_t row = 0;
        for (int j = 0; j < m; ++j) {
            const int64_t N = p[i0 + j].W.rows;
            LSN_CUDA_TRY(cudaMemcpy2DAsync(lb + row * m * r + j * r, (size_t)m * r * 2, p[i0 + j].B, (size_t)r * 2,
                                           (size_t)r * 2, (size_t)N, cudaMemcpyDeviceToDevice, st));
            row += N;
        }
    } else {
        for (int j = 0; j < m; ++j)
            LSN_CUDA_TRY(cudaMemcpyAsync(lb + (int64_t)j * r * K, p[i0 + j].A, (size_t)r * K * 2,
                                         cudaMemcpyDeviceToDevice, st));
    }
    return LSN_OK;
}

// Whether projections 1..n-1 of an ungrouped layer call run as one merged
// GEMM launch (LSN_OPT_LAYER_MERGE): all with bf16 bases (and, backward, all
// asking for dX), at least two, and within the launch's problem and tile
// limits.
bool merge_rest(int n, const lsn_lora_proj* p, int64_t T, bool bwd) {
    // (The stream-K option asks for its own schedule of every GEMM: no merging.)
    if (!gemm_multi() || gemm_stream_k() || T <= 0 || n - 1 < 2 || n - 1 > gemm_multi_max_problems()) return false;
    GemmProblem pr[LSN_LAYER_MAX_PROJ];
    for (int i = 1; i < n; ++i) {
        if (p[i].W.kind != LSN_BASE_BF16 || (bwd && !p[i].dX)) return false;
        pr[i - 1].N = p[i].W.rows;
    }
    return gemm_multi_fits(pr, n - 1, T);
}

// The GEMMs of projections 1..n-1 as one launch: forward y = x W^T + (s u) B^T,
// backward dX = dY W + (s g) A.
lsn_status merged_gemms(int n, const lsn_lora_proj* p, int64_t T, int r, const LayerWs& w, bool bwd,
                        cudaStream_t st) {
    GemmProblem pr[LSN_LAYER_MAX_PROJ];
    double flop = 0.0;
    for (int i = 1; i < n; ++i) {
        GemmProblem& q = pr[i - 1];
        const int64_t N = p[i].W.rows, K = p[i].W.cols;
        const bool lora = !adapter_off(p[i]);
        q.B = p[i].W.bf16;
        q.ldb = K;
        q.LA = lora ? w.s16[i] : nullptr;
        if (!bwd) {
            q.A[0] = p[i].x;
            q.lda[0] = K;
            q.LB = p[i].B;
            q.N = N;
            q.Kc = K;
            q.D = p[i].y;
            q.ldd = N;
            flop += 2.0 * T * N * (double)(K + (lora ? r : 0));
        } else {
            q.A[0] = p[i].dY;
            q.lda[0] = N;
            q.LB = p[i].A;
            q.N = K;
            q.Kc = N;
            q.D = p[i].dX;
            q.ldd = K;
            flop += 2.0 * T * K * (double)(N + (lora ? r : 0));
        }
    }
    TimingScope ts(bwd ? LSN_K_GEMM_BWD : LSN_K_GEMM_FWD, flop, st);
    return launch_gemm_multi(pr, n - 1, bwd, T, r, w.err, st);
}

// A layer call with groups as one merged GEMM launch (LSN_OPT_LAYER_MERGE):
// forward, every projection is a problem of its own (a group's members share
// x; member j's bf16(s u) is column block j of the group's LoRA operand);
// backward, every group (or ungrouped projection) asking for dX is one
// problem whose contraction runs over its members' dY side by side, as in the
// grouped GEMM.  Returns false (nothing launched) when the call does not
// qualify: a base that is not bf16, the stream-K option, or more problems or
// tiles than one launch takes.
bool grouped_problems(int n, const lsn_lora_proj* p, const Groups& g, int64_t T, int r, const LayerWs& w, bool bwd,
                      GemmProblem* pr, int* np, double* flop) {
    if (!gemm_multi() || gemm_stream_k() || T <= 0) return false;
    for (int i = 0; i < n; ++i)
        if (p[i].W.kind != LSN_BASE_BF16) return false;
    int k = 0;
    double f = 0.0;
    for (int gi = 0; gi < g.n; ++gi) {
        const int i0 = g.first[gi], m = g.count[gi];
        const bool lora = !adapter_off(p[i0]);
        const int64_t K = p[i0].W.cols;
        if (!bwd) {
            for (int j = 0; j < m; ++j) {
                if (k == gemm_multi_max_problems()) return false;
                const int i = i0 + j;
                const int64_t N = p[i].W.rows;
                GemmProblem& q = pr[k++];
                q.A[0] = p[i].x;
                q.lda[0] = K;
                q.B = p[i].W.bf16;
                q.ldb = K;
                if (lora) {
                    q.LA = m > 1 ? w.la[i0] + (int64_t)j * r : w.s16[i];
                    q.ld_la = m > 1 ? (int64_t)m * r : r;
                    q.lr = r;
                    q.LB = p[i].B;
                }
                q.N = N;
                q.Kc = K;
                q.D = p[i].y;
                q.ldd = N;
                f += 2.0 * T * N * (double)(K + (lora ? r : 0));
            }
        } else {
            if (!p[i0].dX) continue;
            if (k == gemm_multi_max_problems() || m > kGemmMaxSeg) return false;
            GemmProblem& q = pr[k++];
            int64_t nsum = 0;
            q.na = m;
            for (int j = 0; j < m; ++j) {
                q.A[j] = p[i0 + j].dY;
                q.lda[j] = p[i0 + j].W.rows;
                q.a_kc[j] = p[i0 + j].W.rows;
                nsum += p[i0 + j].W.rows;
            }
            q.B = p[i0].W.bf16;                 // the members' bases back to back: [nsum, K]
            q.ldb = K;
            if (lora) {
                q.LA = m > 1 ? w.la[i0] : w.s16[i0];
                q.ld_la = (int64_t)m * r;
                q.lr = m * r;
                q.LB = m > 1 ? w.lb[i0] : p[i0].A;
            }
            q.N = K;
            q.Kc = nsum;
            q.D = p[i0].dX;
            q.ldd = K;
            f += 2.0 * T * K * (double)(nsum + (lora ? m * r : 0));
        }
    }
    if (k < 2 || !gemm_multi_fits(pr, k, T)) return false;
    *np = k;
    *flop = f;
    return true;
}

lsn_status lora_layer_fwd(int n, const lsn_lora_proj* p, int64_t T, int r, float scale, void* ws, size_t ws_bytes,
                          lsn_stream_t stream) {
    NvtxRange nvtx("lora_layer_fwd");
    lsn_status s = check_layer(n, p, T, r, ws, ws_bytes, false, "lora_layer_fwd");
    if (s != LSN_OK) return s;
    if (T == 0) return LSN_OK;
    if ((s = check_device()) != LSN_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const LayerWs w = carve_layer(ws, n, p, T, r);
    const Groups g = find_groups(n, p);
    bool deq[LSN_LAYER_MAX_PROJ];
    DownSpec dn[LSN_LAYER_MAX_PROJ];
    int nd = 0;
    for (int k = 0; k < g.n; ++k) {
        const int i0 = g.first[k], m = g.count[k];
        for (int j = 0; j < m; ++j) {
            const int i = i0 + j;
            deq[i] = p[i].W.kind == LSN_BASE_NF4 &&
                     (m > 1 || !(fused_here(p[i].W, T, p[i].W.rows) || fused_tmem_fwd(p[i].W, T)));
            if (adapter_off(p[i])) continue;
            // a group's bf16(s u) go side by side into its LoRA operand
            dn[nd++] = m > 1 ? DownSpec{p[i].x, p[i].A, p[i].u, w.la[i0] + j * r, T, p[i].W.cols, scale, m * r}
                             : DownSpec{p[i].x, p[i].A, p[i].u, w.s16[i], T, p[i].W.cols, scale};
        }
    }
    // Two lanes: the down projections (bound by reading x) run beside the
    // dequantisation (bound by writing W); then the GEMMs, which are
    // independent of each other, alternate over the lanes.  With nothing to
    // dequantise and no groups, only the first GEMM's down projection runs
    // ahead of it: the others run on the side lane beside that GEMM, and the
    // main lane's later GEMMs wait for them.
    LaneScope lanes(st, g_layer_lanes.load() == 2);
    bool any_deq = false, any_group = false;
    for (int i = 0; i < n; ++i) any_deq = any_deq || deq[i];
    for (int k = 0; k < g.n; ++k) any_group = any_group || g.count[k] > 1;
    // (One lane: the same order, everything on the caller's stream; taken when
    // merging, so that the merged launch is the same with one lane or two.)
    const bool early = (lanes.two() || gemm_multi()) && !any_deq && !any_group && nd > 0 && !adapter_off(p[0]);
    if (early) {
        if ((s = timed_down_batch(1, dn, true, r, lanes.main())) != LSN_OK) return s;      // dn[0]: projection 0
        if ((s = timed_down_batch(nd - 1, dn + 1, true, r, lanes.side())) != LSN_OK) return s;
    } else {
        for (int k = 0; k < g.n; ++k)
            if (g.count[k] > 1 && !adapter_off(p[g.first[k]]))
                if ((s = build_group_lb(p, g.first[k], g.count[k], r, false, w.lb[g.first[k]], lanes.side())) != LSN_OK)
                    return s;
        if ((s = timed_down_batch(nd, dn, true, r, lanes.side())) != LSN_OK) return s;
        if ((s = layer_dequant(n, p, deq, w, lanes.main())) != LSN_OK) return s;
        if ((s = lanes.barrier()) != LSN_OK) return s;
        GemmProblem pr[LSN_LAYER_MAX_PROJ];
        int np = 0;
        double flop = 0.0;
        if (grouped_problems(n, p, g, T, r, w, false, pr, &np, &flop)) {
            TimingScope ts(LSN_K_GEMM_FWD, flop, lanes.main());
            if ((s = launch_gemm_multi(pr, np, false, T, r, w.err, lanes.main())) != LSN_OK) return s;
            return lanes.join();
        }
    }
    // Merged: after the first GEMM, the other projections' GEMMs as one
    // launch on the side lane, right behind their down projections (so it
    // takes the SMs the first GEMM's last round leaves free).
    const bool merge = early && merge_rest(n, p, T, false);
    for (int k = 0; k < g.n; ++k) {
        if (merge && k == 1) {
            if ((s = merged_gemms(n, p, T, r, w, false, lanes.side())) != LSN_OK) return s;
            break;
        }
        if (early && k == 1 && (s = lanes.main_waits_side()) != LSN_OK) return s;
        const int i = g.first[k], m = g.count[k];
        const int64_t K = p[i].W.cols;
        const cudaStream_t gs = (k & 1) ? lanes.side() : lanes.main();
        const GemmSplitWs* sp = &w.split[k & 1];
        const int ri = adapter_off(p[i]) ? 0 : r;       // no LoRA K-block with the adapter off
        const uint16_t* Wb = p[i].W.kind == LSN_BASE_NF4 ? w.w16[i] : p[i].W.bf16;
        if (m > 1) {
            // one GEMM over the stacked weights, each projection's columns to its own y
            GemmGroup gg;
            gg.A[0] = p[i].x;
            gg.lda[0] = K;
            gg.a_kc[0] = K;
            gg.nseg = m;
            int64_t nsum = 0;
            for (int j = 0; j < m; ++j) {
                gg.seg_cols[j] = p[i + j].W.rows;
                gg.seg_D[j] = p[i + j].y;
                gg.seg_ld[j] = p[i + j].W.rows;
                nsum += p[i + j].W.rows;
            }
            TimingScope ts(LSN_K_GEMM_FWD, 2.0 * T * nsum * (double)(K + m * ri), gs);
            s = launch_gemm_grouped(gg, Wb, K, false, w.la[i], w.lb[i], m * ri, T, nsum, K, nullptr, 0, w.err, gs, sp);
        } else if (fused_tmem_fwd(p[i].W, T)) {
            const int64_t N = p[i].W.rows;
            TimingScope ts(LSN_K_GEMM_FWD, 2.0 * T * N * (double)(K + ri), gs);
            s = launch_gemm_nf4t(p[i].x, K, &p[i].W.nf4, w.s16[i], p[i].B, ri, T, N, K, p[i].y, N, w.err, gs);
        } else if (fused_here(p[i].W, T, p[i].W.rows)) {
            const int64_t N = p[i].W.rows;
            TimingScope ts(LSN_K_GEMM_FWD, 2.0 * T * N * (double)(K + ri), gs);
            s = launch_gemm_nf4(p[i].x, K, &p[i].W.nf4, false, w.s16[i], p[i].B, ri, T, N, K, p[i].y, N, w.err, gs);
        } else {
            const int64_t N = p[i].W.rows;
            s = timed_gemm(LSN_K_GEMM_FWD, p[i].x, K, Wb, K, false, w.s16[i], p[i].B, ri, T, N, K, p[i].y, N, w.err,
                           gs, sp);
        }
        if (s != LSN_OK) return s;
    }
    return lanes.join();
}

lsn_status lora_layer_bwd(int n, const lsn_lora_proj* p, int64_t T, int r, float scale, int accumulate, void* ws,
                          size_t ws_bytes, lsn_stream_t stream) {
    NvtxRange nvtx("lora_layer_bwd");
    lsn_status s = check_layer(n, p, T, r, ws, ws_bytes, true, "lora_layer_bwd");
    if (s != LSN_OK) return s;
    if ((s = check_device()) != LSN_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const LayerWs w = carve_layer(ws, n, p, T, r);
    const Groups g = find_groups(n, p);
    // Two lanes: the down projections (reading dY, and x when no u was kept)
    // run beside the dequantisation; then the token reductions run on the
    // side lane beside the input-gradient GEMMs, which alternate over both.
    LaneScope lanes(st, T > 0 && g_layer_lanes.load() == 2);
    bool early = false;
    if (T > 0) {
        bool deq[LSN_LAYER_MAX_PROJ];
        DownSpec dg[LSN_LAYER_MAX_PROJ], du[LSN_LAYER_MAX_PROJ];
        int ng = 0, nu = 0;
        for (int k = 0; k < g.n; ++k) {
            const int i0 = g.first[k], m = g.count[k];
            const bool want_dx = p[i0].dX != nullptr;    // a group's dX is its first member's
            for (int j = 0; j < m; ++j) {
                const int i = i0 + j;
                const int64_t N = p[i].W.rows, K = p[i].W.cols;
                deq[i] = want_dx && p[i].W.kind == LSN_BASE_NF4 && (m > 1 || !fused_here(p[i].W, T, K));
                if (adapter_off(p[i])) continue;
                dg[ng++] = m > 1 ? DownSpec{p[i].dY, p[i].B, w.g32[i], w.la[i0] + j * r, T, N, scale, m * r}
                                 : DownSpec{p[i].dY, p[i].B, w.g32[i], w.s16[i], T, N, scale};
                if (!p[i].u) du[nu++] = DownSpec{p[i].x, p[i].A, w.u32[i], nullptr, T, K, scale};
            }
        }
        bool any_deq = false, any_group = false;
        for (int i = 0; i < n; ++i) any_deq = any_deq || deq[i];
        for (int k = 0; k < g.n; ++k) any_group = any_group || g.count[k] > 1;
        // With nothing to dequantise and no groups, only the first input-gradient
        // GEMM's g = dY B runs ahead of it (on the main lane); the other down
        // projections and the token reductions run on the side lane beside it.
        early = (lanes.two() || gemm_multi()) && !any_deq && !any_group && ng > 0 && p[0].dX != nullptr &&
                !adapter_off(p[0]);
        if (early) {
            if ((s = timed_down_batch(1, dg, false, r, lanes.main())) != LSN_OK) return s;   // dg[0]: projection 0
            if ((s = timed_down_batch(ng - 1, dg + 1, false, r, lanes.side())) != LSN_OK) return s;
            if ((s = timed_down_batch(nu, du, true, r, lanes.side())) != LSN_OK) return s;
            if ((s = lanes.mark_side()) != LSN_OK) return s;            // every g but the first is made
            if ((s = lanes.side_waits_main()) != LSN_OK) return s;      // the reductions need g of projection 0
        } else {
            for (int k = 0; k < g.n; ++k)
                if (g.count[k] > 1 && p[g.first[k]].dX && !adapter_off(p[g.first[k]]))
                    if ((s = build_group_lb(p, g.first[k], g.count[k], r, true, w.lb[g.first[k]], lanes.side())) != LSN_OK)
                        return s;
            if ((s = timed_down_batch(ng, dg, false, r, lanes.side())) != LSN_OK) return s;
            if ((s = timed_down_batch(nu, du, true, r, lanes.side())) != LSN_OK) return s;
            if ((s = layer_dequant(n, p, deq, w, lanes.main())) != LSN_OK) return s;
            if ((s = lanes.barrier()) != LSN_OK) return s;
        }
    }
    // dA and dB of every projection in one launch (with T == 0: zeros, or the
    // accumulators left as they are); they need only g and u.
    TgSpec tg[2 * LSN_LAYER_MAX_PROJ];
    int nt = 0;
    for (int i = 0; i < n; ++i) {
        if (adapter_off(p[i])) continue;                // no adapter, no adapter gradients
        const int64_t N = p[i].W.rows, K = p[i].W.cols;
        tg[nt++] = TgSpec{w.g32[i], p[i].x, p[i].dA, T, K, true, accumulate, scale};
        tg[nt++] = TgSpec{p[i].u ? p[i].u : w.u32[i], p[i].dY, p[i].dB, T, N, false, accumulate, scale};
    }
    if ((s = timed_tgrad_batch(nt, tg, r, lanes.side())) != LSN_OK) return s;
    if (T > 0 && !early) {
        // Groups (or a call whose first projection runs with the adapter off):
        // every input-gradient GEMM in one merged launch on the main lane.
        GemmProblem pr[LSN_LAYER_MAX_PROJ];
        int np = 0;
        double flop = 0.0;
        if (grouped_problems(n, p, g, T, r, w, true, pr, &np, &flop)) {
            TimingScope ts(LSN_K_GEMM_BWD, flop, lanes.main());
            if ((s = launch_gemm_multi(pr, np, true, T, r, w.err, lanes.main())) != LSN_OK) return s;
            return lanes.join();
        }
    }
    if (T > 0) {
        // Merged: after the first GEMM, the other projections' input-gradient
        // GEMMs as one launch on the main lane (the token reductions keep the
        // side lane).
        const bool merge = early && merge_rest(n, p, T, true);
        for (int k = 0, j = 0; k < g.n; ++k) {
            const int i = g.first[k], m = g.count[k];
            if (!p[i].dX) continue;
            const int64_t K = p[i].W.cols;
            if (early && j == 1 && (s = lanes.main_waits_mark()) != LSN_OK) return s;   // the other g
            if (merge && j == 1) {
                if ((s = merged_gemms(n, p, T, r, w, true, lanes.main())) != LSN_OK) return s;
                break;
            }
            const GemmSplitWs* sp = &w.split[j & 1];
            const cudaStream_t gs = (j++ & 1) ? lanes.side() : lanes.main();
            const int ri = adapter_off(p[i]) ? 0 : r;
            const uint16_t* Wb = p[i].W.kind == LSN_BASE_NF4 ? w.w16[i] : p[i].W.bf16;
            if (m > 1) {
                // dX = [dY_1 .. dY_m] [W_1; ..; W_m] + [s g_1 .. s g_m] [A_1; ..; A_m]
                GemmGroup gg;
                gg.na = m;
                int64_t nsum = 0;
                for (int q = 0; q < m; ++q) {
                    gg.A[q] = p[i + q].dY;
                    gg.lda[q] = p[i + q].W.rows;
                    gg.a_kc[q] = p[i + q].W.rows;
                    nsum += p[i + q].W.rows;
                }
                TimingScope ts(LSN_K_GEMM_BWD, 2.0 * T * K * (double)(nsum + m * ri), gs);
                s = launch_gemm_grouped(gg, Wb, K, true, w.la[i], w.lb[i], m * ri, T, K, nsum, p[i].dX, K, w.err, gs, sp);
            } else if (fused_here(p[i].W, T, K)) {
                const int64_t N = p[i].W.rows;
                TimingScope ts(LSN_K_GEMM_BWD, 2.0 * T * K * (double)(N + ri), gs);
                s = launch_gemm_nf4(p[i].dY, N, &p[i].W.nf4, true, w.s16[i], p[i].A, ri, T, K, N, p[i].dX, K, w.err,
                                    gs);
            } else {
                const int64_t N = p[i].W.rows;
                s = timed_gemm(LSN_K_GEMM_BWD, p[i].dY, N, Wb, K, true, w.s16[i], p[i].A, ri, T, K, N, p[i].dX, K,
                               w.err, gs, sp);
            }
            if (s != LSN_OK) return s;
        }
    }
    return lanes.join();
}

lsn_status lsn_set_option(int option, int value) {
    if (option == LSN_OPT_PDL) {
        g_pdl.store(value != 0 ? 1 : 0);
        return LSN_OK;
    }
    if (option == LSN_OPT_LAYER_LANES) {
        LSN_CHECK_ARG(value == 1 || value == 2, "lsn_set_option: LSN_OPT_LAYER_LANES takes 1 or 2");
        g_layer_lanes.store(value);
        return LSN_OK;
    }
    if (option == LSN_OPT_FUSED_NF4) {
        LSN_CHECK_ARG(value >= 0 && value <= 2, "lsn_set_option: LSN_OPT_FUSED_NF4 takes 0, 1 or 2");
        g_fused_nf4.store(value);
        return LSN_OK;
    }
    if (option == LSN_OPT_STREAM_K) {
        gemm_set_stream_k(value != 0);
        return LSN_OK;
    }
    if (option == LSN_OPT_GEMM_MIN_UNITS) {
        gemm_set_min_units(value != 0);
        return LSN_OK;
    }
    if (option == LSN_OPT_GEMM_TAIL_SPLIT) {
        gemm_set_tail_split(value != 0);
        return LSN_OK;
    }
    if (option == LSN_OPT_LAYER_MERGE) {
        gemm_set_multi(value != 0);
        return LSN_OK;
    }
    if (option == LSN_OPT_DEQUANT_SPARE_SMS) {
        LSN_CHECK_ARG(value >= 0 && value <= 4096, "lsn_set_option: LSN_OPT_DEQUANT_SPARE_SMS out of range");
        dequant_set_spare_sms(value);
        return LSN_OK;
    }
    return fail(LSN_ERR_INVALID_ARG, "lsn_set_option: unknown option");
}

int lsn_get_option(int option) {
    if (option == LSN_OPT_FUSED_NF4) return g_fused_nf4.load();
    if (option == LSN_OPT_LAYER_LANES) return g_layer_lanes.load();
    if (option == LSN_OPT_PDL) return g_pdl.load();
    if (option == LSN_OPT_STREAM_K) return gemm_stream_k() ? 1 : 0;
    if (option == LSN_OPT_GEMM_MIN_UNITS) return gemm_min_units() ? 1 : 0;
    if (option == LSN_OPT_GEMM_TAIL_SPLIT) return gemm_tail_split() ? 1 : 0;
    if (option == LSN_OPT_LAYER_MERGE) return gemm_multi() ? 1 : 0;
    if (option == LSN_OPT_DEQUANT_SPARE_SMS) return dequant_spare_sms();
    return -1;
}

lsn_status lsn_gemm_merged_schedule(int units, int n, const int* ntiles, const int* cost, int* start, int* tile,
                                    int max_tiles) {
    return gemm_merged_schedule(units, n, ntiles, cost, start, tile, max_tiles);
}

lsn_status lsn_ws_status(void* ws, lsn_stream_t stream) {
    LSN_CHECK_ARG(ws != nullptr, "lsn_ws_status: workspace is NULL");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int h = 0;
    LSN_CUDA_TRY(cudaMemcpyAsync(&h, ws, sizeof(int), cudaMemcpyDeviceToHost, st));
    LSN_CUDA_TRY(cudaStreamSynchronize(st));
    if (h != 0) {
        LSN_CUDA_TRY(cudaMemsetAsync(ws, 0, sizeof(int), st));
        LSN_CUDA_TRY(cudaStreamSynchronize(st));
        return fail(LSN_ERR_TIMEOUT, "a tensor-core kernel gave up waiting (code " + std::to_string(h) + ")");
    }
    return LSN_OK;
}

}  // extern "C"
