// NF4 codec: quantisation with double-quantised absmax constants, and the
// standalone dequantisation kernel.
//
// Format ("Can You Fine-Tune a 27B Model on a Laptop? (I Did the Math)",
// 2:19-2:29, names a 4-bit format for bell-curve weights and a second
// quantisation of its constants; the construction followed is QLoRA's, the
// paper linked by "An 8B Fine-Tune Now Fits in 4 GB of VRAM"):
//   levels      normal quantiles, 7 negative, 0, 8 positive, scaled to [-1, 1]
//   level code  nearest level of w / absmax over blocks of 64, ties lower
//   packing     byte j = code[2j] << 4 | code[2j+1]
//   constants   8-bit codes of (absmax - mean) / s2 on the table k/127, one
//               fp32 s2 per 256 blocks, one fp32 mean per tensor
//   dequant     w = bf16(level[q] * (table[c] * s2 + mean)), each op rounded
//
// Every rounding-sensitive operation uses an explicit IEEE intrinsic
// (__fdiv_rn, __fsub_rn, __fmul_rn, __fadd_rn) so the compiler can neither
// contract nor approximate it.
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "launch.cuh"
#include "timing.cuh"

namespace lsn {

// ------------------------------------------------------------ host tables --

namespace {

double std_normal_cdf(double x) { return 0.5 * std::erfc(-x / std::sqrt(2.0)); }

// Quantile of N(0,1) for p in [1/2, 1): bisection on the CDF (bracket [0, 9])
// until the bracket stops shrinking, then two Newton steps on the upper tail
// 1 - Phi(x) = erfc(x / sqrt 2) / 2, which libm evaluates with full relative
// accuracy.
double std_normal_quantile_upper(double p) {
    if (p == 0.5) return 0.0;
    double lo = 0.0, hi = 9.0;
    for (int it = 0; it < 2000; ++it) {
        const double mid = 0.5 * (lo + hi);
        if (mid <= lo || mid >= hi) break;
        if (std_normal_cdf(mid) < p) lo = mid; else hi = mid;
    }
    double x = 0.5 * (lo + hi);
    const double tail = 1.0 - p;
    for (int it = 0; it < 2; ++it) {
        const double f = 0.5 * std::erfc(x / std::sqrt(2.0)) - tail;      // decreasing in x
        const double dens = std::exp(-0.5 * x * x) / std::sqrt(2.0 * M_PI);
        x += f / dens;
    }
    return x;
}

// Largest fp32 value that is <= the exact midpoint of two fp32 levels: an
// fp32 v has its nearest level at index <= i exactly when v <= thr[i]
// (ties go to the lower index).
float threshold_below(float a, float b) {
    const double mid = ((double)a + (double)b) * 0.5;   // exact: two fp32 summands
    float t = (float)mid;
    if ((double)t > mid) t = std::nextafter(t, -INFINITY);
    return t;
}

Nf4Tables build_tables() {
    Nf4Tables t;
    const double p_max = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0);
    double lv[16];
    int n = 0;
    for (int j = 7; j >= 1; --j) lv[n++] = -std_normal_quantile_upper(0.5 + (p_max - 0.5) * j / 7.0);
    lv[n++] = 0.0;
    for (int j = 1; j <= 8; ++j) lv[n++] = std_normal_quantile_upper(0.5 + (p_max - 0.5) * j / 8.0);
    double mx = 0.0;
    for (double v : lv) mx = std::fmax(mx, std::fabs(v));
    for (int i = 0; i < 16; ++i) t.level[i] = (float)(lv[i] / mx);
    for (int i = 0; i < 15; ++i) t.thr[i] = threshold_below(t.level[i], t.level[i + 1]);
    for (int k = -127; k <= 127; ++k) t.dq[k + 127] = (float)((double)k / 127.0);
    t.dq[255] = 0.0f;
    for (int i = 0; i < 254; ++i) t.dq_thr[i] = threshold_below(t.dq[i], t.dq[i + 1]);
    return t;
}

}  // namespace

const Nf4Tables& nf4_tables() {
    static Nf4Tables tables = build_tables();
    return tables;
}

// ---------------------------------------------------------------- kernels --

struct LevelParams { float level[16]; float thr[15]; };
struct DqParams { float dq[256]; float thr[254]; };

// Pass 1: one warp per block of 64 elements.  Lane l owns elements 2l, 2l+1:
// absmax by a warp max, codes by counting thresholds below w / absmax, one
// packed byte per lane (32 contiguous bytes per block).
__global__ void __launch_bounds__(256) nf4_level_codes_kernel(const float2* __restrict__ W, int64_t nblk,
                                                               uint8_t* __restrict__ packed,
                                                               float* __restrict__ absmax, LevelParams P) {
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t b = warp0; b < nblk; b += nwarps) {
        const float2 w = W[b * 32 + lane];
        float a = fmaxf(fabsf(w.x), fabsf(w.y));
        #pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        uint32_t q0 = 7, q1 = 7;
        if (a > 0.0f) {
            const float v0 = __fdiv_rn(w.x, a), v1 = __fdiv_rn(w.y, a);
            q0 = 0; q1 = 0;
            #pragma unroll
            for (int i = 0; i < 15; ++i) { q0 += (v0 > P.thr[i]); q1 += (v1 > P.thr[i]); }
        }
        packed[b * 32 + lane] = (uint8_t)((q0 << 4) | q1);
        if (lane == 0) absmax[b] = a;
    }
}

// Pass 2: one thread per group of 256 blocks, sequential fp64 sum.
__global__ void dq_group_sum_kernel(const float* __restrict__ absmax, int64_t nblk, int64_t ngrp,
                                    double* __restrict__ partial) {
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= ngrp) return;
    const int64_t b1 = (g * 256 + 256 < nblk) ? g * 256 + 256 : nblk;
    double s = 0.0;
    for (int64_t b = g * 256; b < b1; ++b) s = __dadd_rn(s, (double)absmax[b]);
    partial[g] = s;
}

// Pass 3: one thread: sum of the group partials in group order, mean, fp32.
__global__ void dq_offset_kernel(const double* __restrict__ partial, int64_t ngrp, int64_t nblk,
                                 float* __restrict__ offset) {
    if (blockIdx.x != 0 || threadIdx.x != 0) return;
    double s = 0.0;
    for (int64_t g = 0; g < ngrp; ++g) s = __dadd_rn(s, partial[g]);
    *offset = __double2float_rn(__ddiv_rn(s, (double)nblk));
}

// Pass 4: one warp per group: s2 = max |absmax - offset|, then the 8-bit
// code of each block by binary search over the 254 thresholds.
__global__ void __launch_bounds__(256) dq_codes_kernel(const float* __restrict__ absmax, int64_t nblk,
                                                        int64_t ngrp, const float* __restrict__ offset,
                                                        uint8_t* __restrict__ absmax_q, float* __restrict__ s2,
                                                        DqParams P) {
    __shared__ float thr[256];
    for (int i = threadIdx.x; i < 254; i += blockDim.x) thr[i] = P.thr[i];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const float off = *offset;
    for (int64_t g = warp0; g < ngrp; g += nwarps) {
        float c[8];
        float m = 0.0f;
        #pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int64_t b = g * 256 + i * 32 + lane;
            c[i] = (b < nblk) ? __fsub_rn(absmax[b], off) : 0.0f;
            m = fmaxf(m, fabsf(c[i]));
        }
        #pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) s2[g] = m;
        #pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int64_t b = g * 256 + i * 32 + lane;
            if (b >= nblk) continue;
            uint32_t code = 127;
            if (m > 0.0f) {
                const float v = __fdiv_rn(c[i], m);
                int lo = 0, hi = 254;                 // count of thresholds strictly below v
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if (thr[mid] < v) lo = mid + 1; else hi = mid;
                }
                code = (uint32_t)lo;
            }
            absmax_q[b] = (uint8_t)code;
        }
    }
}

// Standalone dequantisation: each thread turns one 32-bit word of packed
// codes (8 weights, always inside one 64-block) into 8 bf16 = one 16-byte
// store.  Loads are 4 bytes per lane (128 B per warp), stores 16 bytes per
// lane (512 B per warp), both contiguous across the warp.
struct DequantParams { float level[16]; float dq[256]; };

// One NF4 weight of a dequantisation batch, counted in 16-byte vectors of
// packed codes (32 elements, half of a 64-element absmax block).
struct DqItem {
    const uint4* packed;
    const uint8_t* absmax_q;
    const float* s2;
    const float* offset;
    uint4* out;          // bf16 output, 64 bytes per vector
    int64_t nvec;
    int64_t first;       // first blockIdx.x of the item
};
constexpr int kDqMax = 16;
constexpr int kDqThreads = 256;
constexpr int kDqUnroll = 4;                       // vectors per thread
constexpr int kDqVecPerBlock = kDqThreads * kDqUnroll;
struct DqBatch {
    int n;
    DqItem it[kDqMax];
};

// Standalone dequantisation of a batch of weights: each thread reads four
// 128-bit words of packed codes (coalesced across the warp, all four in
// flight at once), builds the block's 16 scaled levels bf16(level *
// absmax_hat) in registers and maps the 32 codes of a word onto them with
// byte permutes (no shared-memory lookup per element).  The 64 bytes of bf16
// a thread makes for one word are passed through a per-warp staging buffer
// in shared memory (16-byte chunks XOR-swizzled, conflict-free both ways) so
// that every global store instruction of the warp writes 512 contiguous
// bytes.  A block covers 1024 consecutive words of one weight.  Codes are
// read and bf16 written with the streaming (evict-first) cache hint: each byte
// is touched once here, and the GEMMs running beside this kernel keep their
// operand tiles in L2 (measured 0.2-0.5 ms faster per 8B step).
constexpr int kDqWarps = kDqThreads / 32;

__device__ __forceinline__ int dq_stage_chunk(int c) { return c ^ ((c >> 3) & 7); }

__global__ void __launch_bounds__(kDqThreads) nf4_dequant_kernel(const __grid_constant__ DqBatch bt,
                                                                 const __grid_constant__ DequantParams P,
                                                                 int64_t units) {
    __shared__ float dq[256];
    __shared__ uint4 stage[kDqWarps][128];                 // 2 KB per warp: 32 lanes x 64 bytes
    for (int i = threadIdx.x; i < 256; i += blockDim.x) dq[i] = P.dq[i];
    pdl_launch_dependents();
    pdl_wait();
    __syncthreads();                                     // the code table is in shared memory
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint4* st = stage[warp];
    // One unit = 1024 consecutive words of one weight; a full grid has one
    // block per unit, a smaller one loops over them with the grid's stride.
    for (int64_t unit = blockIdx.x; unit < units; unit += gridDim.x) {
        int ii = 0;
        while (ii + 1 < bt.n && unit >= bt.it[ii + 1].first) ++ii;
        const DqItem& it = bt.it[ii];
        const uint4* __restrict__ packed = it.packed;
        const uint8_t* __restrict__ absmax_q = it.absmax_q;
        const float* __restrict__ s2 = it.s2;
        uint4* __restrict__ out = it.out;
        const float off = *it.offset;
        const int64_t v0 = (unit - it.first) * kDqVecPerBlock + threadIdx.x;
        uint4 p[kDqUnroll];
        uint32_t code[kDqUnroll];
        float sc[kDqUnroll];
        #pragma unroll
        for (int u = 0; u < kDqUnroll; ++u) {
            const int64_t v = v0 + u * kDqThreads;
            const bool ok = v < it.nvec;
            const int64_t b = (ok ? v : 0) >> 1;         // absmax block of the vector
            p[u] = ok ? __ldcs(packed + v) : make_uint4(0, 0, 0, 0);
            code[u] = __ldg(absmax_q + b);
            sc[u] = __ldg(s2 + (b >> 8));
        }
        #pragma unroll
        for (int u = 0; u < kDqUnroll; ++u) {
            const float ah = __fadd_rn(__fmul_rn(dq[code[u]], sc[u]), off);
            uint32_t lo[4], hi[4];
            nf4_scaled_table(P.level, ah, lo, hi);
            st[dq_stage_chunk(4 * lane + 0)] = nf4x8_to_bf16(p[u].x, lo, hi);
            st[dq_stage_chunk(4 * lane + 1)] = nf4x8_to_bf16(p[u].y, lo, hi);
            st[dq_stage_chunk(4 * lane + 2)] = nf4x8_to_bf16(p[u].z, lo, hi);
            st[dq_stage_chunk(4 * lane + 3)] = nf4x8_to_bf16(p[u].w, lo, hi);
            __syncwarp();
            // The warp's 32 consecutive words start at word w0; their output is
            // 2 KB at out + 4 * w0, written as four 512-byte rows.
            const int64_t w0 = v0 - lane + u * kDqThreads;
            #pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int c = 32 * i + lane;             // output chunk of the warp, in 16-byte units
                if (w0 + (c >> 2) < it.nvec) __stcs(out + 4 * w0 + c, st[dq_stage_chunk(c)]);
            }
            __syncwarp();
        }
    }
}

// ------------------------------------------------------------ launchers ---

size_t quantize_ws_bytes(int64_t rows, int64_t cols) {
    const int64_t nblk = rows * cols / 64;
    const int64_t ngrp = (nblk + 255) / 256;
    return round_up((size_t)nblk * sizeof(float), 256) + (size_t)ngrp * sizeof(double);
}

static int grid_for(int64_t work_items, int per_block, int waves_cap) {
    int64_t g = (work_items + per_block - 1) / per_block;
    const int64_t cap = (int64_t)sm_count() * waves_cap;
    if (g > cap) g = cap;
    if (g < 1) g = 1;
    return (int)g;
}

lsn_status launch_quantize(const float* W, const lsn_nf4_weight* out, void* ws, size_t ws_bytes,
                           cudaStream_t st) {
    const int64_t numel = out->rows * out->cols;
    const int64_t nblk = numel / 64;
    const int64_t ngrp = (nblk + 255) / 256;
    const Nf4Tables& T = nf4_tables();
    float* absmax = reinterpret_cast<float*>(ws);
    double* partial = reinterpret_cast<double*>(reinterpret_cast<char*>(ws) + round_up((size_t)nblk * 4, 256));
    LevelParams lp;
    std::memcpy(lp.level, T.level, sizeof(lp.level));
    std::memcpy(lp.thr, T.thr, sizeof(lp.thr));
    nf4_level_codes_kernel<<<grid_for(nblk, 8, 16), 256, 0, st>>>(reinterpret_cast<const float2*>(W), nblk,
                                                                  out->packed, absmax, lp);
    dq_group_sum_kernel<<<(int)ceil_div(ngrp, 128), 128, 0, st>>>(absmax, nblk, ngrp, partial);
    dq_offset_kernel<<<1, 32, 0, st>>>(partial, ngrp, nblk, out->offset);
    DqParams dp;
    std::memcpy(dp.dq, T.dq, sizeof(dp.dq));
    std::memcpy(dp.thr, T.dq_thr, sizeof(dp.thr));
    dq_codes_kernel<<<grid_for(ngrp, 8, 16), 256, 0, st>>>(absmax, nblk, ngrp, out->offset, out->absmax_q,
                                                          out->absmax_s2, dp);
    LSN_CUDA_TRY(cudaGetLastError());
    (void)ws_bytes;
    return LSN_OK;
}

namespace {
std::atomic<int> g_spare_sms{0};
// Dynamic shared memory a dequantisation block reserves when it must run on
// SMs of its own (LSN_OPT_DEQUANT_SPARE_SMS): with it no block fits beside a
// GEMM CTA, and at most three fit on an SM.
constexpr int kDqSpareSmem = 56 * 1024;
}

void dequant_set_spare_sms(int n) { g_spare_sms.store(n < 0 ? 0 : n); }
int dequant_spare_sms() { return g_spare_sms.load(); }

lsn_status launch_dequant_batch(int n, const lsn_nf4_weight* const* w, uint16_t* const* out, cudaStream_t st,
                                int blocks_per_sm) {
    const int spare = blocks_per_sm > 0 ? dequant_spare_sms() : 0;
    if (spare > 0) {
        static std::once_flag once;
        static cudaError_t attr_err = cudaSuccess;
        std::call_once(once, [] {
            attr_err = cudaFuncSetAttribute(nf4_dequant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDqSpareSmem);
        });
        if (attr_err != cudaSuccess) return fail_cuda(attr_err, "cudaFuncSetAttribute(dequant smem)");
    }
    const Nf4Tables& T = nf4_tables();
    DequantParams P;
    std::memcpy(P.level, T.level, sizeof(P.level));
    std::memcpy(P.dq, T.dq, sizeof(P.dq));
    DqBatch bt{};
    int64_t blocks = 0;
    auto flush = [&]() -> lsn_status {
        if (bt.n == 0) return LSN_OK;
        cudaLaunchConfig_t cfg = {};
        int64_t grid = blocks;
        const int64_t sms = spare > 0 ? spare : sm_count();
        if (blocks_per_sm > 0 && grid > sms * blocks_per_sm) grid = sms * blocks_per_sm;
        cfg.gridDim = dim3((unsigned)grid);
        cfg.blockDim = dim3(kDqThreads);
        cfg.dynamicSmemBytes = spare > 0 ? kDqSpareSmem : 0;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        cfg.attrs = attr;
        cfg.numAttrs = pdl_attr(&attr[0]);
        LSN_CUDA_TRY(cudaLaunchKernelEx(&cfg, nf4_dequant_kernel, bt, P, blocks));
        bt = DqBatch{};
        blocks = 0;
        return LSN_OK;
    };
    for (int i = 0; i < n; ++i) {
        const int64_t nvec = w[i]->rows * w[i]->cols / 32;
        if (nvec == 0) continue;
        if (bt.n == kDqMax) {
            const lsn_status s = flush();
            if (s != LSN_OK) return s;
        }
        DqItem& it = bt.it[bt.n++];
        it.packed = reinterpret_cast<const uint4*>(w[i]->packed);
        it.absmax_q = w[i]->absmax_q;
        it.s2 = w[i]->absmax_s2;
        it.offset = w[i]->offset;
        it.out = reinterpret_cast<uint4*>(out[i]);
        it.nvec = nvec;
        it.first = blocks;
        blocks += ceil_div(nvec, (int64_t)kDqVecPerBlock);
    }
    return flush();
}

lsn_status launch_dequant(const lsn_nf4_weight* w, uint16_t* out, cudaStream_t st) {
    return launch_dequant_batch(1, &w, &out, st);
}

}  // namespace lsn

// ------------------------------------------------- allocation-free variant --
//
// nf4_quantize needs scratch memory (one fp32 absmax per 64-block and one
// fp64 partial sum per group of 256 blocks) and takes it from the caller.
// Some callers cannot hand out device memory at the moment they quantise: a
// host whose allocator has reserved all device memory up front and allows no
// other allocation, a latency-critical loop that must not pay for
// cudaMalloc's implicit device synchronisation, or a plug-in that has no
// allocator at all.  nf4_quantize_noalloc serves them with a fixed scratch
// array that lives in this library's device image: it is allocated by the
// CUDA runtime when the library's module is loaded on a device and stays
// there until the process exits.

namespace lsn {
namespace {

constexpr int64_t kNoAllocMaxElems = (int64_t)1 << 26;               // 67,108,864 weight elements
constexpr int64_t kNoAllocMaxBlocks = kNoAllocMaxElems / 64;         // 1,048,576 absmax values
constexpr int64_t kNoAllocMaxGroups = kNoAllocMaxBlocks / 256;       // 4,096 partial sums
constexpr size_t kNoAllocScratchBytes =
    (size_t)kNoAllocMaxBlocks * sizeof(float) + (size_t)kNoAllocMaxGroups * sizeof(double);

// Shared by every call on a device; holds whatever the last call left.  The
// quantisation passes write every absmax and partial they later read, so
// nothing in it has to start at zero.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device.  The host-side
// name g_noalloc_scratch is only a stand-in for the symbol, never a device
// address, so it is resolved once per device with cudaGetSymbolAddress.
lsn_status noalloc_scratch(void** out) {
    int dev = 0;
    LSN_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return fail(LSN_ERR_UNSUPPORTED, "nf4_quantize_noalloc: device index too large");
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return fail_cuda(e, "nf4_quantize_noalloc: cudaGetSymbolAddress(scratch)");
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return LSN_OK;
}

}  // namespace

}  // namespace lsn

extern "C" lsn_status nf4_quantize_noalloc(const float* W, const lsn_nf4_weight* out, lsn_stream_t stream) {
    using namespace lsn;
    NvtxRange nvtx("nf4_quantize_noalloc");
    lsn_status s = check_nf4(out, "nf4_quantize_noalloc");
    if (s != LSN_OK) return s;
    // The limit is tested by division, before rows * cols is formed.
    LSN_CHECK_ARG(out->cols == 0 || out->rows <= kNoAllocMaxElems / out->cols,
                  "nf4_quantize_noalloc: rows*cols = " + std::to_string(out->rows) + "*" + std::to_string(out->cols) +
                      " exceeds the fixed scratch limit of " + std::to_string(kNoAllocMaxElems) +
                      " elements; use nf4_quantize with a caller workspace");
    const int64_t numel = out->rows * out->cols;
    if (numel == 0) return LSN_OK;
    LSN_CHECK_ARG(W != nullptr && aligned16(W), "nf4_quantize_noalloc: W must be a 16-byte aligned device pointer");
    if ((s = check_device()) != LSN_OK) return s;
    void* scratch = nullptr;
    if ((s = noalloc_scratch(&scratch)) != LSN_OK) return s;
    const double n = (double)numel;
    TimingScope ts(LSN_K_QUANTIZE, n * 4.0 + n / 2.0 + n / 64.0 * 6.0, reinterpret_cast<cudaStream_t>(stream), 4);
    return launch_quantize(W, out, scratch, kNoAllocScratchBytes, reinterpret_cast<cudaStream_t>(stream));
}
