// Host-side launchers of the library's kernels (defined in codec.cu, gemm.cu
// and lora_small.cu), called by the C entry points in api.cu.
#pragma once

#include "common.cuh"

namespace lsn {

// One rank-r down projection: out[t, j] = sum_k X[t, k] W(j, k) for j < r,
// W either A [r, Kd] or B [Kd, r]; written as fp32 (u32, row stride r) and/or
// as bf16(scale * out) (u16, row stride ld16, r when 0), either may be NULL.
struct DownSpec {
    const uint16_t* X;
    const uint16_t* W;
    float* u32;
    uint16_t* u16;
    int64_t T, Kd;
    float scale;
    int ld16 = 0;
};

// One token reduction: R[j, k] = sum_t G[t, j] X[t, k], written (or, with
// accumulate, added) as scale * R into out, [r, Kd] when out_rk else [Kd, r].
struct TgSpec {
    const float* G;
    const uint16_t* X;
    float* out;
    int64_t T, Kd;
    bool out_rk;
    int accumulate;
    float scale;
};

// Launch attribute of the hot-path kernels: programmatic dependent launch
// when enabled (LSN_OPT_PDL), so a kernel's set-up overlaps the tail of the
// kernel before it on the stream.  Returns the number of attributes written (0 or 1).
bool pdl_enabled();
inline int pdl_attr(cudaLaunchAttribute* a) {
    if (!pdl_enabled()) return 0;
    a->id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a->val.programmaticStreamSerializationAllowed = 1;
    return 1;
}

// Argument checks shared by the entry points (api.cu): the current device is
// an sm_100 part; an NF4 weight descriptor is well formed (shape, arrays,
// alignment, rows * cols <= kMaxNf4Elems checked without overflow).
constexpr int64_t kMaxNf4Elems = (int64_t)1 << 46;
lsn_status check_device();
lsn_status check_nf4(const lsn_nf4_weight* w, const char* who);

size_t quantize_ws_bytes(int64_t rows, int64_t cols);
lsn_status launch_quantize(const float* W, const lsn_nf4_weight* out, void* ws, size_t ws_bytes, cudaStream_t st);
lsn_status launch_dequant(const lsn_nf4_weight* w, uint16_t* out, cudaStream_t st);
// Several NF4 weights dequantised by one launch (at most 16 per launch; more take several).
// blocks_per_sm > 0 caps the grid at that many blocks per SM (which then loop
// over the work), for a dequantisation meant to run beside other kernels.
lsn_status launch_dequant_batch(int n, const lsn_nf4_weight* const* w, uint16_t* const* out, cudaStream_t st,
                                int blocks_per_sm = 0);

// Grouped GEMM operands: the A operand as na tensors side by side along the
// contraction (tensor i: [M, a_kc[i]] row-major with row stride lda[i]; every
// a_kc but the last a multiple of 128), and the output columns split into
// nseg segments (segment i: seg_cols[i] columns, a multiple of 64, written at
// seg_D[i] with row stride seg_ld[i]); nseg == 0: the single output D.
constexpr int kGemmMaxSeg = 4;
struct GemmGroup {
    int na = 1;
    const uint16_t* A[kGemmMaxSeg] = {};
    int64_t lda[kGemmMaxSeg] = {};
    int64_t a_kc[kGemmMaxSeg] = {};
    int nseg = 0;
    int64_t seg_cols[kGemmMaxSeg] = {};
    uint16_t* seg_D[kGemmMaxSeg] = {};
    int64_t seg_ld[kGemmMaxSeg] = {};
};
// Scratch of the GEMM's stream-K schedule (one region per stream that runs
// GEMMs concurrently): arrival counters (zero between launches; the region
// must be zero-filled once before its first use) and fp32 partial tiles.
constexpr int kSplitMaxUnits = 160;                // workers the region is sized for (CTAs; pairs: half)
constexpr size_t kSplitCntBytes = 4096;
struct GemmSplitWs {
    int* cnt = nullptr;
    float* part = nullptr;
};
size_t gemm_split_ws_bytes();
GemmSplitWs gemm_split_ws(void* base);
void gemm_set_stream_k(bool on);
bool gemm_stream_k();
void gemm_set_min_units(bool on);
bool gemm_min_units();
void gemm_set_tail_split(bool on);
bool gemm_tail_split();
int gemm_units(int64_t tiles, bool pair);
// Dequantisation beside other work (LSN_OPT_DEQUANT_SPARE_SMS).
void dequant_set_spare_sms(int n);
int dequant_spare_sms();

// One of several independent GEMMs launched together (launch_gemm_multi): the
// arguments of launch_gemm for one problem, on the 2-SM kernel.  A may be
// split along the contraction into na parts as for a grouped GEMM (part j:
// A[j] [M, a_kc[j]] with row stride lda[j]; all parts but the last a multiple
// of 128 wide; na == 1: A[0] covers Kc).  The LoRA term: LA [M, lr] with row
// stride ld_la (lr = 0 or LA == NULL: none; lr == 0 means the call's r), LB
// [N, lr] (K-major B) or [lr, N] (MN-major B).
struct GemmProblem {
    int na = 1;
    const uint16_t* A[kGemmMaxSeg] = {};
    int64_t lda[kGemmMaxSeg] = {};
    int64_t a_kc[kGemmMaxSeg] = {};
    const uint16_t* B = nullptr;
    int64_t ldb = 0;
    const uint16_t* LA = nullptr;
    const uint16_t* LB = nullptr;
    int lr = 0;
    int64_t ld_la = 0;
    int64_t N = 0, Kc = 0;
    uint16_t* D = nullptr;
    int64_t ldd = 0;
};
int gemm_multi_max_problems();
lsn_status gemm_merged_schedule(int units, int n, const int* ntiles, const int* cost, int* start, int* tile,
                                int max_tiles);
// Whether n problems of M rows fit one launch (problem and tile limits).
bool gemm_multi_fits(const GemmProblem* pr, int n, int64_t M);
// D_i = A_i . op(B_i) + LA_i . op(LB_i) for every problem i, one persistent
// launch with a balanced static tile schedule (b_mn as for launch_gemm; all
// problems share M and r).
lsn_status launch_gemm_multi(const GemmProblem* pr, int n, bool b_mn, int64_t M, int r, int* err,
                             cudaStream_t st);
void gemm_set_multi(bool on);
bool gemm_multi();

// split == NULL: whole tiles round robin (no stream-K scratch).
lsn_status launch_gemm_grouped(const GemmGroup& g, const uint16_t* B, int64_t ldb, bool b_mn, const uint16_t* LA,
                               const uint16_t* LB, int r, int64_t M, int64_t N, int64_t Kc, uint16_t* D,
                               int64_t ldd, int* err, cudaStream_t st, const GemmSplitWs* split);
lsn_status launch_gemm(const uint16_t* A, int64_t lda, const uint16_t* B, int64_t ldb, bool b_mn, const uint16_t* LA,
                       const uint16_t* LB, int r, int64_t M, int64_t N, int64_t Kc, uint16_t* D, int64_t ldd,
                       int* err, cudaStream_t st, const GemmSplitWs* split);
lsn_status launch_gemm_nf4(const uint16_t* A, int64_t lda, const lsn_nf4_weight* w, bool b_mn, const uint16_t* LA,
                           const uint16_t* LB, int r, int64_t M, int64_t N, int64_t Kc, uint16_t* D, int64_t ldd,
                           int* err, cudaStream_t st);
bool gemm_use_pairs(int64_t M, int64_t N);

// A 2-D tensor map of a row-major [outer, inner] tensor with row stride
// stride_elems, read in boxes of box_inner x box_outer: bf16 with the
// 128-byte swizzle, or (bytes) uint8 with the 64-byte swizzle.
lsn_status make_tmap_2d(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, int64_t stride_elems,
                        int box_inner, int box_outer, bool bytes);

// The forward GEMM of an NF4 base with W converted straight into tensor
// memory (gemm_nf4t.cu): y [M, N] = x [M, Kc] W^T + LA [M, r] LB^T with
// W = w [N, Kc] NF4, LB [N, r].  LSN_ERR_UNSUPPORTED when the shape has fewer
// output tiles than SM pairs (the caller dequantises instead).
bool gemm_nf4t_supported(int64_t M, int64_t N, int64_t Kc);
lsn_status launch_gemm_nf4t(const uint16_t* x, int64_t ldx, const lsn_nf4_weight* w, const uint16_t* LA,
                            const uint16_t* LB, int r, int64_t M, int64_t N, int64_t Kc, uint16_t* y, int64_t ldy,
                            int* err, cudaStream_t st);

lsn_status launch_lora_down(const uint16_t* X, const uint16_t* W, bool w_rk, int64_t T, int64_t Kd, int r,
                            float scale, float* u32, uint16_t* u16, cudaStream_t st);
lsn_status launch_lora_down_batch(int n, const DownSpec* specs, bool w_rk, int r, cudaStream_t st);
lsn_status launch_lora_tgrad(const float* G, const uint16_t* X, bool out_rk, int64_t T, int64_t Kd, int r,
                             float scale, int accumulate, float* out, cudaStream_t st);
lsn_status launch_lora_tgrad_batch(int n, const TgSpec* specs, int r, cudaStream_t st);
int down_splits(int64_t T, int64_t Kd);
int tgrad_splits(int64_t T, int64_t Kd);

}  // namespace lsn
