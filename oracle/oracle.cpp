// Oracle for the layer-streamed NF4 LoRA linear: a plain, slow, obviously
// correct CPU implementation in fp64.
//
// TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
// call this file: only the test-suite, the smoke check and the CPU-baseline
// leg of the benchmark do.  It shares no code, header, table or constant
// generator with the CUDA library.
//
// What the method computes, and where the pages say so:
//  * "Exact Layer Streaming: LoRA Fine-Tuning of an 8B Model on a 4 GB Laptop
//    GPU" (abstract): LoRA training over a frozen NF4 or bf16 base whose
//    decoder layers stream from host RAM through a small VRAM pool; the
//    streamed run must equal a resident run of the same numerics.
//  * "Can You Fine-Tune a 27B Model on a Laptop? (I Did the Math)", 1:25-2:29:
//    the base is frozen and squeezed to four bits with a format built for
//    bell-curve weights (NF4), the constants of that first pass are quantised
//    again (double quantisation), and the trained part is a thin pair of
//    matrices per layer (LoRA).
//  The pages print neither the NF4 levels, the block sizes, the packing nor the
//  LoRA layouts.  The readings taken here (each marked READING below):
//    - NF4 levels: the normal-quantile construction of the QLoRA paper that
//      the sourcefeed article links (arXiv 2305.14314, section 3), 8 positive
//      and 7 negative quantiles of N(0,1) plus an exact zero, normalised so the
//      end points are exactly -1 and +1;
//    - first-level blocks of 64 consecutive elements of the row-major weight,
//      second level: 8-bit codes of (absmax - mean) over groups of 256 blocks,
//      on a linear signed table k/127;
//    - "nearest level" means smallest exact distance, ties to the lower index;
//    - packing: two codes per byte, the even element in the high nibble;
//    - y = x W^T + s (x A^T) B^T with s = alpha / r; W [N,K], A [r,K], B [N,r].
//
// Precision: every decision that yields an integer (a code) is taken in fp32
// exactly as written (a correctly rounded fp32 division, subtraction, product
// or sum, obtained here by computing in fp64 and rounding once, which is exact
// for a single operation on fp32 operands); every matmul is accumulated in
// fp64 from the exact bf16/fp32 input values.
#include <omp.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

// ---------------------------------------------------------------- scalars --

inline float bits_to_f32(uint32_t u) { float f; std::memcpy(&f, &u, 4); return f; }
inline uint32_t f32_to_bits(float f) { uint32_t u; std::memcpy(&u, &f, 4); return u; }

// bf16 = the upper 16 bits of an fp32; rounding is to nearest, ties to even.
inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u = f32_to_bits(f);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0)
        return 0x7fc0;                                  // quiet NaN
    uint32_t lsb = (u >> 16) & 1u;
    return (uint16_t)((u + 0x7fffu + lsb) >> 16);
}
inline double bf16_to_f64(uint16_t h) { return (double)bits_to_f32((uint32_t)h << 16); }

// Correctly rounded fp32 operations (single fp64 operation then one rounding).
inline float f32_div(float a, float b) { return (float)((double)a / (double)b); }
inline float f32_sub(float a, float b) { return (float)((double)a - (double)b); }
inline float f32_mul(float a, float b) { return (float)((double)a * (double)b); }
inline float f32_add(float a, float b) { return (float)((double)a + (double)b); }

// Inverse of the standard normal CDF: Wichura, "Algorithm AS 241: The
// percentage points of the normal distribution", Applied Statistics 37(3),
// 1988 (PPND16, about 1e-16 relative accuracy).
double ppnd16(double p) {
    const double q = p - 0.5;
    if (std::fabs(q) <= 0.425) {
        const double r = 0.180625 - q * q;
        const double num =
            (((((((2509.0809287301226727 * r + 33430.575583588128105) * r +
                  67265.770927008700853) * r + 45921.953931549871457) * r +
                13731.693765509461125) * r + 1971.5909503065514427) * r +
              133.14166789178437745) * r + 3.387132872796366608);
        const double den =
            (((((((5226.495278852545925 * r + 28729.085735721942674) * r +
                  39307.89580009271061) * r + 21213.794301586595867) * r +
                5394.1960214247511077) * r + 687.1870074920579083) * r +
              42.313330701600911252) * r + 1.0);
        return q * num / den;
    }
    double r = (q < 0.0) ? p : 1.0 - p;
    r = std::sqrt(-std::log(r));
    double val;
    if (r <= 5.0) {
        r -= 1.6;
        const double num =
            (((((((7.7454501427834140764e-4 * r + 0.0227238449892691845833) * r +
                  0.24178072517745061177) * r + 1.27045825245236838258) * r +
                3.64784832476320460504) * r + 5.7694972214606914055) * r +
              4.6303378461565452959) * r + 1.42343711074968357734);
        const double den =
            (((((((1.05075007164441684324e-9 * r + 5.475938084995344946e-4) * r +
                  0.0151986665636164571966) * r + 0.14810397642748007459) * r +
                0.68976733498510000455) * r + 1.6763848301838038494) * r +
              2.05319162663775882187) * r + 1.0);
        val = num / den;
    } else {
        r -= 5.0;
        const double num =
            (((((((2.01033439929228813265e-7 * r + 2.71155556874348757815e-5) * r +
                  0.0012426609473880784386) * r + 0.026532189526576123093) * r +
                0.29656057182850489123) * r + 1.7848265399172913358) * r +
              5.4637849111641143699) * r + 6.6579046435011037772);
        const double den =
            (((((((2.04426310338993978564e-15 * r + 1.4215117583164458887e-7) * r +
                  1.8463183175100546818e-5) * r + 7.868691311456132591e-4) * r +
                0.0148753612908506148525) * r + 0.13692988092273580531) * r +
              0.59983220655588793769) * r + 1.0);
        val = num / den;
    }
    return (q < 0.0) ? -val : val;
}

// READING (NF4 levels, QLoRA section 3): the quantile range is cut at
// p_max = 1 - (1/32 + 1/30)/2; positive levels are the quantiles of 8 equal
// steps from 1/2 to p_max, negative levels the negated quantiles of 7 equal
// steps, zero is added, the set is sorted and divided by its largest
// magnitude, then rounded once to fp32.
void build_nf4_levels(float out[16]) {
    const double p_max = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0);
    double lv[16];
    int n = 0;
    for (int j = 7; j >= 1; --j)                       // negatives, ascending
        lv[n++] = -ppnd16(0.5 + (p_max - 0.5) * j / 7.0);
    lv[n++] = 0.0;
    for (int j = 1; j <= 8; ++j)                       // positives, ascending
        lv[n++] = ppnd16(0.5 + (p_max - 0.5) * j / 8.0);
    double mx = 0.0;
    for (int i = 0; i < 16; ++i) mx = std::fmax(mx, std::fabs(lv[i]));
    for (int i = 0; i < 16; ++i) out[i] = (float)(lv[i] / mx);
}

// READING (second-level code): 255 linear signed levels k/127, k = -127..127,
// at index k + 127; index 255 is unused and holds 0.
void build_dq_table(float out[256]) {
    for (int k = -127; k <= 127; ++k) out[k + 127] = (float)((double)k / 127.0);
    out[255] = 0.0f;
}

// READING ("nearest level"): the level at the smallest exact distance from v,
// the lower index on a tie.  levels[0..n) ascending.  A plain scan.
int nearest_level(float v, const float* levels, int n) {
    int best = 0;
    double bd = std::fabs((double)v - (double)levels[0]);
    for (int i = 1; i < n; ++i) {
        double d = std::fabs((double)v - (double)levels[i]);
        if (d < bd) { bd = d; best = i; }
    }
    return best;
}

}  // namespace

extern "C" {

// ------------------------------------------------------------------ codec --

double orc_ppnd16(double p) { return ppnd16(p); }
void orc_nf4_codebook(float out[16]) { build_nf4_levels(out); }
void orc_dq_table(float out[256]) { build_dq_table(out); }
uint16_t orc_f32_to_bf16(float f) { return f32_to_bf16_rne(f); }
int orc_nearest_nf4(float v) { float c[16]; build_nf4_levels(c); return nearest_level(v, c, 16); }
int orc_nearest_dq(float v) { float t[256]; build_dq_table(t); return nearest_level(v, t, 255); }

// Number of first-level blocks (64 elements) and of second-level groups
// (256 blocks) of a weight with `numel` elements.
int64_t orc_nblocks(int64_t numel) { return numel / 64; }
int64_t orc_ngroups(int64_t numel) { return (numel / 64 + 255) / 256; }

// Quantise an fp32 weight (row-major, numel a multiple of 64) to NF4 with
// double-quantised absmax constants.
//   packed   [numel/2]   two 4-bit codes per byte, element 2j in the high nibble
//   absmax_q [nblk]      8-bit second-level codes
//   s2       [ngroups]   fp32 scale of each group of 256 blocks
//   offset   [1]         fp32 mean of all block absmax values
//   absmax   [nblk]      (optional, may be NULL) the exact first-level absmax
// Returns 0, or -1 for a non-finite input or numel not a multiple of 64.
int orc_nf4_quantize(const float* W, int64_t numel, uint8_t* packed, uint8_t* absmax_q,
                     float* s2, float* offset, float* absmax_out) {
    if (numel % 64 != 0) return -1;
    for (int64_t i = 0; i < numel; ++i)
        if (!std::isfinite(W[i])) return -1;
    float code[16];
    build_nf4_levels(code);
    float tab[256];
    build_dq_table(tab);
    const int64_t nblk = numel / 64;
    const int64_t ngrp = (nblk + 255) / 256;
    std::vector<float> absmax(nblk);
    std::vector<uint8_t> q(numel);

    // First level: per block of 64, absmax and the nearest level of w / absmax.
    for (int64_t b = 0; b < nblk; ++b) {
        float a = 0.0f;
        for (int i = 0; i < 64; ++i) a = std::fmax(a, std::fabs(W[b * 64 + i]));
        absmax[b] = a;
        for (int i = 0; i < 64; ++i) {
            if (a == 0.0f) { q[b * 64 + i] = 7; continue; }     // index of the zero level
            float v = f32_div(W[b * 64 + i], a);
            q[b * 64 + i] = (uint8_t)nearest_level(v, code, 16);
        }
    }
    for (int64_t j = 0; j < numel / 2; ++j)
        packed[j] = (uint8_t)((q[2 * j] << 4) | q[2 * j + 1]);

    // Second level.  READING: the offset is the mean of all absmax values,
    // summed in fp64 sequentially inside each group of 256 blocks, then the
    // group partials summed sequentially in group order, divided by the block
    // count and rounded to fp32.
    double total = 0.0;
    for (int64_t g = 0; g < ngrp; ++g) {
        double part = 0.0;
        for (int64_t b = g * 256; b < std::min<int64_t>(nblk, g * 256 + 256); ++b) part += (double)absmax[b];
        total += part;
    }
    const float off = (float)(total / (double)nblk);
    *offset = off;
    for (int64_t g = 0; g < ngrp; ++g) {
        const int64_t b0 = g * 256, b1 = std::min<int64_t>(nblk, g * 256 + 256);
        float sc = 0.0f;
        for (int64_t b = b0; b < b1; ++b) sc = std::fmax(sc, std::fabs(f32_sub(absmax[b], off)));
        s2[g] = sc;
        for (int64_t b = b0; b < b1; ++b) {
            if (sc == 0.0f) { absmax_q[b] = 127; continue; }      // index of the zero entry
            float v = f32_div(f32_sub(absmax[b], off), sc);
            absmax_q[b] = (uint8_t)nearest_level(v, tab, 255);
        }
    }
    if (absmax_out) std::memcpy(absmax_out, absmax.data(), sizeof(float) * nblk);
    return 0;
}

// Reconstructed absmax of block b: table[code] * s2 + offset, each operation
// rounded to fp32 separately (no fused multiply-add).
float orc_absmax_hat(const uint8_t* absmax_q, const float* s2, float offset, int64_t b) {
    float tab[256];
    build_dq_table(tab);
    return f32_add(f32_mul(tab[absmax_q[b]], s2[b / 256]), offset);
}

// Dequantise to bf16 bits: w = bf16_rne(fp32(level[q] * absmax_hat)).
void orc_nf4_dequant(const uint8_t* packed, const uint8_t* absmax_q, const float* s2, float offset,
                     int64_t numel, uint16_t* out) {
    float code[16];
    build_nf4_levels(code);
    float tab[256];
    build_dq_table(tab);
    for (int64_t b = 0; b < numel / 64; ++b) {
        const float ah = f32_add(f32_mul(tab[absmax_q[b]], s2[b / 256]), offset);
        for (int i = 0; i < 64; ++i) {
            const int64_t e = b * 64 + i;
            const uint8_t byte = packed[e / 2];
            const int qq = (e % 2 == 0) ? (byte >> 4) : (byte & 15);
            out[e] = f32_to_bf16_rne(f32_mul(code[qq], ah));
        }
    }
}

// ------------------------------------------------------------ LoRA linear --
//
// All tensors row-major.  x [T,K], W [N,K], A [r,K], B [N,r], dY [T,N] are
// bf16 bit patterns; s = alpha / r.  Results in fp64.
// `rows` (length nrows) selects the token rows of y / dX to compute; when
// rows is NULL every row 0..T-1 is computed and nrows is ignored.  The output
// of a selected row i goes to out[i * width].

// Forward: y = x W^T + s (x A^T) B^T.
void orc_lora_fwd(const uint16_t* x, const uint16_t* W, const uint16_t* A, const uint16_t* B,
                  int64_t T, int64_t K, int64_t N, int64_t r, double s,
                  const int64_t* rows, int64_t nrows, double* y) {
    const int64_t nr = rows ? nrows : T;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nr; ++i) {
        const int64_t t = rows ? rows[i] : i;
        std::vector<double> xt(K), u(r, 0.0);
        for (int64_t k = 0; k < K; ++k) xt[k] = bf16_to_f64(x[t * K + k]);
        for (int64_t j = 0; j < r; ++j)
            for (int64_t k = 0; k < K; ++k) u[j] += xt[k] * bf16_to_f64(A[j * K + k]);
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += xt[k] * bf16_to_f64(W[n * K + k]);
            double lo = 0.0;
            for (int64_t j = 0; j < r; ++j) lo += u[j] * bf16_to_f64(B[n * r + j]);
            y[i * N + n] = acc + s * lo;
        }
    }
}

// Backward input gradient: dX = dY W + s (dY B) A.
void orc_lora_bwd_dx(const uint16_t* dY, const uint16_t* W, const uint16_t* A, const uint16_t* B,
                     int64_t T, int64_t K, int64_t N, int64_t r, double s,
                     const int64_t* rows, int64_t nrows, double* dX) {
    const int64_t nr = rows ? nrows : T;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nr; ++i) {
        const int64_t t = rows ? rows[i] : i;
        std::vector<double> acc(K, 0.0), g(r, 0.0);
        for (int64_t n = 0; n < N; ++n) {
            const double d = bf16_to_f64(dY[t * N + n]);
            for (int64_t j = 0; j < r; ++j) g[j] += d * bf16_to_f64(B[n * r + j]);
            for (int64_t k = 0; k < K; ++k) acc[k] += d * bf16_to_f64(W[n * K + k]);
        }
        for (int64_t k = 0; k < K; ++k) {
            double lo = 0.0;
            for (int64_t j = 0; j < r; ++j) lo += g[j] * bf16_to_f64(A[j * K + k]);
            dX[i * K + k] = acc[k] + s * lo;
        }
    }
}

// Backward adapter gradients (full, every token contributes):
//   dA = s (dY B)^T x      [r,K]
//   dB = s dY^T (x A^T)    [N,r]
void orc_lora_bwd_dadb(const uint16_t* x, const uint16_t* dY, const uint16_t* A, const uint16_t* B,
                       int64_t T, int64_t K, int64_t N, int64_t r, double s,
                       double* dA, double* dB) {
    std::vector<double> g(T * r, 0.0), u(T * r, 0.0);
#pragma omp parallel for
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t j = 0; j < r; ++j) {
            double gg = 0.0, uu = 0.0;
            for (int64_t n = 0; n < N; ++n) gg += bf16_to_f64(dY[t * N + n]) * bf16_to_f64(B[n * r + j]);
            for (int64_t k = 0; k < K; ++k) uu += bf16_to_f64(x[t * K + k]) * bf16_to_f64(A[j * K + k]);
            g[t * r + j] = gg;
            u[t * r + j] = uu;
        }
    }
#pragma omp parallel for
    for (int64_t k = 0; k < K; ++k)
        for (int64_t j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t t = 0; t < T; ++t) acc += g[t * r + j] * bf16_to_f64(x[t * K + k]);
            dA[j * K + k] = s * acc;
        }
#pragma omp parallel for
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t t = 0; t < T; ++t) acc += bf16_to_f64(dY[t * N + n]) * u[t * r + j];
            dB[n * r + j] = s * acc;
        }
}

// Threads the parallel loops above use (OpenMP's count for this process).
int orc_threads() { return omp_get_max_threads(); }

}  // extern "C"
