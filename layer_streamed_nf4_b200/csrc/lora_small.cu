// The rank-r side of the LoRA linear ("Can You Fine-Tune a 27B Model on a
// Laptop? (I Did the Math)", 1:47-1:58: a thin pair of matrices bolted onto
// each layer):
//   down projection   u = x A^T  [T,r]   (forward; backward recomputes it)
//                     g = dY B   [T,r]   (backward)
//   token reductions  dA = s g^T x  [r,K],   dB = s dY^T u  [N,r]
// u and g are produced in fp32 (for dA/dB) and as bf16(s * .) (the extra
// K-block of the tensor-core contraction).  All sums run in a fixed order, so
// results are bitwise reproducible.
#include "common.cuh"

namespace lsn {

namespace {

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

constexpr int kDownRows = 4;   // token rows per warp
constexpr int kJ = 16;         // rank columns per pass

// Down projection out[t, j] = sum_k X[t, k] * Wt(j, k), j < r.
//   W_RK: Wt(j, k) = W[j * Kd + k]   (A, [r, K])
//   else: Wt(j, k) = W[k * r + j]    (B, [N, r])
// Each warp owns kDownRows token rows; lane l walks 8-element chunks
// l, l+32, ...; partial sums are combined by a warp butterfly.
template <bool W_RK>
__global__ void __launch_bounds__(128) lora_down_kernel(const uint16_t* __restrict__ X, const uint16_t* __restrict__ W,
                                                        int64_t T, int64_t Kd, int r, float scale,
                                                        float* __restrict__ u32, uint16_t* __restrict__ u16) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t t0 = warp * kDownRows;
    if (t0 >= T) return;
    const int64_t nch = Kd / 8;
    for (int j0 = 0; j0 < r; j0 += kJ) {
        const int nj = (r - j0 < kJ) ? (r - j0) : kJ;
        float acc[kDownRows][kJ];
        #pragma unroll
        for (int a = 0; a < kDownRows; ++a)
            #pragma unroll
            for (int j = 0; j < kJ; ++j) acc[a][j] = 0.0f;
        for (int64_t c = lane; c < nch; c += 32) {
            float xv[kDownRows][8];
            #pragma unroll
            for (int a = 0; a < kDownRows; ++a) {
                if (t0 + a < T) {
                    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(X + (t0 + a) * Kd) + c), xv[a]);
                } else {
                    #pragma unroll
                    for (int i = 0; i < 8; ++i) xv[a][i] = 0.0f;
                }
            }
            if (W_RK) {
                #pragma unroll
                for (int j = 0; j < kJ; ++j) {
                    if (j >= nj) break;
                    float wv[8];
                    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(W + (int64_t)(j0 + j) * Kd) + c), wv);
                    #pragma unroll
                    for (int a = 0; a < kDownRows; ++a)
                        #pragma unroll
                        for (int i = 0; i < 8; ++i) acc[a][j] = fmaf(xv[a][i], wv[i], acc[a][j]);
                }
            } else {
                #pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint16_t* row = W + (c * 8 + i) * (int64_t)r + j0;
                    #pragma unroll
                    for (int h = 0; h < kJ / 8; ++h) {
                        if (h * 8 >= nj) break;
                        float wv[8];
                        bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(row) + h), wv);
                        #pragma unroll
                        for (int a = 0; a < kDownRows; ++a)
                            #pragma unroll
                            for (int q = 0; q < 8; ++q) acc[a][h * 8 + q] = fmaf(xv[a][i], wv[q], acc[a][h * 8 + q]);
                    }
                }
            }
        }
        #pragma unroll
        for (int a = 0; a < kDownRows; ++a)
            #pragma unroll
            for (int j = 0; j < kJ; ++j)
                #pragma unroll
                for (int o = 16; o > 0; o >>= 1) acc[a][j] += __shfl_xor_sync(0xffffffffu, acc[a][j], o);
        #pragma unroll
        for (int a = 0; a < kDownRows; ++a) {
            if (t0 + a >= T) break;
            #pragma unroll
            for (int j = 0; j < kJ; ++j) {
                if (j < nj && lane == j) {
                    const int64_t o = (t0 + a) * r + j0 + j;
                    if (u32) u32[o] = acc[a][j];
                    if (u16) u16[o] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(scale, acc[a][j])));
                }
            }
        }
    }
}

constexpr int kTgCols = 64;     // output columns per CTA
constexpr int kTgWarps = 8;

// Token reduction R[j, k] = sum_{t in split} G[t, j] * X[t, k] for one tile of
// 64 columns k and one split of tokens.  Lane l owns columns 2l, 2l+1; warp w
// takes tokens w, w+8, ...; the eight warp partials are added in warp order.
// With one split the result is finished here (scale, optional accumulate);
// otherwise partial [split][r][Kd] is written for lora_tgrad_finish.
//   OUT_RK: out[j * Kd + k] (dA layout), else out[k * r + j] (dB layout).
template <bool OUT_RK>
__global__ void __launch_bounds__(256) lora_tgrad_kernel(const float* __restrict__ G, const uint16_t* __restrict__ X,
                                                         int64_t T, int64_t Kd, int r, int nsplit, float scale,
                                                         int accumulate, float* __restrict__ out,
                                                         float* __restrict__ partial) {
    __shared__ float red[kTgWarps][kJ][kTgCols + 1];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t k0 = (int64_t)blockIdx.x * kTgCols;
    const int split = blockIdx.y;
    const int64_t per = (T + nsplit - 1) / nsplit;
    const int64_t tb = split * per;
    const int64_t te = (tb + per < T) ? tb + per : T;
    for (int j0 = 0; j0 < r; j0 += kJ) {
        const int nj = (r - j0 < kJ) ? (r - j0) : kJ;
        float acc[kJ][2];
        #pragma unroll
        for (int j = 0; j < kJ; ++j) acc[j][0] = acc[j][1] = 0.0f;
        for (int64_t t = tb + warp; t < te; t += kTgWarps) {
            const uint32_t xp = __ldg(reinterpret_cast<const uint32_t*>(X + t * Kd + k0) + lane);
            const float x0 = __uint_as_float(xp << 16), x1 = __uint_as_float(xp & 0xffff0000u);
            const float* grow = G + t * r + j0;
            #pragma unroll
            for (int j = 0; j < kJ; ++j) {
                if (j >= nj) break;
                const float gv = __ldg(grow + j);
                acc[j][0] = fmaf(gv, x0, acc[j][0]);
                acc[j][1] = fmaf(gv, x1, acc[j][1]);
            }
        }
        #pragma unroll
        for (int j = 0; j < kJ; ++j) {
            red[warp][j][2 * lane] = acc[j][0];
            red[warp][j][2 * lane + 1] = acc[j][1];
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < nj * kTgCols; idx += blockDim.x) {
            const int j = idx / kTgCols, c = idx % kTgCols;
            float s = 0.0f;
            #pragma unroll
            for (int w = 0; w < kTgWarps; ++w) s += red[w][j][c];
            const int64_t k = k0 + c;
            if (nsplit == 1) {
                const int64_t o = OUT_RK ? (int64_t)(j0 + j) * Kd + k : k * r + (j0 + j);
                const float v = __fmul_rn(scale, s);
                out[o] = accumulate ? __fadd_rn(out[o], v) : v;
            } else {
                partial[((int64_t)split * r + (j0 + j)) * Kd + k] = s;
            }
        }
        __syncthreads();
    }
}

// Sum the split partials in split order, scale, optionally accumulate.
template <bool OUT_RK>
__global__ void lora_tgrad_finish(const float* __restrict__ partial, int64_t Kd, int r, int nsplit, float scale,
                                  int accumulate, float* __restrict__ out) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)r * Kd) return;
    const int64_t j = idx / Kd, k = idx % Kd;
    float s = 0.0f;
    for (int sp = 0; sp < nsplit; ++sp) s += partial[(int64_t)sp * r * Kd + idx];
    const int64_t o = OUT_RK ? idx : k * r + j;
    const float v = __fmul_rn(scale, s);
    out[o] = accumulate ? __fadd_rn(out[o], v) : v;
}

}  // namespace

// Number of token splits of a reduction over T tokens into Kd/64 column
// tiles: enough CTAs for two per SM of a 148-SM part, at least 128 tokens per
// split.  Depends on the shape only, so results do not depend on the device.
int tgrad_splits(int64_t T, int64_t Kd) {
    const int64_t tiles = Kd / kTgCols;
    int64_t s = (296 + tiles - 1) / tiles;
    const int64_t by_t = (T + 127) / 128;
    if (s > by_t) s = by_t;
    if (s > 32) s = 32;
    if (s < 1) s = 1;
    return (int)s;
}

size_t tgrad_ws_bytes(int64_t T, int64_t Kd, int r) {
    const int s = tgrad_splits(T, Kd);
    return s > 1 ? (size_t)s * r * Kd * sizeof(float) : 0;
}

lsn_status launch_lora_down(const uint16_t* X, const uint16_t* W, bool w_rk, int64_t T, int64_t Kd, int r,
                            float scale, float* u32, uint16_t* u16, cudaStream_t st) {
    if (T == 0) return LSN_OK;
    const int64_t warps = (T + kDownRows - 1) / kDownRows;
    const int grid = (int)((warps + 3) / 4);
    if (w_rk)
        lora_down_kernel<true><<<grid, 128, 0, st>>>(X, W, T, Kd, r, scale, u32, u16);
    else
        lora_down_kernel<false><<<grid, 128, 0, st>>>(X, W, T, Kd, r, scale, u32, u16);
    LSN_CUDA_TRY(cudaGetLastError());
    return LSN_OK;
}

lsn_status launch_lora_tgrad(const float* G, const uint16_t* X, bool out_rk, int64_t T, int64_t Kd, int r,
                             float scale, int accumulate, float* out, float* partial, cudaStream_t st) {
    const int ns = tgrad_splits(T, Kd);
    dim3 grid((unsigned)(Kd / kTgCols), (unsigned)ns);
    if (out_rk)
        lora_tgrad_kernel<true><<<grid, 256, 0, st>>>(G, X, T, Kd, r, ns, scale, accumulate, out, partial);
    else
        lora_tgrad_kernel<false><<<grid, 256, 0, st>>>(G, X, T, Kd, r, ns, scale, accumulate, out, partial);
    if (ns > 1) {
        const int64_t n = (int64_t)r * Kd;
        if (out_rk)
            lora_tgrad_finish<true><<<(int)ceil_div(n, 256), 256, 0, st>>>(partial, Kd, r, ns, scale, accumulate, out);
        else
            lora_tgrad_finish<false><<<(int)ceil_div(n, 256), 256, 0, st>>>(partial, Kd, r, ns, scale, accumulate, out);
    }
    LSN_CUDA_TRY(cudaGetLastError());
    return LSN_OK;
}

}  // namespace lsn
