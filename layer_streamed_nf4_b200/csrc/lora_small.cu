// The rank-r side of the LoRA linear ("Can You Fine-Tune a 27B Model on a
// Laptop? (I Did the Math)", 1:47-1:58: a thin pair of matrices bolted onto
// each layer):
//   down projection   u = x A^T  [T,r]   (forward; backward recomputes it)
//                     g = dY B   [T,r]   (backward)
//   token reductions  dA = s g^T x  [r,K],   dB = s dY^T u  [N,r]
// u and g are produced in fp32 (for dA/dB) and as bf16(s * .) (the extra
// K-block of the tensor-core contraction).  Both kernels are bound by the
// HBM read of the activation (x or dY); every sum runs in a fixed order that
// depends on the shape only, so results are bitwise reproducible.
#include "common.cuh"

namespace lsn {

namespace {

// ----------------------------------------------------------- down proj ---
//
// out[t, j] = sum_k X[t, k] * W[j, k] for j < r (W row-major [r, Kd]; the
// backward's B [N, r] is first transposed into that layout).  A CTA owns 64
// token rows and one split of the K range; 64-wide K chunks of X and W are
// staged in shared memory by cp.async through a 4-stage ring (rows padded to
// 144 bytes so ldmatrix is conflict-free), and each warp multiplies its 16
// rows with W on the warp-level tensor-core instruction (mma.sync m16n8k16,
// bf16 in, fp32 accumulate): the inputs are exact bf16 values, so this is the
// exact product rounded only by fp32 accumulation.  The big contractions use
// tcgen05; this skinny one is bound by the HBM read of X.
constexpr int kDnWarps = 4;
constexpr int kDnRows = 16 * kDnWarps;       // token rows per CTA
constexpr int kDnStages = 4;
constexpr int kDnPitch = 72;                 // bf16 per staged row (64 + 8 padding)

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t saddr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(saddr));
}

// 16-byte global -> shared copy; src_bytes == 0 writes zeros.
__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* gptr, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr), "l"(gptr), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int NT>   // NT n-tiles of 8 rank columns: r = 8 * NT
__global__ void __launch_bounds__(128) lora_down_kernel(const uint16_t* __restrict__ X, const uint16_t* __restrict__ W,
                                                        int64_t T, int64_t Kd, int chunks_per_split, float scale,
                                                        float* __restrict__ u32, uint16_t* __restrict__ u16,
                                                        float* __restrict__ partial) {
    constexpr int R = 8 * NT;
    constexpr int NP = (NT + 1) / 2;          // n-tile pairs (W rows padded to 16 * NP with zeros)
    constexpr int WR = 16 * NP;
    extern __shared__ __align__(16) uint8_t dn_smem[];
    auto xs = reinterpret_cast<uint16_t (*)[kDnRows][kDnPitch]>(dn_smem);
    auto ws = reinterpret_cast<uint16_t (*)[WR][kDnPitch]>(dn_smem + sizeof(uint16_t) * kDnStages * kDnRows * kDnPitch);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t row_base = (int64_t)blockIdx.x * kDnRows;
    const int64_t nchunks = Kd / 64;
    const int64_t c_begin = (int64_t)blockIdx.y * chunks_per_split;
    const int64_t c_end = (c_begin + chunks_per_split < nchunks) ? c_begin + chunks_per_split : nchunks;
    const int64_t nc = c_end > c_begin ? c_end - c_begin : 0;

    auto load = [&](int stage, int64_t c) {
        // X: 64 rows x 128 bytes = 512 pieces of 16 bytes, 4 per thread.
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int p = tid + i * 128, row = p >> 3, piece = p & 7;
            const int64_t t = row_base + row;
            const bool ok = t < T;
            const uint16_t* src = X + (ok ? t : 0) * Kd + c * 64 + piece * 8;
            cp_async16(smem_u32(&xs[stage][row][piece * 8]), src, ok ? 16u : 0u);
        }
        // W: WR rows x 128 bytes; rows >= R are zero.
        for (int p = tid; p < WR * 8; p += 128) {
            const int row = p >> 3, piece = p & 7;
            const bool ok = row < R;
            const uint16_t* src = W + (int64_t)(ok ? row : 0) * Kd + c * 64 + piece * 8;
            cp_async16(smem_u32(&ws[stage][row][piece * 8]), src, ok ? 16u : 0u);
        }
    };

    float acc[2 * NP][4];
    #pragma unroll
    for (int n = 0; n < 2 * NP; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;

    #pragma unroll
    for (int s = 0; s < kDnStages - 1; ++s) {
        if (s < nc) load(s, c_begin + s);
        cp_async_commit();
    }
    // ldmatrix row addresses: A (16 rows of the warp, 16 columns), B (16 W rows, 16 columns).
    const int a_row = warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
    const int a_col = 8 * (lane >> 4);
    const int b_row = (lane & 7) + 8 * (lane >> 4);
    const int b_col = 8 * ((lane >> 3) & 1);
    for (int64_t i = 0; i < nc; ++i) {
        cp_async_wait<kDnStages - 2>();
        __syncthreads();
        const int st = (int)(i % kDnStages);
        #pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(smem_u32(&xs[st][a_row][ks * 16 + a_col]), a0, a1, a2, a3);
            #pragma unroll
            for (int p = 0; p < NP; ++p) {
                uint32_t b00, b01, b10, b11;
                ldmatrix_x4(smem_u32(&ws[st][p * 16 + b_row][ks * 16 + b_col]), b00, b01, b10, b11);
                mma_bf16_16816(acc[2 * p], a0, a1, a2, a3, b00, b01);
                mma_bf16_16816(acc[2 * p + 1], a0, a1, a2, a3, b10, b11);
            }
        }
        // Refill the stage consumed one iteration ago (all warps are past it).
        const int64_t nxt = i + kDnStages - 1;
        if (nxt < nc) load((int)(nxt % kDnStages), c_begin + nxt);
        cp_async_commit();
    }
    cp_async_wait<0>();

    // acc[n] = { (row g, col 8n+2q), (row g, col 8n+2q+1), (row g+8, ...), (row g+8, ...) }
    const int g = lane >> 2, q = lane & 3;
    const int64_t row0 = row_base + warp * 16 + g, row1 = row0 + 8;
    const bool ok0 = row0 < T, ok1 = row1 < T;
    #pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int j = n * 8 + 2 * q;
        if (partial != nullptr) {
            float* pp = partial + (int64_t)blockIdx.y * T * R;
            if (ok0) { pp[row0 * R + j] = acc[n][0]; pp[row0 * R + j + 1] = acc[n][1]; }
            if (ok1) { pp[row1 * R + j] = acc[n][2]; pp[row1 * R + j + 1] = acc[n][3]; }
        } else {
            if (ok0) {
                if (u32) { u32[row0 * R + j] = acc[n][0]; u32[row0 * R + j + 1] = acc[n][1]; }
                if (u16) {
                    u16[row0 * R + j] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(scale, acc[n][0])));
                    u16[row0 * R + j + 1] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(scale, acc[n][1])));
                }
            }
            if (ok1) {
                if (u32) { u32[row1 * R + j] = acc[n][2]; u32[row1 * R + j + 1] = acc[n][3]; }
                if (u16) {
                    u16[row1 * R + j] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(scale, acc[n][2])));
                    u16[row1 * R + j + 1] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(scale, acc[n][3])));
                }
            }
        }
    }
}

// Sum the K-split partials of the down projection in split order.
__global__ void lora_down_finish(const float* __restrict__ partial, int64_t n, int nsplit, float scale,
                                 float* __restrict__ u32, uint16_t* __restrict__ u16) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    float s = 0.0f;
    for (int k = 0; k < nsplit; ++k) s += partial[(int64_t)k * n + i];
    if (u32) u32[i] = s;
    if (u16) u16[i] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(scale, s)));
}

// B [N, r] -> Bt [r, N] (bf16), so the backward's g = dY B uses the same
// down-projection kernel as u = x A^T.
__global__ void transpose_nr_kernel(const uint16_t* __restrict__ B, int64_t N, int r, uint16_t* __restrict__ Bt) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= N * r) return;
    const int64_t n = i / r, j = i % r;
    Bt[j * N + n] = B[i];
}

// -------------------------------------------------------- token reduce ---
//
// R[j, k] = sum_{t in split} G[t, j] * X[t, k].  A CTA owns 128 columns k
// (lane l owns k0 + 4l .. 4l+3) and one split of the tokens, staged 32
// tokens at a time (X tile 32 x 128 bf16, G tile 32 x NJ fp32) by cp.async
// through a 4-stage ring; its four warps take tokens w, w+4, ... of each tile
// and keep NJ x 4 fp32 accumulators per lane (register-resident: all indices
// are compile-time constants), reading G rows as broadcast 16-byte loads.
// The four warp partials are added in warp order.  With one split the result
// is finished here (scale, optional accumulate); otherwise partial
// [split][r][Kd] is written and summed in split order by lora_tgrad_finish.
constexpr int kTgCols = 128;
constexpr int kTgWarps = 4;
constexpr int kTgTok = 32;          // tokens per staged tile
constexpr int kTgStages = 4;

template <int NJ, bool OUT_RK>
__global__ void __launch_bounds__(128) lora_tgrad_kernel(const float* __restrict__ G, const uint16_t* __restrict__ X,
                                                         int64_t T, int64_t Kd, int r, int j0, int64_t per_split,
                                                         int nsplit, float scale, int accumulate,
                                                         float* __restrict__ out, float* __restrict__ partial) {
    // Dynamic shared memory: the staging ring, later reused for the warp
    // partials (red) once every copy has landed.
    extern __shared__ __align__(16) uint8_t tg_smem[];
    auto xs = reinterpret_cast<uint16_t (*)[kTgTok][kTgCols]>(tg_smem);
    auto gs = reinterpret_cast<float (*)[kTgTok][NJ]>(tg_smem + sizeof(uint16_t) * kTgStages * kTgTok * kTgCols);
    auto red = reinterpret_cast<float (*)[NJ][kTgCols + 4]>(tg_smem);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t k0 = (int64_t)blockIdx.x * kTgCols;
    const int split = blockIdx.y;
    const int64_t tb = split * per_split;
    const int64_t te = (tb + per_split < T) ? tb + per_split : T;
    const int64_t ntiles = te > tb ? (te - tb + kTgTok - 1) / kTgTok : 0;

    auto load = [&](int stage, int64_t tile) {
        const int64_t t0 = tb + tile * kTgTok;
        // X: 32 rows x 256 bytes = 512 pieces, 4 per thread.
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int p = tid + i * 128, row = p >> 4, piece = p & 15;
            const int64_t t = t0 + row, k = k0 + piece * 8;
            const bool ok = t < te && k < Kd;
            const uint16_t* src = X + (ok ? t : 0) * Kd + (ok ? k : 0);
            cp_async16(smem_u32(&xs[stage][row][piece * 8]), src, ok ? 16u : 0u);
        }
        // G: 32 rows x NJ floats (NJ/4 pieces per row).
        for (int p = tid; p < kTgTok * (NJ / 4); p += 128) {
            const int row = p / (NJ / 4), piece = p % (NJ / 4);
            const int64_t t = t0 + row;
            const bool ok = t < te && j0 + piece * 4 < r;
            const float* src = G + (ok ? t : 0) * r + (ok ? j0 + piece * 4 : 0);
            cp_async16(smem_u32(&gs[stage][row][piece * 4]), src, ok ? 16u : 0u);
        }
    };

    float acc[NJ][4];
    #pragma unroll
    for (int j = 0; j < NJ; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;

    #pragma unroll
    for (int s = 0; s < kTgStages - 1; ++s) {
        if (s < ntiles) load(s, s);
        cp_async_commit();
    }
    for (int64_t i = 0; i < ntiles; ++i) {
        cp_async_wait<kTgStages - 2>();
        __syncthreads();
        const int st = (int)(i % kTgStages);
        #pragma unroll 2
        for (int tt = warp; tt < kTgTok; tt += kTgWarps) {
            const uint2 xp = *reinterpret_cast<const uint2*>(&xs[st][tt][4 * lane]);
            const float x0 = __uint_as_float(xp.x << 16), x1 = __uint_as_float(xp.x & 0xffff0000u);
            const float x2 = __uint_as_float(xp.y << 16), x3 = __uint_as_float(xp.y & 0xffff0000u);
            #pragma unroll
            for (int j4 = 0; j4 < NJ; j4 += 4) {
                const float4 gv = *reinterpret_cast<const float4*>(&gs[st][tt][j4]);
                const float gg[4] = {gv.x, gv.y, gv.z, gv.w};
                #pragma unroll
                for (int u = 0; u < 4; ++u) {
                    acc[j4 + u][0] = fmaf(gg[u], x0, acc[j4 + u][0]);
                    acc[j4 + u][1] = fmaf(gg[u], x1, acc[j4 + u][1]);
                    acc[j4 + u][2] = fmaf(gg[u], x2, acc[j4 + u][2]);
                    acc[j4 + u][3] = fmaf(gg[u], x3, acc[j4 + u][3]);
                }
            }
        }
        const int64_t nxt = i + kTgStages - 1;
        if (nxt < ntiles) load((int)(nxt % kTgStages), nxt);
        cp_async_commit();
    }
    cp_async_wait<0>();
    __syncthreads();                          // staging ring is dead from here on
    #pragma unroll
    for (int j = 0; j < NJ; ++j)
        #pragma unroll
        for (int c = 0; c < 4; ++c) red[warp][j][4 * lane + c] = acc[j][c];
    __syncthreads();
    const int nj = (r - j0 < NJ) ? (r - j0) : NJ;
    for (int idx = tid; idx < nj * kTgCols; idx += blockDim.x) {
        const int j = idx / kTgCols, c = idx % kTgCols;
        const int64_t k = k0 + c;
        if (k >= Kd) continue;
        float s = 0.0f;
        #pragma unroll
        for (int w = 0; w < kTgWarps; ++w) s += red[w][j][c];
        if (nsplit == 1) {
            const int64_t o = OUT_RK ? (int64_t)(j0 + j) * Kd + k : k * r + (j0 + j);
            const float v = __fmul_rn(scale, s);
            out[o] = accumulate ? __fadd_rn(out[o], v) : v;
        } else {
            partial[((int64_t)split * r + (j0 + j)) * Kd + k] = s;
        }
    }
}

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

template <int NT>
constexpr size_t down_smem_bytes() {
    return sizeof(uint16_t) * kDnStages * (kDnRows + 16 * ((NT + 1) / 2)) * kDnPitch;
}

template <int NJ>
constexpr size_t tgrad_smem_bytes() {
    const size_t ring = sizeof(uint16_t) * kTgStages * kTgTok * kTgCols + sizeof(float) * kTgStages * kTgTok * NJ;
    const size_t red = sizeof(float) * kTgWarps * NJ * (kTgCols + 4);
    return ring > red ? ring : red;
}

// Opt a kernel into its dynamic shared-memory size once.
template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int NT>
lsn_status launch_down_nt(dim3 grid, cudaStream_t st, const uint16_t* X, const uint16_t* W, int64_t T, int64_t Kd,
                          int cps, float scale, float* u32, uint16_t* u16, float* part) {
    static const cudaError_t attr = allow_smem(lora_down_kernel<NT>, down_smem_bytes<NT>());
    if (attr != cudaSuccess) return fail_cuda(attr, "cudaFuncSetAttribute(lora_down smem)");
    lora_down_kernel<NT><<<grid, 128, down_smem_bytes<NT>(), st>>>(X, W, T, Kd, cps, scale, u32, u16, part);
    return LSN_OK;
}

template <int NJ, bool OUT_RK>
lsn_status launch_tgrad_nj(dim3 grid, cudaStream_t st, const float* G, const uint16_t* X, int64_t T, int64_t Kd, int r,
                           int j0, int64_t per, int ns, float scale, int accumulate, float* out, float* partial) {
    static const cudaError_t attr = allow_smem(lora_tgrad_kernel<NJ, OUT_RK>, tgrad_smem_bytes<NJ>());
    if (attr != cudaSuccess) return fail_cuda(attr, "cudaFuncSetAttribute(lora_tgrad smem)");
    lora_tgrad_kernel<NJ, OUT_RK><<<grid, 128, tgrad_smem_bytes<NJ>(), st>>>(G, X, T, Kd, r, j0, per, ns, scale,
                                                                             accumulate, out, partial);
    return LSN_OK;
}

}  // namespace

// ----------------------------------------------------------- planning ---
// Split counts depend on the shape only (never on the device or pointers), so
// a given shape always sums in the same order.

// K-splits of the down projection: about four 128-thread CTAs per SM of a
// 148-SM part, at least eight 64-wide chunks per split.
int down_splits(int64_t T, int64_t Kd) {
    const int64_t row_blocks = (T + kDnRows - 1) / kDnRows;
    if (row_blocks <= 0 || Kd < 64) return 1;
    const int64_t chunks = Kd / 64;
    int64_t s = (592 + row_blocks - 1) / row_blocks;
    const int64_t cap = chunks / 8 > 0 ? chunks / 8 : 1;
    if (s > cap) s = cap;
    if (s < 1) s = 1;
    return (int)s;
}

size_t down_ws_bytes(int64_t T, int64_t Kd, int r) {
    const int s = down_splits(T, Kd);
    return s > 1 ? (size_t)s * T * r * sizeof(float) : 0;
}

// Token splits of a reduction: about two 128-thread CTAs per SM of a 148-SM
// part, at least 128 tokens per split.
int tgrad_splits(int64_t T, int64_t Kd) {
    const int64_t tiles = (Kd + kTgCols - 1) / kTgCols;
    if (tiles <= 0 || T <= 0) return 1;
    int64_t s = (296 + tiles - 1) / tiles;
    const int64_t by_t = (T + 127) / 128;
    if (s > by_t) s = by_t;
    if (s > 64) s = 64;
    if (s < 1) s = 1;
    return (int)s;
}

size_t tgrad_ws_bytes(int64_t T, int64_t Kd, int r) {
    const int s = tgrad_splits(T, Kd);
    return s > 1 ? (size_t)s * r * Kd * sizeof(float) : 0;
}

// X [T, Kd] times W: w_rk ? W is A [r, Kd] : W is B [Kd, r] (transposed into
// `wt` [r, Kd] first).  `partial` must hold down_ws_bytes(T, Kd, r).
lsn_status launch_lora_down(const uint16_t* X, const uint16_t* W, bool w_rk, int64_t T, int64_t Kd, int r,
                            float scale, float* u32, uint16_t* u16, uint16_t* wt, float* partial, cudaStream_t st) {
    if (T == 0) return LSN_OK;
    if (!w_rk) {
        const int64_t n = Kd * r;
        transpose_nr_kernel<<<(int)ceil_div(n, 256), 256, 0, st>>>(W, Kd, r, wt);
        W = wt;
    }
    const int ns = down_splits(T, Kd);
    const int64_t chunks = Kd / 64;
    const int cps = (int)((chunks + ns - 1) / ns);
    dim3 grid((unsigned)((T + kDnRows - 1) / kDnRows), (unsigned)ns);
    float* part = ns > 1 ? partial : nullptr;
    lsn_status ls;
    switch (r / 8) {
        case 1: ls = launch_down_nt<1>(grid, st, X, W, T, Kd, cps, scale, u32, u16, part); break;
        case 2: ls = launch_down_nt<2>(grid, st, X, W, T, Kd, cps, scale, u32, u16, part); break;
        case 3: ls = launch_down_nt<3>(grid, st, X, W, T, Kd, cps, scale, u32, u16, part); break;
        case 4: ls = launch_down_nt<4>(grid, st, X, W, T, Kd, cps, scale, u32, u16, part); break;
        case 5: ls = launch_down_nt<5>(grid, st, X, W, T, Kd, cps, scale, u32, u16, part); break;
        case 6: ls = launch_down_nt<6>(grid, st, X, W, T, Kd, cps, scale, u32, u16, part); break;
        case 7: ls = launch_down_nt<7>(grid, st, X, W, T, Kd, cps, scale, u32, u16, part); break;
        case 8: ls = launch_down_nt<8>(grid, st, X, W, T, Kd, cps, scale, u32, u16, part); break;
        default: return fail(LSN_ERR_INVALID_ARG, "rank must be a multiple of 8 in [8, 64]");
    }
    if (ls != LSN_OK) return ls;
    if (ns > 1) {
        const int64_t n = T * r;
        lora_down_finish<<<(int)ceil_div(n, 256), 256, 0, st>>>(partial, n, ns, scale, u32, u16);
    }
    LSN_CUDA_TRY(cudaGetLastError());
    return LSN_OK;
}

lsn_status launch_lora_tgrad(const float* G, const uint16_t* X, bool out_rk, int64_t T, int64_t Kd, int r,
                             float scale, int accumulate, float* out, float* partial, cudaStream_t st) {
    const int ns = tgrad_splits(T, Kd);
    const int64_t per = ((T + ns - 1) / ns + 15) / 16 * 16;
    dim3 grid((unsigned)((Kd + kTgCols - 1) / kTgCols), (unsigned)ns);
    for (int j0 = 0; j0 < r; j0 += 16) {
        const bool wide = r - j0 > 8;
        lsn_status ls;
        if (out_rk)
            ls = wide ? launch_tgrad_nj<16, true>(grid, st, G, X, T, Kd, r, j0, per, ns, scale, accumulate, out, partial)
                      : launch_tgrad_nj<8, true>(grid, st, G, X, T, Kd, r, j0, per, ns, scale, accumulate, out, partial);
        else
            ls = wide ? launch_tgrad_nj<16, false>(grid, st, G, X, T, Kd, r, j0, per, ns, scale, accumulate, out, partial)
                      : launch_tgrad_nj<8, false>(grid, st, G, X, T, Kd, r, j0, per, ns, scale, accumulate, out, partial);
        if (ls != LSN_OK) return ls;
    }
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
