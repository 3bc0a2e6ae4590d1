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
#include "launch.cuh"

namespace lsn {

namespace {

// ------------------------------------------------------------- helpers ---

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t saddr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(saddr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t saddr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
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

// Two bf16 values packed low/high into one register.
__device__ __forceinline__ uint32_t pack2(float lo, float hi) { return pack_bf16x2(lo, hi); }

// Split reductions inside a thread-block cluster: the CTAs of one output tile
// (one per K- or token-split, cluster rank = split index) each leave their
// partial tile in shared memory; after a cluster barrier, CTA y adds slice y
// of the tile over ranks 0, 1, ..., S-1 in that order, reading the other
// CTAs' shared memory directly (DSMEM).  The order depends on the shape only.
__device__ __forceinline__ float ld_dsmem_f32(const float* local_ptr, uint32_t rank) {
    float v;
    const uint32_t a = mapa_shared(smem_u32(local_ptr), rank);
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
    return v;
}

// ----------------------------------------------------------- down proj ---
//
// out[t, j] = sum_k X[t, k] * Wt(j, k) for j < r, with W given either as
// A [r, Kd] (u = x A^T) or as B [Kd, r] (g = dY B).  A CTA owns 64 token rows
// and one split of the K range; 64-wide K chunks of X and W are staged in
// shared memory by cp.async through a 3-stage ring (16-byte chunks XOR-
// swizzled by row, so ldmatrix is conflict-free without padding), and each
// warp multiplies its 16 rows with W on the warp-level tensor-core
// instruction (mma.sync m16n8k16, bf16 in, fp32 accumulate; the inputs are
// exact bf16 values).  W in the B layout is read
// with ldmatrix.trans, so no transposed copy is made.  The big contractions
// use tcgen05; this skinny one is bound by the HBM read of X.
//
// At r = 16 the ring takes 30 KB, small enough for one CTA to share an SM
// with a running GEMM CTA (about 194 KB), so the side work of one
// projection can proceed underneath another projection's GEMM when the
// caller issues them on two streams.
//
// One launch serves a batch of up to kMaxProbs problems of the same rank and
// W layout (the projections of a layer): blockIdx.x runs over the row blocks
// of all problems, blockIdx.y is the split, and a problem with fewer splits
// than the launch leaves its extra CTAs without work.  Each problem keeps
// the split count and summation order it has when launched alone.
constexpr int kDnWarps = 4;
constexpr int kDnRows = 16 * kDnWarps;       // token rows per CTA
constexpr int kDnStages = 3;
constexpr int kMaxProbs = 16;

struct DownProb {
    const uint16_t* X;   // [T, Kd]
    const uint16_t* W;   // A [r, Kd] or B [Kd, r]
    float* u32;          // [T, r] fp32, or NULL
    uint16_t* u16;       // [T, r] bf16(scale * .), or NULL
    int64_t T, Kd;
    int cps, ns;         // 64-wide K chunks per split, splits
    int first;           // first blockIdx.x of the problem
    int ld16;            // row stride of u16
    float scale;
};
struct DownBatch {
    int n;
    DownProb p[kMaxProbs];
};

// Offset (in bf16) of element (row, col) of a staged tile whose rows hold
// `pitch` bf16, with the 16-byte chunk index XOR-ed by `swz`.
__device__ __forceinline__ int swz_off(int row, int col, int pitch, int swz) {
    return row * pitch + (((col >> 3) ^ swz) << 3) + (col & 7);
}

template <int NT, bool B_KR>
struct DownSmem {
    static constexpr int R = 8 * NT;
    static constexpr int NP = (NT + 1) / 2;                       // n-tile pairs
    static constexpr int WROWS = B_KR ? 64 : 16 * NP;             // staged W rows
    // B [Kd, r] rows hold 16*NP rank columns: 32, 64 or 128 bytes, swizzled
    // so eight consecutive rows hit distinct banks; 96-byte rows are padded.
    static constexpr int WPITCH = B_KR ? (NP == 3 ? 16 * NP + 8 : 16 * NP) : 64;
    static constexpr int X_TILE = kDnRows * 64;                   // bf16 per X stage
    static constexpr int W_TILE = WROWS * WPITCH;                 // bf16 per W stage
    static constexpr size_t X_BYTES = sizeof(uint16_t) * kDnStages * X_TILE;
    static constexpr size_t W_BYTES = sizeof(uint16_t) * kDnStages * W_TILE;
    static constexpr size_t RING = X_BYTES + W_BYTES;
    static constexpr size_t RED = sizeof(float) * kDnRows * R;
    static constexpr size_t BYTES = RING > RED ? RING : RED;
    // chunk swizzle of a staged W row
    __device__ static __forceinline__ int wswz(int row) {
        if (!B_KR) return row & 7;
        return NP == 1 ? (row >> 2) & 1 : NP == 2 ? (row >> 1) & 3 : NP == 4 ? row & 7 : 0;
    }
};

template <int NT, bool B_KR>
__global__ void __launch_bounds__(128) lora_down_kernel(const __grid_constant__ DownBatch bt) {
    using L = DownSmem<NT, B_KR>;
    int pi = 0;
    while (pi + 1 < bt.n && (int)blockIdx.x >= bt.p[pi + 1].first) ++pi;
    const DownProb& pb = bt.p[pi];
    const uint16_t* __restrict__ X = pb.X;
    const uint16_t* __restrict__ W = pb.W;
    float* __restrict__ u32 = pb.u32;
    uint16_t* __restrict__ u16 = pb.u16;
    const int64_t T = pb.T, Kd = pb.Kd;
    const int chunks_per_split = pb.cps, nsplit = pb.ns, ld16 = pb.ld16;
    const float scale = pb.scale;
    pdl_launch_dependents();
    pdl_wait();
    constexpr int R = L::R, NP = L::NP, WROWS = L::WROWS, WPITCH = L::WPITCH;
    extern __shared__ __align__(128) uint8_t dn_smem[];
    uint16_t* xs = reinterpret_cast<uint16_t*>(dn_smem);                 // [stage][64 rows][64], swizzled
    uint16_t* ws = reinterpret_cast<uint16_t*>(dn_smem + L::X_BYTES);    // [stage][WROWS][WPITCH]
    auto xa = [&](int st, int row, int col) { return smem_u32(xs + st * L::X_TILE + swz_off(row, col, 64, row & 7)); };
    auto wa = [&](int st, int row, int col) {
        return smem_u32(ws + st * L::W_TILE + swz_off(row, col, WPITCH, L::wswz(row)));
    };
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t row_base = (int64_t)((int)blockIdx.x - pb.first) * kDnRows;
    const int64_t nchunks = Kd / 64;
    const int64_t c_begin = (int64_t)blockIdx.y * chunks_per_split;
    const int64_t c_end = (c_begin + chunks_per_split < nchunks) ? c_begin + chunks_per_split : nchunks;
    const int64_t nc = c_end > c_begin ? c_end - c_begin : 0;

    // X loads: thread tid copies the 16-byte piece xpc of rows xr0 + 16 i
    // (i = 0..3) of every chunk; those rows share one swizzle pattern
    // (row & 7 = xr0 & 7), so the shared-memory offsets and the row pointers
    // are fixed for the whole kernel.
    const int xr0 = tid >> 3, xpc = tid & 7;
    const uint32_t xoff = (uint32_t)(xr0 * 64 + ((xpc ^ (xr0 & 7)) << 3)) * 2u;
    const uint16_t* xsrc[4];
    bool xok[4];
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t t = row_base + xr0 + 16 * i;
        xok[i] = t < T;
        xsrc[i] = X + (xok[i] ? t : 0) * Kd + xpc * 8;
    }
    auto load = [&](int stage, int64_t c) {
        const uint32_t dst = smem_u32(xs + stage * L::X_TILE) + xoff;
        #pragma unroll
        for (int i = 0; i < 4; ++i)                       // X: 64 rows x 8 pieces of 16 bytes
            cp_async16(dst + (uint32_t)(i * 16 * 64 * 2), xsrc[i] + c * 64, xok[i] ? 16u : 0u);
        if (B_KR) {                                       // W = B [Kd, r]: 64 rows x r/8 pieces
            for (int p = tid; p < 64 * NT; p += 128) {
                const int row = p / NT, piece = p % NT;
                cp_async16(wa(stage, row, piece * 8), W + (c * 64 + row) * (int64_t)R + piece * 8, 16u);
            }
        } else {                                          // W = A [r, Kd]: WROWS rows x 8 pieces
            for (int p = tid; p < WROWS * 8; p += 128) {
                const int row = p >> 3, piece = p & 7;
                const bool ok = row < R;
                cp_async16(wa(stage, row, piece * 8), W + (int64_t)(ok ? row : 0) * Kd + c * 64 + piece * 8,
                           ok ? 16u : 0u);
            }
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
    // ldmatrix lane addresses (matrix i = lanes 8i..8i+7):
    //   X (A operand): rows warp*16 + {0-7, 8-15, 0-7, 8-15}, columns {0, 0, 8, 8}
    //   A [r, Kd]:     W rows {0-7, 0-7, 8-15, 8-15} of the pair, columns {0, 8, 0, 8}
    //   B [Kd, r]:     K rows {0-7, 8-15, 0-7, 8-15}, rank columns {0, 0, 8, 8}, transposed
    const int a_row = warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
    const int a_col = 8 * (lane >> 4);
    const int w_row = B_KR ? (lane & 7) + 8 * ((lane >> 3) & 1) : (lane & 7) + 8 * (lane >> 4);
    const int w_col = B_KR ? 8 * (lane >> 4) : 8 * ((lane >> 3) & 1);
    for (int64_t i = 0; i < nc; ++i) {
        cp_async_wait<kDnStages - 2>();
        __syncthreads();                                  // chunk i landed; chunk i-1's stage is free
        const int64_t nxt = i + kDnStages - 1;            // refill it before computing on chunk i
        if (nxt < nc) load((int)(nxt % kDnStages), c_begin + nxt);
        cp_async_commit();
        const int st = (int)(i % kDnStages);
        #pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(xa(st, a_row, ks * 16 + a_col), a0, a1, a2, a3);
            #pragma unroll
            for (int p = 0; p < NP; ++p) {
                uint32_t b00, b01, b10, b11;
                if (B_KR) ldsm_x4_t(wa(st, ks * 16 + w_row, p * 16 + w_col), b00, b01, b10, b11);
                else      ldsm_x4(wa(st, p * 16 + w_row, ks * 16 + w_col), b00, b01, b10, b11);
                mma_bf16_16816(acc[2 * p], a0, a1, a2, a3, b00, b01);
                mma_bf16_16816(acc[2 * p + 1], a0, a1, a2, a3, b10, b11);
            }
        }
    }
    cp_async_wait<0>();

    // acc[n] = { (row g, col 8n+2q), (row g, col 8n+2q+1), (row g+8, ...), (row g+8, ...) }
    const int g = lane >> 2, q = lane & 3;
    const int64_t row0 = row_base + warp * 16 + g, row1 = row0 + 8;
    const bool ok0 = row0 < T, ok1 = row1 < T;
    auto emit = [&](int64_t row, int j, float v) {
        if (u32) u32[row * R + j] = v;
        if (u16) u16[row * ld16 + j] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(scale, v)));
    };
    if (nsplit == 1) {                  // every CTA of the cluster takes this branch
        if (blockIdx.y != 0) return;
        #pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int j = n * 8 + 2 * q;
            if (ok0) { emit(row0, j, acc[n][0]); emit(row0, j + 1, acc[n][1]); }
            if (ok1) { emit(row1, j, acc[n][2]); emit(row1, j + 1, acc[n][3]); }
        }
        return;
    }
    // Partial tile [64 rows][R] in shared memory (the staging ring is dead).
    __syncthreads();
    float* red = reinterpret_cast<float*>(dn_smem);
    #pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int j = n * 8 + 2 * q, rl = warp * 16 + g;
        red[rl * R + j] = acc[n][0];
        red[rl * R + j + 1] = acc[n][1];
        red[(rl + 8) * R + j] = acc[n][2];
        red[(rl + 8) * R + j + 1] = acc[n][3];
    }
    cluster_sync_all();
    const int rank = (int)cluster_ctarank();
    constexpr int V = kDnRows * R;
    const int per = (V + nsplit - 1) / nsplit;
    for (int v = rank * per + tid; v < (rank + 1) * per && v < V; v += 128) {
        const int64_t row = row_base + v / R;
        float sum = 0.0f;
        for (int sp = 0; sp < nsplit; ++sp) sum += ld_dsmem_f32(red + v, (uint32_t)sp);
        if (row < T) emit(row, v % R, sum);
    }
    cluster_sync_all();                 // partials stay readable until every CTA is done
}

// -------------------------------------------------------- token reduce ---
//
// R[j, k] = sum_{t in split} G[t, j] * X[t, k] (dA with G = g, X = x; dB with
// G = u, X = dY).  On the warp-level tensor-core instruction with M = k, N = j
// and the tokens as the contraction: X tiles [32 t x 256 k] are staged by
// cp.async (3 stages, 16-byte chunks XOR-swizzled by token row) and read
// transposed with ldmatrix.trans; G is fp32, so
// each element enters as two bf16 MMAs, hi = bf16(G) and lo = bf16(G - hi),
// which leaves a relative error below 2^-17 per product before fp32
// accumulation.  A CTA owns 256 columns k (warp w: k0+64w .. +63, so each
// warp's conversion of G feeds four 16-column MMA rows) and one token split;
// the splits of a column tile form one thread-block cluster and are added in
// split order through distributed shared memory.  At r = 16 the ring takes
// 55.5 KB.  (With 128 columns per CTA and the G conversion feeding two MMA
// rows the kernel was bound by issue slots and barrier waits: the 32 launches
// of an 8B step at T = 2048 (14 reductions each) took 3.91-4.06 ms against
// 3.33-3.46 ms with 256, one B200, events on one lane.)  Batched like the down projection: blockIdx.x
// runs over the column tiles of all problems (dA and dB of several
// projections), blockIdx.y is the token split.
constexpr int kTgCols = 256;
constexpr int kTgTok = 32;          // tokens per staged tile (two MMA k-steps)
constexpr int kTgStages = 3;
static_assert(kTgCols == 32 * 8, "a tile row is 32 pieces of 16 bytes, one per lane (the X load's thread map)");

struct TgProb {
    const float* G;      // [T, r] fp32
    const uint16_t* X;   // [T, Kd]
    float* out;          // [r, Kd] when out_rk, else [Kd, r]
    int64_t T, Kd, per;  // tokens, columns, tokens per split
    int ns, first;       // splits, first blockIdx.x of the problem
    int out_rk, accumulate;
    float scale;
};
struct TgBatch {
    int n;
    TgProb p[kMaxProbs];
};

template <int NT>
struct TgSmem {
    static constexpr int GPITCH = 8 * NT + 4;
    static constexpr int X_TILE = kTgTok * kTgCols;                // bf16 per X stage
    static constexpr size_t X_BYTES = sizeof(uint16_t) * kTgStages * X_TILE;
    static constexpr size_t G_BYTES = sizeof(float) * kTgStages * kTgTok * GPITCH;
    static constexpr size_t RING = X_BYTES + G_BYTES;
    static constexpr size_t RED = sizeof(float) * 8 * NT * kTgCols;
    static constexpr size_t BYTES = RING > RED ? RING : RED;
};

template <int NT>
__global__ void __launch_bounds__(128) lora_tgrad_kernel(const __grid_constant__ TgBatch bt) {
    using L = TgSmem<NT>;
    int pi = 0;
    while (pi + 1 < bt.n && (int)blockIdx.x >= bt.p[pi + 1].first) ++pi;
    const TgProb& pb = bt.p[pi];
    const float* __restrict__ G = pb.G;
    const uint16_t* __restrict__ X = pb.X;
    float* __restrict__ out = pb.out;
    const int64_t T = pb.T, Kd = pb.Kd, per_split = pb.per;
    const int nsplit = pb.ns, accumulate = pb.accumulate;
    const bool out_rk = pb.out_rk != 0;
    const float scale = pb.scale;
    pdl_launch_dependents();
    pdl_wait();
    constexpr int R = 8 * NT, GPITCH = L::GPITCH;
    extern __shared__ __align__(128) uint8_t tg_smem[];
    uint16_t* xs = reinterpret_cast<uint16_t*>(tg_smem);                 // [stage][32 tokens][128], swizzled
    auto xa = [&](int st, int row, int col) {
        return smem_u32(xs + st * L::X_TILE + swz_off(row, col, kTgCols, row & 7));
    };
    auto gs = reinterpret_cast<float (*)[kTgTok][GPITCH]>(tg_smem + L::X_BYTES);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t k0 = (int64_t)((int)blockIdx.x - pb.first) * kTgCols;
    const int64_t tb = (int64_t)blockIdx.y * per_split;
    const int64_t te = (tb + per_split < T) ? tb + per_split : T;
    const int64_t ntiles = te > tb ? (te - tb + kTgTok - 1) / kTgTok : 0;

    // X loads: thread tid copies the 16-byte piece xpc of rows xr0 + 4 i
    // (i = 0..7) of every tile, so its column offset, its row stride and the
    // two swizzle patterns of its rows (xr0 < 4: row & 7 = xr0 + 4 (i & 1))
    // are fixed for the whole kernel.
    const int xr0 = tid >> 5, xpc = tid & 31;
    const bool k_ok = k0 + xpc * 8 < Kd;
    const uint16_t* const xcol = X + (k_ok ? k0 + xpc * 8 : 0);
    const int64_t xstride4 = 4 * Kd;
    const uint32_t xoff0 = (uint32_t)(xr0 * kTgCols + ((xpc ^ xr0) << 3)) * 2u;
    const uint32_t xoff1 = (uint32_t)(xr0 * kTgCols + ((xpc ^ (xr0 + 4)) << 3)) * 2u;
    auto load = [&](int stage, int64_t tile) {
        const int64_t t0 = tb + tile * kTgTok;
        const uint32_t dst = smem_u32(xs + stage * L::X_TILE);
        const uint16_t* src = xcol + (t0 + xr0) * Kd;
        #pragma unroll
        for (int i = 0; i < kTgTok / 4; ++i) {            // X: 32 rows x 32 pieces of 16 bytes
            const bool ok = k_ok && t0 + xr0 + 4 * i < te;
            const uint32_t off = ((i & 1) ? xoff1 : xoff0) + (uint32_t)(4 * i * kTgCols * 2);
            cp_async16(dst + off, ok ? src : X, ok ? 16u : 0u);
            src += xstride4;
        }
        for (int p = tid; p < kTgTok * (R / 4); p += 128) {   // G: 32 rows x R/4 pieces
            const int row = p / (R / 4), piece = p % (R / 4);
            const int64_t t = t0 + row;
            const bool ok = t < te;
            cp_async16(smem_u32(&gs[stage][row][piece * 4]), G + (ok ? t : 0) * R + piece * 4, ok ? 16u : 0u);
        }
    };

    float acc[4][NT][4];
    #pragma unroll
    for (int m = 0; m < 4; ++m)
        #pragma unroll
        for (int n = 0; n < NT; ++n) acc[m][n][0] = acc[m][n][1] = acc[m][n][2] = acc[m][n][3] = 0.0f;

    #pragma unroll
    for (int s = 0; s < kTgStages - 1; ++s) {
        if (s < ntiles) load(s, s);
        cp_async_commit();
    }
    // A = X^T read transposed: matrix i = lanes 8i..8i+7 covers tokens
    // {0-7, 0-7, 8-15, 8-15} and columns {0, 8, 0, 8} of a 16 x 16 block.
    const int a_t = (lane & 7) + 8 * (lane >> 4);
    const int a_k = 8 * ((lane >> 3) & 1);
    const int g = lane >> 2, q = lane & 3;
    for (int64_t i = 0; i < ntiles; ++i) {
        cp_async_wait<kTgStages - 2>();
        __syncthreads();                                  // tile i landed; tile i-1's stage is free
        const int64_t nxt = i + kTgStages - 1;            // refill it before computing on tile i
        if (nxt < ntiles) load((int)(nxt % kTgStages), nxt);
        cp_async_commit();
        const int st = (int)(i % kTgStages);
        #pragma unroll
        for (int kk = 0; kk < kTgTok / 16; ++kk) {
            uint32_t bh[NT][2], bl[NT][2];
            #pragma unroll
            for (int n = 0; n < NT; ++n) {
                #pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float v0 = gs[st][kk * 16 + 8 * h + 2 * q][8 * n + g];
                    const float v1 = gs[st][kk * 16 + 8 * h + 2 * q + 1][8 * n + g];
                    const float h0 = __bfloat162float(__float2bfloat16_rn(v0));
                    const float h1 = __bfloat162float(__float2bfloat16_rn(v1));
                    bh[n][h] = pack2(h0, h1);
                    bl[n][h] = pack2(__fsub_rn(v0, h0), __fsub_rn(v1, h1));
                }
            }
            #pragma unroll
            for (int m = 0; m < 4; ++m) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4_t(xa(st, kk * 16 + a_t, warp * 64 + m * 16 + a_k), a0, a1, a2, a3);
                #pragma unroll
                for (int n = 0; n < NT; ++n) {
                    mma_bf16_16816(acc[m][n], a0, a1, a2, a3, bh[n][0], bh[n][1]);
                    mma_bf16_16816(acc[m][n], a0, a1, a2, a3, bl[n][0], bl[n][1]);
                }
            }
        }
    }
    cp_async_wait<0>();

    // acc[m][n] = { (k = base+g, j = 8n+2q), (k, j+1), (k+8, j), (k+8, j+1) }, base = k0 + 32 warp + 16 m
    auto out_index = [&](int64_t k, int j) -> int64_t { return out_rk ? (int64_t)j * Kd + k : k * R + j; };
    auto finish = [&](int64_t k, int j, float v) {
        const int64_t o = out_index(k, j);
        const float w = __fmul_rn(scale, v);
        out[o] = accumulate ? __fadd_rn(out[o], w) : w;
    };
    if (nsplit == 1) {                  // every CTA of the cluster takes this branch
        if (blockIdx.y != 0) return;
        #pragma unroll
        for (int m = 0; m < 4; ++m)
            #pragma unroll
            for (int n = 0; n < NT; ++n) {
                const int64_t k = k0 + warp * 64 + m * 16 + g;
                const int j = 8 * n + 2 * q;
                if (k < Kd) { finish(k, j, acc[m][n][0]); finish(k, j + 1, acc[m][n][1]); }
                if (k + 8 < Kd) { finish(k + 8, j, acc[m][n][2]); finish(k + 8, j + 1, acc[m][n][3]); }
            }
        return;
    }
    // Partial tile [R][128 columns] in shared memory (the staging ring is dead).
    __syncthreads();
    float* red = reinterpret_cast<float*>(tg_smem);
    #pragma unroll
    for (int m = 0; m < 4; ++m)
        #pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int c = warp * 64 + m * 16 + g;
            const int j = 8 * n + 2 * q;
            red[j * kTgCols + c] = acc[m][n][0];
            red[(j + 1) * kTgCols + c] = acc[m][n][1];
            red[j * kTgCols + c + 8] = acc[m][n][2];
            red[(j + 1) * kTgCols + c + 8] = acc[m][n][3];
        }
    cluster_sync_all();
    const int rank = (int)cluster_ctarank();
    constexpr int V = R * kTgCols;
    const int per = (V + nsplit - 1) / nsplit;
    for (int v = rank * per + tid; v < (rank + 1) * per && v < V; v += 128) {
        const int64_t k = k0 + v % kTgCols;
        float sum = 0.0f;
        for (int sp = 0; sp < nsplit; ++sp) sum += ld_dsmem_f32(red + v, (uint32_t)sp);
        if (k < Kd) finish(k, v / kTgCols, sum);
    }
    cluster_sync_all();
}

template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    // Prefer the largest shared-memory carveout, the one a GEMM CTA runs
    // with, so these CTAs can be placed beside it.
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    return e;
}

// Launch with the splits of one output tile as one cluster along y.
template <typename Kern, typename... Args>
cudaError_t launch_split(Kern kernel, dim3 grid, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (grid.y > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = 1;
        attr[na].val.clusterDim.y = grid.y;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    na += pdl_attr(&attr[na]);
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <int NT, bool B_KR>
lsn_status launch_down_nt(dim3 grid, cudaStream_t st, const DownBatch& bt) {
    constexpr size_t bytes = DownSmem<NT, B_KR>::BYTES;
    static const cudaError_t attr = allow_smem(lora_down_kernel<NT, B_KR>, bytes);
    if (attr != cudaSuccess) return fail_cuda(attr, "cudaFuncSetAttribute(lora_down smem)");
    LSN_CUDA_TRY(launch_split(lora_down_kernel<NT, B_KR>, grid, bytes, st, bt));
    return LSN_OK;
}

template <int NT>
lsn_status launch_tgrad_nt(dim3 grid, cudaStream_t st, const TgBatch& bt) {
    constexpr size_t bytes = TgSmem<NT>::BYTES;
    static const cudaError_t attr = allow_smem(lora_tgrad_kernel<NT>, bytes);
    if (attr != cudaSuccess) return fail_cuda(attr, "cudaFuncSetAttribute(lora_tgrad smem)");
    LSN_CUDA_TRY(launch_split(lora_tgrad_kernel<NT>, grid, bytes, st, bt));
    return LSN_OK;
}

template <bool B_KR>
lsn_status dispatch_down(int r, dim3 grid, cudaStream_t st, const DownBatch& bt) {
    switch (r / 8) {
        case 1: return launch_down_nt<1, B_KR>(grid, st, bt);
        case 2: return launch_down_nt<2, B_KR>(grid, st, bt);
        case 3: return launch_down_nt<3, B_KR>(grid, st, bt);
        case 4: return launch_down_nt<4, B_KR>(grid, st, bt);
        case 5: return launch_down_nt<5, B_KR>(grid, st, bt);
        case 6: return launch_down_nt<6, B_KR>(grid, st, bt);
        case 7: return launch_down_nt<7, B_KR>(grid, st, bt);
        case 8: return launch_down_nt<8, B_KR>(grid, st, bt);
        default: return fail(LSN_ERR_INVALID_ARG, "rank must be a multiple of 8 in [8, 64]");
    }
}

lsn_status dispatch_tgrad(int r, dim3 grid, cudaStream_t st, const TgBatch& bt) {
    switch (r / 8) {
        case 1: return launch_tgrad_nt<1>(grid, st, bt);
        case 2: return launch_tgrad_nt<2>(grid, st, bt);
        case 3: return launch_tgrad_nt<3>(grid, st, bt);
        case 4: return launch_tgrad_nt<4>(grid, st, bt);
        case 5: return launch_tgrad_nt<5>(grid, st, bt);
        case 6: return launch_tgrad_nt<6>(grid, st, bt);
        case 7: return launch_tgrad_nt<7>(grid, st, bt);
        case 8: return launch_tgrad_nt<8>(grid, st, bt);
        default: return fail(LSN_ERR_INVALID_ARG, "rank must be a multiple of 8 in [8, 64]");
    }
}

}  // namespace

// ----------------------------------------------------------- planning ---
// Split counts depend on the shape only (never on the device or pointers), so
// a given shape always sums in the same order.

// K-splits of the down projection: up to 8 (one cluster), aiming at about
// four 128-thread CTAs per SM of a 148-SM part, at least four 64-wide chunks
// per split.
int down_splits(int64_t T, int64_t Kd) {
    const int64_t row_blocks = (T + kDnRows - 1) / kDnRows;
    if (row_blocks <= 0 || Kd < 64) return 1;
    const int64_t chunks = Kd / 64;
    int64_t s = (592 + row_blocks - 1) / row_blocks;
    const int64_t cap = chunks / 4 > 0 ? chunks / 4 : 1;
    if (s > cap) s = cap;
    if (s > 8) s = 8;
    if (s < 1) s = 1;
    return (int)s;
}


// Token splits of a reduction: up to 8 (one cluster), aiming at about four
// 128-thread CTAs per SM, at least 64 tokens per split.
int tgrad_splits(int64_t T, int64_t Kd) {
    const int64_t tiles = (Kd + kTgCols - 1) / kTgCols;
    if (tiles <= 0 || T <= 0) return 1;
    int64_t s = (592 + tiles - 1) / tiles;
    const int64_t by_t = (T + 63) / 64;
    if (s > by_t) s = by_t;
    if (s > 8) s = 8;
    if (s < 1) s = 1;
    return (int)s;
}


// Down projections of a batch of problems, all with W in the same layout
// (w_rk: A [r, Kd]; otherwise B [Kd, r]) and the same rank.  Problems with
// T == 0 are skipped; more than kMaxProbs problems take several launches.
lsn_status launch_lora_down_batch(int n, const DownSpec* specs, bool w_rk, int r, cudaStream_t st) {
    DownBatch bt{};
    int blocks = 0, smax = 1;
    auto flush = [&]() -> lsn_status {
        if (bt.n == 0) return LSN_OK;
        dim3 grid((unsigned)blocks, (unsigned)smax);
        const lsn_status s = w_rk ? dispatch_down<false>(r, grid, st, bt) : dispatch_down<true>(r, grid, st, bt);
        bt = DownBatch{};
        blocks = 0;
        smax = 1;
        return s;
    };
    for (int i = 0; i < n; ++i) {
        const DownSpec& d = specs[i];
        if (d.T == 0) continue;
        if (bt.n == kMaxProbs) {
            const lsn_status s = flush();
            if (s != LSN_OK) return s;
        }
        DownProb& pb = bt.p[bt.n++];
        pb.X = d.X;
        pb.W = d.W;
        pb.u32 = d.u32;
        pb.u16 = d.u16;
        pb.T = d.T;
        pb.Kd = d.Kd;
        pb.ns = down_splits(d.T, d.Kd);
        pb.cps = (int)((d.Kd / 64 + pb.ns - 1) / pb.ns);
        pb.first = blocks;
        pb.ld16 = d.ld16 > 0 ? d.ld16 : r;
        pb.scale = d.scale;
        blocks += (int)((d.T + kDnRows - 1) / kDnRows);
        smax = pb.ns > smax ? pb.ns : smax;
    }
    return flush();
}

// Token reductions of a batch of problems of the same rank.
lsn_status launch_lora_tgrad_batch(int n, const TgSpec* specs, int r, cudaStream_t st) {
    TgBatch bt{};
    int blocks = 0, smax = 1;
    auto flush = [&]() -> lsn_status {
        if (bt.n == 0) return LSN_OK;
        const lsn_status s = dispatch_tgrad(r, dim3((unsigned)blocks, (unsigned)smax), st, bt);
        bt = TgBatch{};
        blocks = 0;
        smax = 1;
        return s;
    };
    for (int i = 0; i < n; ++i) {
        const TgSpec& d = specs[i];
        if (d.Kd == 0) continue;
        if (bt.n == kMaxProbs) {
            const lsn_status s = flush();
            if (s != LSN_OK) return s;
        }
        TgProb& pb = bt.p[bt.n++];
        pb.G = d.G;
        pb.X = d.X;
        pb.out = d.out;
        pb.T = d.T;
        pb.Kd = d.Kd;
        pb.ns = tgrad_splits(d.T, d.Kd);
        pb.per = ((d.T + pb.ns - 1) / pb.ns + kTgTok - 1) / kTgTok * kTgTok;
        pb.first = blocks;
        pb.out_rk = d.out_rk ? 1 : 0;
        pb.accumulate = d.accumulate;
        pb.scale = d.scale;
        blocks += (int)((d.Kd + kTgCols - 1) / kTgCols);
        smax = pb.ns > smax ? pb.ns : smax;
    }
    return flush();
}

// X [T, Kd] times W: w_rk ? W is A [r, Kd] : W is B [Kd, r].
lsn_status launch_lora_down(const uint16_t* X, const uint16_t* W, bool w_rk, int64_t T, int64_t Kd, int r,
                            float scale, float* u32, uint16_t* u16, cudaStream_t st) {
    const DownSpec d{X, W, u32, u16, T, Kd, scale};
    return launch_lora_down_batch(1, &d, w_rk, r, st);
}

lsn_status launch_lora_tgrad(const float* G, const uint16_t* X, bool out_rk, int64_t T, int64_t Kd, int r,
                             float scale, int accumulate, float* out, cudaStream_t st) {
    const TgSpec d{G, X, out, T, Kd, out_rk, accumulate, scale};
    return launch_lora_tgrad_batch(1, &d, r, st);
}

}  // namespace lsn
