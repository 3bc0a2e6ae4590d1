// Tensor-core GEMM of the LoRA linear on sm_100a (tcgen05 + TMEM + TMA):
//
//   D[M, N] (bf16) = Aop[M, Kc] . Bop[Kc, N]  +  LA[M, r] . LB[r, N]
//
// with fp32 accumulation in tensor memory.  The forward pass uses it as
// y = x . W^T + (s u) . B^T  (Bop = W^T: W [N,K] is K-major), the backward
// pass as dX = dY . W + (s g) . A  (Bop = W: MN-major, the W tile is read
// transposed by the MMA straight from the same row-major weight).  The LoRA
// term is one extra K-block of ceil(r/16) MMAs into the same accumulator, so
// y and dX leave the tensor cores once ("Can You Fine-Tune a 27B Model on a
// Laptop? (I Did the Math)", 1:47-1:58: the adapter rides alongside the
// frozen weights).
//
// Grouped projections (several linears reading the same x, e.g. q, k, v):
// the forward is one GEMM over their stacked weights whose output columns are
// routed to each projection's y (up to kMaxSeg segments); the backward is one
// GEMM whose contraction runs over the projections' dY side by side (one A
// tensor map per projection, chosen per 128-wide K-block), giving the summed
// input gradient.
//
// Structure (one persistent CTA per SM, or one CTA pair per two SMs, 192
// threads):
//   warp 0     TMA producer: one elected lane streams 128-wide contraction
//              stages (two 64-wide 128-byte-swizzled sub-tiles per operand)
//              into a 3-stage ring; with CTA pairs each CTA loads its own
//              128 rows of A and half of B, completing on the leader's
//              barrier;
//   warp 1     allocates 2*BN TMEM columns; one lane of the leader issues
//              tcgen05.mma (M = 128, or 256 across a pair with
//              cta_group::2; N = BN; K = 16) and commits each stage back to
//              the producers and each finished accumulator to the epilogue;
//   warps 2-5  epilogue: tcgen05.ld 32 columns at a time from their TMEM lane
//              quadrant, round to bf16, store; the two accumulator buffers
//              let the epilogue of tile i overlap the main loop of tile i+1.
// Every wait is bounded; a wait that runs out sets *err and the CTA winds
// down (after letting its issued copies and MMAs finish) instead of hanging.
#include <algorithm>
#include <atomic>
#include <cstring>
#include <map>
#include <mutex>
#include <type_traits>
#include <vector>

#include "common.cuh"
#include "launch.cuh"

namespace lsn {

constexpr int kMaxSeg = kGemmMaxSeg;   // output segments / A tensor maps of a grouped GEMM

struct GemmArgs {
    int M, N;            // output rows (tokens) and columns
    int num_kb;          // 128-wide contraction blocks of the base term
    int lora_k16;        // K=16 MMAs of the LoRA term (0: none)
    uint16_t* D;         // bf16 output, row-major
    int64_t ldd;         // elements
    int* err;            // device error flag (set on a timed-out wait)
    // Output segments: columns [seg_col[i], seg_col[i+1]) go to seg_D[i] with
    // row stride seg_ld[i] (column 0 of the segment at seg_D[i]); nseg == 0
    // means the single output D.
    int nseg;
    int seg_col[kMaxSeg + 1];
    uint16_t* seg_D[kMaxSeg];
    int64_t seg_ld[kMaxSeg];
    // A operand split along the contraction: K-blocks [a_kb[i], a_kb[i+1])
    // come from A tensor map i at contraction coordinate (kb - a_kb[i]) * 128;
    // na == 1 means the single map.
    int na;
    int a_kb[kMaxSeg + 1];
    // NF4 base converted in the kernel (fused variant only):
    const uint8_t* absmax_q;   // [wrows * wcols / 64] second-level codes
    const float* absmax_s2;    // [ceil(nblk / 256)]
    const float* absmax_off;   // [1]
    int wrows, wcols;          // W is [wrows, wcols] row-major (N_out x K_in)
    float level[16];           // NF4 levels
    float dq[256];             // second-level table
    const uint16_t* lora_b;    // LoRA operand of the last K-block (fwd: B [N, r]; bwd: A [r, N])
    int lora_r;
    // Stream-K schedule (sk != 0).  The num_tiles x num_kb contraction blocks
    // of the base term, tile after tile, are cut into consecutive ranges of
    // sk_per blocks, one per worker (CTA pair or CTA), so every worker does
    // the same work (a tile's LoRA block goes with its last piece).  A
    // tile cut by a range boundary is computed in two pieces (by the workers
    // on either side of the boundary); each writes its fp32 partial tile to
    // sk_part and counts itself in sk_cnt (one counter per boundary and CTA
    // of a pair); the one that counts second adds the two partials and
    // stores the tile.  fp32 addition is commutative, so the result does not
    // depend on which piece finishes first.  Counters are zero between
    // launches (the second piece resets its counter).
    int sk;
    int64_t sk_per;
    float* sk_part;
    int* sk_cnt;
    // Tail split (tq > 0; whole-tile schedule of the pair kernel only): the
    // tiles of the last, partial round, [num_tiles - num_tiles % workers,
    // num_tiles), are cut along N into quanta of tq columns, and every worker
    // takes a contiguous run of about the same number of quanta (cut at tile
    // ends into narrower tiles of whole quanta).  Each output element is still
    // the same chain of MMAs over the whole contraction, so the bits are those
    // of whole tiles.
    int tq;
};

// Several independent GEMMs of one shape family (same M and contraction
// layout, e.g. the projections of a decoder layer) in one persistent launch:
// problem i has its own A, B, LA and LB tensor maps, N, contraction blocks,
// LoRA MMAs and output.  The launch's tiles are numbered problem after
// problem (tile0[i] .. tile0[i+1]-1 belong to problem i, M-fastest inside a
// problem), and worker (CTA pair) u takes tile[start[u] .. start[u+1]) in
// that order: a schedule made on the host that balances the workers' summed
// tile costs (tiles of different problems can differ in contraction length).
// Every tile is whole and computed by one worker, so each output element is
// the same chain of MMAs as in a launch of its problem alone.
constexpr int kMultiMaxProb = 8;
constexpr int kMultiMaxUnits = 80;
constexpr int kMultiMaxTiles = 5120;
struct MultiProbs {
    // Problem i's A operand may be split along the contraction like a grouped
    // GEMM's: K-blocks [a_kb[i][j], a_kb[i][j+1]) from map a[i * kMaxSeg + j].
    CUtensorMap a[kMultiMaxProb * kMaxSeg], b[kMultiMaxProb], la[kMultiMaxProb], lb[kMultiMaxProb];
    int na[kMultiMaxProb];
    int a_kb[kMultiMaxProb][kMaxSeg + 1];
    int nprob;
    int tile0[kMultiMaxProb + 1];
    int N[kMultiMaxProb];
    int num_kb[kMultiMaxProb];
    int lora_k16[kMultiMaxProb];
    uint16_t* D[kMultiMaxProb];
    int64_t ldd[kMultiMaxProb];
    uint16_t start[kMultiMaxUnits + 1];
    uint16_t tile[kMultiMaxTiles];
};
struct NoMulti {
    int unused;
};

namespace {

// Tile geometry.  A stage holds a 128-wide slice of the contraction as two
// 64-wide sub-tiles per operand (each one 128-byte-swizzle atom wide), so one
// full/empty barrier round trip feeds eight K=16 MMAs: with four, the
// handshake between producer and MMA issuer kept the tensor pipe measurably
// idle.
constexpr int BM = 128;          // rows of A per CTA
constexpr int BK = 128;          // contraction per stage
constexpr int SUB = 64;          // contraction per sub-tile (one swizzle atom)
constexpr int STAGES = 3;
constexpr int CONV_WARPS = 8;    // NF4 converter warps (fused variant)

// PAIR = false: one CTA per SM, tile 128 x BN.
// PAIR = true : a CTA pair (cluster of 2) issues the 2-SM MMA, tile 256 x BN,
//               each CTA staging its 128 rows of A and BN/2 rows of B.
template <bool PAIR, int BN, bool B_MN>
struct Cfg {
    static constexpr int B_ROWS = PAIR ? BN / 2 : BN;     // B rows (N extent) staged per CTA
    static constexpr int A_SUB = BM * SUB * 2;             // bytes of one A sub-tile
    static constexpr int A_BYTES = 2 * A_SUB;
    static constexpr int B_SUB = B_ROWS * SUB * 2;         // K-major: bytes of one B sub-tile
    static constexpr int B_BYTES = 2 * B_SUB;              // MN-major: B_ROWS/64 atom columns of 128 x 64
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
    static constexpr uint32_t IDESC = idesc_bf16(PAIR ? 2 * BM : BM, BN, 0, B_MN ? 1 : 0);
    static constexpr uint32_t TMEM_COLS = 2 * BN;
    static constexpr int TILE_M = PAIR ? 2 * BM : BM;
    static constexpr uint32_t ACC_EMPTY_ARRIVALS = (PAIR ? 2 : 1) * 4;
    static constexpr int THREADS = 192;
};

__device__ __forceinline__ void raise_error(volatile int* abort_flag, int* err, int code) {
    *abort_flag = 1;
    if (err) atomicExch(err, code);
}

// The work of one worker: (tile, columns, first contraction block, end block)
// items: whole tiles round robin (tile = unit, unit + nunits, ...), then, with
// the tail split, the worker's run of quanta of the last round's tiles; or the
// worker's stream-K range.  Stream-K ranges count the base term's blocks
// only; the LoRA block (the last of a tile's nkb) always goes with the piece
// that ends the tile, so a tile is cut at the same place with the adapter on
// or off (its block adds exact zeros when B = 0).
struct Items {
    bool sk;
    int nkb, nbase, num_tiles, nunits, tile;
    int64_t cur, hi;
    int full_end, tq, qpt, qcur, qhi, num_m, n, bn;
    const MultiProbs* mp;      // several problems: the worker's tile list (else nullptr)
    int prob;                  // problem of the last item (0 with one problem)
    __device__ Items(const GemmArgs& p, int unit, int nunits_, int num_tiles_, int nkb_, int num_m_, int bn_,
                     const MultiProbs* mp_ = nullptr)
        : sk(p.sk != 0), nkb(nkb_), nbase(p.num_kb), num_tiles(num_tiles_), nunits(nunits_), tile(unit),
          tq(p.tq), num_m(num_m_), n(p.N), bn(bn_), mp(mp_), prob(0) {
        if (mp) {                              // tile list positions [cur, hi)
            cur = mp->start[unit];
            hi = mp->start[unit + 1];
            full_end = 0;
            qpt = qcur = qhi = 0;
            return;
        }
        const int64_t total = (int64_t)num_tiles_ * p.num_kb;
        cur = (int64_t)unit * p.sk_per;
        hi = cur + p.sk_per < total ? cur + p.sk_per : total;
        full_end = num_tiles_;
        qpt = qcur = qhi = 0;
        if (tq > 0) {
            full_end = num_tiles_ - num_tiles_ % nunits_;
            qpt = bn_ / tq;
            const int rq = (num_tiles_ - full_end) * qpt;
            qcur = (int)((int64_t)unit * rq / nunits_);
            qhi = (int)((int64_t)(unit + 1) * rq / nunits_);
        }
    }
    // t: tile index; c0, nw: the item's first column inside the tile and its
    // width (a multiple of 32; columns at or beyond N are never stored).
    __device__ bool next(int& t, int& c0, int& nw, int& kb0, int& kb1) {
        if (mp) {
            if (cur >= hi) return false;
            const int g = mp->tile[cur++];
            int pi = 0;
            while (pi + 1 < mp->nprob && g >= mp->tile0[pi + 1]) ++pi;
            prob = pi;
            t = g - mp->tile0[pi];
            c0 = 0;
            nw = bn;
            kb0 = 0;
            kb1 = mp->num_kb[pi] + (mp->lora_k16[pi] > 0 ? 1 : 0);
            return true;
        }
        if (!sk) {
            kb0 = 0;
            kb1 = nkb;
            if (tile < full_end) {
                t = tile;
                c0 = 0;
                nw = bn;
                tile += nunits;
                return true;
            }
            while (qcur < qhi) {
                const int ti = qcur / qpt, qi = qcur - ti * qpt;
                const int w = qpt - qi < qhi - qcur ? qpt - qi : qhi - qcur;
                qcur += w;
                t = full_end + ti;
                c0 = qi * tq;
                nw = w * tq;
                if ((t / num_m) * bn + c0 < n) return true;    // else: quanta past N, nothing to do
            }
            return false;
        }
        if (cur >= hi) return false;
        t = (int)(cur / nbase);
        kb0 = (int)(cur - (int64_t)t * nbase);
        const int64_t left = hi - cur;
        kb1 = (int64_t)(nbase - kb0) <= left ? nbase : kb0 + (int)left;
        cur += kb1 - kb0;
        if (kb1 == nbase) kb1 = nkb;           // the tile's end: its LoRA block too
        c0 = 0;
        nw = bn;
        return true;
    }
};

// Named barrier 1 over the four epilogue warps (128 threads): a plain
// barrier, and barriers that also reduce a predicate over the 128 threads.
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ bool epi_all(bool v) {
    uint32_t r;
    asm volatile("{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 1, 128, p;\n selp.u32 %0, 1, 0, q;\n}"
                 : "=r"(r) : "r"((uint32_t)v) : "memory");
    return r != 0;
}
__device__ __forceinline__ bool epi_any(bool v) {
    uint32_t r;
    asm volatile("{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, 128, p;\n selp.u32 %0, 1, 0, q;\n}"
                 : "=r"(r) : "r"((uint32_t)v) : "memory");
    return r != 0;
}

// Round 32 fp32 values to bf16 and store them as 4 x 16 bytes.
__device__ __forceinline__ void store_bf16x32(uint16_t* dst16, const float (&f)[32]) {
    uint4* dst = reinterpret_cast<uint4*>(dst16);
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint4 o;
        o.x = pack_bf16x2(f[8 * i + 0], f[8 * i + 1]);
        o.y = pack_bf16x2(f[8 * i + 2], f[8 * i + 3]);
        o.z = pack_bf16x2(f[8 * i + 4], f[8 * i + 5]);
        o.w = pack_bf16x2(f[8 * i + 6], f[8 * i + 7]);
        dst[i] = o;
    }
}


// The bf16 output address of 32 columns starting at `col` of row `row`
// (routed to its segment's output for a grouped GEMM).
__device__ __forceinline__ uint16_t* out_ptr(const GemmArgs& p, int row, int col) {
    uint16_t* base = p.D;
    int64_t ld = p.ldd;
    int lc = col;
    if (p.nseg > 0) {                          // the segment of these 32 columns (widths: multiples of 64)
        int sgi = 0;
        while (sgi + 1 < p.nseg && col >= p.seg_col[sgi + 1]) ++sgi;
        base = p.seg_D[sgi];
        ld = p.seg_ld[sgi];
        lc = col - p.seg_col[sgi];
    }
    return base + (int64_t)row * ld + lc;
}

// The epilogue of one of the two pieces of a stream-K tile (see GemmArgs):
// write this CTA's fp32 partial, free the accumulator, count the piece and,
// if it is the second, add both partials and store the tile.  Kept out of
// line so that the common path of the epilogue keeps its few registers.
template <bool PAIR, int BN>
__device__ __noinline__ void split_piece(const GemmArgs& p, uint32_t tm, uint64_t* acc_empty, int piece, int unit,
                                         uint32_t rank, int q, int lane, int row, int col0) {
    const int bnd = piece == 0 ? unit + 1 : unit;
    const int64_t tile_floats = (int64_t)BM * BN;
    constexpr int CTAS = PAIR ? 2 : 1;
    float* mine = p.sk_part + (((int64_t)bnd * 2 + piece) * CTAS + rank) * tile_floats;
    const int rl = q * 32 + lane;
    #pragma unroll 1
    for (int c = 0; c < BN / 16; ++c) {
        uint32_t v[16];
        tmem_ld16(tm + (uint32_t)(c * 16), v);
        tmem_ld_wait(v);
        float4* d = reinterpret_cast<float4*>(mine + ((int64_t)(c >> 1) * BM + rl) * 32 + (c & 1) * 16);
        #pragma unroll
        for (int i = 0; i < 4; ++i)
            d[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]), __uint_as_float(v[4 * i + 2]),
                               __uint_as_float(v[4 * i + 3]));
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {                    // the accumulator is free again
        if constexpr (PAIR) mbar_arrive_cluster(mapa_shared(smem_u32(acc_empty), 0));
        else                mbar_arrive(acc_empty);
    }
    __threadfence();                    // this thread's partial, visible device-wide ...
    epi_sync();                         // ... for all 128 threads, before the count
    int* cnt = p.sk_cnt + bnd * CTAS + rank;
    int old = 0;
    if (q == 0 && lane == 0) old = atomicAdd(cnt, 1);
    if (!epi_any(old == 1)) return;     // the first piece: the second one stores the tile
    __threadfence();
    const float* other = p.sk_part + (((int64_t)bnd * 2 + (1 - piece)) * CTAS + rank) * tile_floats;
    #pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
        const int col = col0 + c * 32;
        if (col >= p.N) break;
        if (row < p.M) {
            const float4* a = reinterpret_cast<const float4*>(mine + ((int64_t)c * BM + rl) * 32);
            const float4* b = reinterpret_cast<const float4*>(other + ((int64_t)c * BM + rl) * 32);
            uint4* dst = reinterpret_cast<uint4*>(out_ptr(p, row, col));
            #pragma unroll 1
            for (int i = 0; i < 4; ++i) {           // 8 columns at a time
                const float4 x0 = __ldcg(a + 2 * i), x1 = __ldcg(a + 2 * i + 1);
                const float4 y0 = __ldcg(b + 2 * i), y1 = __ldcg(b + 2 * i + 1);
                uint4 o;
                o.x = pack_bf16x2(x0.x + y0.x, x0.y + y0.y);
                o.y = pack_bf16x2(x0.z + y0.z, x0.w + y0.w);
                o.z = pack_bf16x2(x1.x + y1.x, x1.y + y1.y);
                o.w = pack_bf16x2(x1.z + y1.z, x1.w + y1.w);
                dst[i] = o;
            }
        }
    }
    if (q == 0 && lane == 0) *cnt = 0;      // ready for the next launch on this workspace
}

// The A tensor maps of a grouped GEMM (the caller's separate dY tensors).
struct AMaps {
    CUtensorMap m[kMaxSeg];
};

template <bool MULTI>
using MultiParam = std::conditional_t<MULTI, MultiProbs, NoMulti>;

template <bool PAIR, int BN, bool B_MN, bool MULTI>
__global__ void __launch_bounds__(Cfg<PAIR, BN, B_MN>::THREADS, 1)
    lsn_gemm_kernel(const __grid_constant__ AMaps tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmLA, const __grid_constant__ CUtensorMap tmLB,
                    const __grid_constant__ GemmArgs p, const __grid_constant__ MultiParam<MULTI> mpar) {
    using C = Cfg<PAIR, BN, B_MN>;
    const MultiProbs* mp = nullptr;
    if constexpr (MULTI) mp = &mpar;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
    uint64_t* full = bars;                    // TMA landed (A and B of the stage, both CTAs of a pair)
    uint64_t* empty = bars + STAGES;          // MMAs done reading the stage
    uint64_t* acc_full = bars + 2 * STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t rank = 0;
    if constexpr (PAIR) rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int nunits = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    const int num_m = (p.M + C::TILE_M - 1) / C::TILE_M;
    const int num_n = (p.N + BN - 1) / BN;
    const int num_tiles = num_m * num_n;
    const int nkb = p.num_kb + (p.lora_k16 > 0 ? 1 : 0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], C::ACC_EMPTY_ARRIVALS); }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        if constexpr (MULTI) {
            for (int i = 0; i < mp->nprob; ++i) {
                for (int j = 0; j < mp->na[i]; ++j) tma_prefetch_desc(&mp->a[i * kMaxSeg + j]);
                tma_prefetch_desc(&mp->b[i]);
                if (mp->lora_k16[i] > 0) { tma_prefetch_desc(&mp->la[i]); tma_prefetch_desc(&mp->lb[i]); }
            }
        } else {
            for (int i = 0; i < p.na; ++i) tma_prefetch_desc(&tmA.m[i]);
            tma_prefetch_desc(&tmB);
            if (p.lora_k16 > 0) { tma_prefetch_desc(&tmLA); tma_prefetch_desc(&tmLB); }
        }
    }
    if (warp == 1) {
        if constexpr (PAIR) { tmem_alloc_pair(tmem_holder, C::TMEM_COLS); tmem_relinquish_pair(); }
        else                { tmem_alloc(tmem_holder, C::TMEM_COLS); tmem_relinquish(); }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync_all();   // both CTAs' barriers initialised before any remote use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_launch_dependents();
    pdl_wait();

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------- producer --
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            Items items(p, unit, nunits, num_tiles, nkb, num_m, BN, mp);
            int tile, c0, nw, kb0, kb1;
            while (ok && items.next(tile, c0, nw, kb0, kb1)) {
                const int pi = items.prob;
                const int nbase = MULTI ? mp->num_kb[pi] : p.num_kb;
                const int mb = tile % num_m, nb = tile / num_m;
                const int m_row = mb * C::TILE_M + (int)rank * BM;
                // This CTA's share of the item's B rows (a pair splits N in halves);
                // the stage is always filled with B_ROWS rows, the MMA reads the share.
                const int n_off = nb * BN + c0 + (int)rank * (PAIR ? nw / 2 : 0);
                int ai = 0;                                   // A map of the current K-block
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    uint8_t* sA = smem + stage * C::STAGE_BYTES;
                    uint8_t* sB = sA + C::A_BYTES;
                    const bool lora = kb >= nbase;
                    const CUtensorMap* ma;
                    const CUtensorMap* mbp;
                    int ka;
                    const int kc = lora ? 0 : kb * BK;                       // contraction coordinate of B
                    if constexpr (MULTI) {
                        while (!lora && ai + 1 < mp->na[pi] && kb >= mp->a_kb[pi][ai + 1]) ++ai;
                        ma = lora ? &mp->la[pi] : &mp->a[pi * kMaxSeg + ai];
                        mbp = lora ? &mp->lb[pi] : &mp->b[pi];
                        ka = lora ? 0 : (kb - mp->a_kb[pi][ai]) * BK;
                    } else {
                        while (!lora && ai + 1 < p.na && kb >= p.a_kb[ai + 1]) ++ai;
                        ma = lora ? &tmLA : &tmA.m[ai];
                        mbp = lora ? &tmLB : &tmB;
                        ka = lora ? 0 : (kb - p.a_kb[ai]) * BK;              // ... and of the A map
                    }
                    uint32_t fbar = smem_u32(&full[stage]);
                    if constexpr (PAIR) fbar = mapa_shared(fbar, 0);
                    if (leader) mbar_arrive_expect_tx(&full[stage], (PAIR ? 2 : 1) * (C::A_BYTES + C::B_BYTES));
                    auto load = [&](void* dst, const CUtensorMap* m, int x, int y) {
                        if constexpr (PAIR) tma_load_2d_pair(dst, m, x, y, fbar);
                        else                tma_load_2d(dst, m, x, y, &full[stage]);
                    };
                    load(sA, ma, ka, m_row);
                    load(sA + C::A_SUB, ma, ka + SUB, m_row);
                    if (!B_MN) {
                        load(sB, mbp, kc, n_off);
                        load(sB + C::B_SUB, mbp, kc + SUB, n_off);
                    } else {
                        #pragma unroll
                        for (int a = 0; a < C::B_ROWS / 64; ++a) load(sB + a * (BK * 128), mbp, n_off + a * 64, kc);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) raise_error(abort_flag, p.err, 1);
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // -------------------------------------------------- MMA issuer --
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            Items items(p, unit, nunits, num_tiles, nkb, num_m, BN, mp);
            int tile, c0, nw, kb0, kb1;
            while (ok && items.next(tile, c0, nw, kb0, kb1)) {
                const int nbase = MULTI ? mp->num_kb[items.prob] : p.num_kb;
                const int lk16 = MULTI ? mp->lora_k16[items.prob] : p.lora_k16;
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                const uint32_t idesc = nw == BN ? C::IDESC : idesc_bf16(C::TILE_M, nw, 0, B_MN ? 1 : 0);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(smem + stage * C::STAGE_BYTES);
                    const uint32_t b0 = a0 + C::A_BYTES;
                    const int nk = (kb < nbase) ? BK / 16 : lk16;
                    for (int k = 0; k < nk; ++k) {
                        const int j = k >> 2, kk = k & 3;       // sub-tile, step inside it
                        const uint64_t ad = smem_desc_sw128(a0 + j * C::A_SUB + kk * 32, 16, 1024);
                        const uint64_t bd = B_MN ? smem_desc_sw128(b0 + k * 2048, BK * 128, 1024)
                                                 : smem_desc_sw128(b0 + j * C::B_SUB + kk * 32, 16, 1024);
                        const uint32_t accum = (kb > kb0 || k > 0) ? 1u : 0u;
                        if constexpr (PAIR) umma_bf16_pair(d_tmem, ad, bd, idesc, accum);
                        else                umma_bf16(d_tmem, ad, bd, idesc, accum);
                    }
                    if constexpr (PAIR) umma_commit_pair(&empty[stage]);
                    else                umma_commit(&empty[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                if constexpr (PAIR) umma_commit_pair(&acc_full[acc]);
                else                umma_commit(&acc_full[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
            if (!ok) raise_error(abort_flag, p.err, 2);
            // Every MMA issued here completes before TMEM is freed.
            if constexpr (PAIR) umma_commit_pair(drain);
            else                umma_commit(drain);
            mbar_wait(drain, 0, nullptr);
        }
    } else {
        // -------------------------------------------------------- epilogue --
        const int q = warp & 3;                    // TMEM lanes 32q .. 32q+31
        const int rloc = (int)rank * BM + q * 32 + lane;   // row of the tile this thread drains
        int acc = 0;
        uint32_t acc_phase = 0;
        Items items(p, unit, nunits, num_tiles, nkb, num_m, BN, mp);
        int tile, c0, nw, kb0, kb1;
        while (items.next(tile, c0, nw, kb0, kb1)) {
            const int mb = tile % num_m, nb = tile / num_m;
            const int n_out = MULTI ? mp->N[items.prob] : p.N;
            const bool got = mbar_wait(&acc_full[acc], acc_phase, abort_flag);
            // With stream-K every epilogue warp takes the same path through the
            // named barriers below, so they decide together.
            if (p.sk ? !epi_all(got) : !__all_sync(0xffffffffu, got)) {
                if (lane == 0) raise_error(abort_flag, p.err, 3);
                break;
            }
            tc_fence_after();
            const int row = mb * C::TILE_M + rloc;
            const uint32_t tm = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
            const bool split = p.sk && (kb0 > 0 || kb1 < nkb);
            if (!split) {
                #pragma unroll 1
                for (int c = 0; c < nw / 32; ++c) {
                    const int col = nb * BN + c0 + c * 32;
                    if (col >= n_out) break;
                    uint32_t v[32];
                    tmem_ld32(tm + (uint32_t)(c * 32), v);
                    tmem_ld_wait(v);
                    if (row < p.M) {
                        float f[32];
                        #pragma unroll
                        for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
                        uint16_t* dst;
                        if constexpr (MULTI) dst = mp->D[items.prob] + (int64_t)row * mp->ldd[items.prob] + col;
                        else                 dst = out_ptr(p, row, col);
                        store_bf16x32(dst, f);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (PAIR) mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[acc]), 0));
                    else                mbar_arrive(&acc_empty[acc]);
                }
            } else {
                split_piece<PAIR, BN>(p, tm, &acc_empty[acc], kb0 == 0 ? 0 : 1, unit, rank, q, lane, row, nb * BN);
            }
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync_all();   // no CTA leaves while its peer may still touch its memory
    if (warp == 1) {
        tc_fence_after();
        if constexpr (PAIR) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
        else                tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ------------------------------------------------ fused NF4 pair kernel ---
//
// The pair GEMM with the NF4 weight as B, converted in shared memory.  Three
// rings advance in lockstep, one slot per 128-wide K-block, each with its own
// barriers so that no stage waits on a chain of the others' latencies:
//   A ring   TMA of this CTA's 128 A rows (counted on the leader), released
//            by the MMA (a commit that arrives on both CTAs' barriers);
//   P ring   TMA of this CTA's packed NF4 tile (128 rows x 64 bytes, 64-byte
//            swizzle), issued by its own producer warp and released by the
//            converters as soon as they have read it;
//   B ring   the converted bf16 tile (128-byte swizzle, the MMA operand),
//            written by 8 converter warps, released by the MMA.
// The LoRA K-block's B (B_lora or A_lora) is copied into the B ring by the
// same converters, so every ring has the same slot sequence.
template <bool B_MN>
struct CfgN {
    static constexpr int BN = 256;
    static constexpr int A_SUB = BM * SUB * 2;      // 16 KB
    static constexpr int A_BYTES = 2 * A_SUB;       // 32 KB
    static constexpr int B_BYTES = 128 * BK * 2;    // 32 KB: 128 B rows x 128 contraction
    static constexpr int P_BYTES = 128 * 64;        // 8 KB packed
    static constexpr int RING_A = STAGES * A_BYTES;
    static constexpr int RING_B = STAGES * B_BYTES;
    static constexpr int RING_P = STAGES * P_BYTES;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = RING_A + RING_B + RING_P + BAR_BYTES + 1024 + 1024;
    static constexpr uint32_t IDESC = idesc_bf16(2 * BM, BN, 0, B_MN ? 1 : 0);
    static constexpr uint32_t TMEM_COLS = 2 * BN;
    static constexpr int THREADS = 192 + 32 * CONV_WARPS + 32;   // + converters + packed producer
};

template <bool B_MN>
__global__ void __launch_bounds__(CfgN<B_MN>::THREADS, 1)
    lsn_gemm_nf4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmP,
                        const __grid_constant__ CUtensorMap tmLA, const __grid_constant__ GemmArgs p) {
    using C = CfgN<B_MN>;
    constexpr int BN = C::BN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ringA = smem;
    uint8_t* ringB = smem + C::RING_A;
    uint8_t* ringP = ringB + C::RING_B;
    uint64_t* bars = reinterpret_cast<uint64_t*>(ringP + C::RING_P);
    uint64_t* fullA = bars;
    uint64_t* emptyA = fullA + STAGES;
    uint64_t* fullP = emptyA + STAGES;
    uint64_t* emptyP = fullP + STAGES;
    uint64_t* readyB = emptyP + STAGES;
    uint64_t* emptyB = readyB + STAGES;
    uint64_t* acc_full = emptyB + STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    float* dq_s = reinterpret_cast<float*>(ringP + C::RING_P + C::BAR_BYTES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int unit = (int)(blockIdx.x >> 1), nunits = (int)(gridDim.x >> 1);
    const int num_m = (p.M + 2 * BM - 1) / (2 * BM);
    const int num_n = (p.N + BN - 1) / BN;
    const int num_tiles = num_m * num_n;
    const int nkb = p.num_kb + (p.lora_k16 > 0 ? 1 : 0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&fullA[s], 1);
            mbar_init(&emptyA[s], 1);
            mbar_init(&fullP[s], 1);
            mbar_init(&emptyP[s], CONV_WARPS);
            mbar_init(&readyB[s], 2 * CONV_WARPS);
            mbar_init(&emptyB[s], 1);
        }
        for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 8); }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    for (int i = threadIdx.x; i < 256; i += blockDim.x) dq_s[i] = p.dq[i];
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA); tma_prefetch_desc(&tmP); tma_prefetch_desc(&tmLA);
    }
    if (warp == 1) { tmem_alloc_pair(tmem_holder, C::TMEM_COLS); tmem_relinquish_pair(); }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_launch_dependents();
    pdl_wait();
    const int conv_first_warp = 6, ppro_warp = 6 + CONV_WARPS;

    if (warp == 0) {
        if (lane == 0) {
            // -------------------------------------------------- A producer --
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = unit; tile < num_tiles && ok; tile += nunits) {
                const int m_row = (tile % num_m) * 2 * BM + (int)rank * BM;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&emptyA[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    uint8_t* sA = ringA + stage * C::A_BYTES;
                    const uint32_t fbar = mapa_shared(smem_u32(&fullA[stage]), 0);
                    if (leader) mbar_arrive_expect_tx(&fullA[stage], 2 * C::A_BYTES);
                    const bool lora = kb >= p.num_kb;
                    const CUtensorMap* ma = lora ? &tmLA : &tmA;
                    const int kc = lora ? 0 : kb * BK;
                    tma_load_2d_pair(sA, ma, kc, m_row, fbar);
                    tma_load_2d_pair(sA + C::A_SUB, ma, kc + SUB, m_row, fbar);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) raise_error(abort_flag, p.err, 1);
        }
    } else if (warp == ppro_warp) {
        if (lane == 0) {
            // --------------------------------------------- packed producer --
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = unit; tile < num_tiles && ok; tile += nunits) {
                const int n_off = (tile / num_m) * BN + (int)rank * 128;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&emptyP[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    const bool lora = kb >= p.num_kb;
                    mbar_arrive_expect_tx(&fullP[stage], lora ? 0u : (uint32_t)C::P_BYTES);
                    if (!lora) {
                        uint8_t* sP = ringP + stage * C::P_BYTES;
                        if (!B_MN) tma_load_2d(sP, &tmP, kb * 64, n_off, &fullP[stage]);
                        else       tma_load_2d(sP, &tmP, n_off / 2, kb * BK, &fullP[stage]);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) raise_error(abort_flag, p.err, 5);
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // -------------------------------------------------- MMA issuer --
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int tile = unit; tile < num_tiles && ok; tile += nunits) {
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&fullA[stage], phase, abort_flag)) { ok = false; break; }
                    if (!mbar_wait_cluster(&readyB[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(ringA + stage * C::A_BYTES);
                    const uint32_t b0 = smem_u32(ringB + stage * C::B_BYTES);
                    const int nk = (kb < p.num_kb) ? BK / 16 : p.lora_k16;
                    for (int k = 0; k < nk; ++k) {
                        const int j = k >> 2, kk = k & 3;
                        const uint64_t ad = smem_desc_sw128(a0 + j * C::A_SUB + kk * 32, 16, 1024);
                        const uint64_t bd = B_MN ? smem_desc_sw128(b0 + k * 2048, BK * 128, 1024)
                                                 : smem_desc_sw128(b0 + j * (BK * 128) + kk * 32, 16, 1024);
                        umma_bf16_pair(d_tmem, ad, bd, C::IDESC, (kb | k) ? 1u : 0u);
                    }
                    umma_commit_pair(&emptyA[stage]);
                    umma_commit_pair(&emptyB[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                umma_commit_pair(&acc_full[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
            if (!ok) raise_error(abort_flag, p.err, 2);
            umma_commit_pair(drain);
            mbar_wait(drain, 0, nullptr);
        }
    } else if (warp < conv_first_warp) {
        // -------------------------------------------------------- epilogue --
        const int q = warp & 3;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = unit; tile < num_tiles; tile += nunits) {
            const int mb = tile % num_m, nb = tile / num_m;
            const bool got = mbar_wait(&acc_full[acc], acc_phase, abort_flag);
            if (!__all_sync(0xffffffffu, got)) { if (lane == 0) raise_error(abort_flag, p.err, 3); break; }
            tc_fence_after();
            const int row = mb * 2 * BM + (int)rank * BM + q * 32 + lane;
            #pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                const int col = nb * BN + c * 32;
                if (col >= p.N) break;
                uint32_t v[32];
                tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + c * 32), v);
                tmem_ld_wait(v);
                if (row < p.M) {
                    uint4* dst = reinterpret_cast<uint4*>(p.D + (int64_t)row * p.ldd + col);
                    #pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        uint4 o;
                        o.x = pack_bf16x2(__uint_as_float(v[8 * i + 0]), __uint_as_float(v[8 * i + 1]));
                        o.y = pack_bf16x2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3]));
                        o.z = pack_bf16x2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5]));
                        o.w = pack_bf16x2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7]));
                        dst[i] = o;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[acc]), 0));
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
        }
    } else {
        // ------------------------------------------------------- converters --
        // Thread t owns one (row, 64-block) of the CTA's 128 x 128 B tile per
        // K-block: row = t % 128 (a B row: forward W row n; backward the
        // contraction row n of W), block = t / 128 (64 consecutive W
        // columns).  Its 64 bf16 land in one 128-byte row of a 128-byte
        // swizzled atom: block b's atom at b * 16 KB, row at (row/8)*1024 +
        // (row%8)*128, 16-byte chunk c at position c ^ (row % 8).
        const int t = threadIdx.x - 32 * conv_first_warp;
        const int row = t & 127, blk = t >> 7;
        const int64_t nblk_row = p.wcols / 64;
        const float off = *p.absmax_off;
        struct Meta { uint32_t code; float s2; bool ok; };
        auto fetch = [&](int tl, int k) -> Meta {
            Meta m{0u, 0.0f, false};
            if (tl >= num_tiles || k >= p.num_kb) return m;
            const int n_off = (tl / num_m) * BN + (int)rank * 128;
            const int64_t wr = B_MN ? (int64_t)k * BK + row : (int64_t)n_off + row;
            const int64_t wb = B_MN ? (int64_t)(n_off / 64) + blk : (int64_t)k * 2 + blk;
            if (wr < p.wrows && wb < nblk_row) {
                const int64_t bi = wr * nblk_row + wb;
                m.code = __ldg(p.absmax_q + bi);
                m.s2 = __ldg(p.absmax_s2 + (bi >> 8));
                m.ok = true;
            }
            return m;
        };
        int ft = unit, fk = 0;
        auto step = [&]() { if (++fk == nkb) { fk = 0; ft += nunits; } };
        Meta m0 = fetch(ft, fk);
        step();
        Meta m1 = fetch(ft, fk);
        step();
        int stage = 0;
        uint32_t phase = 0;
        bool bad = false;
        for (int tile = unit; tile < num_tiles && !bad; tile += nunits) {
            const int n_off = (tile / num_m) * BN + (int)rank * 128;
            for (int kb = 0; kb < nkb; ++kb) {
                const Meta cur = m0;
                m0 = m1;
                m1 = fetch(ft, fk);
                step();
                const bool got = mbar_wait(&fullP[stage], phase, abort_flag) &&
                                 mbar_wait(&emptyB[stage], phase ^ 1, abort_flag);
                if (!__all_sync(0xffffffffu, got)) { if (lane == 0) raise_error(abort_flag, p.err, 4); bad = true; break; }
                uint8_t* dst = ringB + stage * C::B_BYTES + blk * (BK * 128) + (row >> 3) * 1024 + (row & 7) * 128;
                if (kb < p.num_kb) {
                    if (cur.ok) {
                        const float ah = __fadd_rn(__fmul_rn(dq_s[cur.code], cur.s2), off);
                        uint32_t e[8];
                        #pragma unroll
                        for (int i = 0; i < 8; ++i)
                            e[i] = pack_bf16x2(__fmul_rn(p.level[2 * i], ah), __fmul_rn(p.level[2 * i + 1], ah));
                        uint32_t lo[4], hi[4];
                        #pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            lo[i] = prmt(e[2 * i], e[2 * i + 1], 0x6420u);
                            hi[i] = prmt(e[2 * i], e[2 * i + 1], 0x7531u);
                        }
                        const uint8_t* prow = ringP + stage * C::P_BYTES + row * 64;
                        uint4 pk[2];
                        #pragma unroll
                        for (int h = 0; h < 2; ++h)
                            pk[h] = *reinterpret_cast<const uint4*>(prow + (((2 * blk + h) ^ ((row >> 1) & 3)) << 4));
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&emptyP[stage]);   // packed slot read: release it early
                        #pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t w[4] = {pk[h].x, pk[h].y, pk[h].z, pk[h].w};
                            #pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int c = h * 4 + i;
                                *reinterpret_cast<uint4*>(dst + ((c ^ (row & 7)) << 4)) = nf4x8_to_bf16(w[i], lo, hi);
                            }
                        }
                    } else {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&emptyP[stage]);
                        #pragma unroll
                        for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(dst + (c << 4)) = make_uint4(0, 0, 0, 0);
                    }
                } else {
                    // LoRA K-block: copy the bf16 LoRA operand (zero-padded).
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&emptyP[stage]);
                    int64_t src_row = -1, col0 = 0;
                    int ncols = 0, ld = 0;
                    if (!B_MN) {            // B_lora [N, r]: row n, columns 0..r-1 (block 0 only)
                        const int64_t n = (int64_t)n_off + row;
                        if (blk == 0 && n < p.N) { src_row = n; col0 = 0; ncols = p.lora_r; ld = p.lora_r; }
                    } else {                // A_lora [r, N]: row j, columns n_off + 64 blk ..
                        const int64_t c0 = (int64_t)n_off + 64 * blk;
                        if (row < p.lora_r && c0 < p.N) { src_row = row; col0 = c0; ncols = 64; ld = p.N; }
                    }
                    #pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        uint4 v = make_uint4(0, 0, 0, 0);
                        if (src_row >= 0 && c * 8 < ncols)
                            v = __ldg(reinterpret_cast<const uint4*>(p.lora_b + src_row * ld + col0) + c);
                        *reinterpret_cast<uint4*>(dst + ((c ^ (row & 7)) << 4)) = v;
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&readyB[stage]), 0));
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

// --------------------------------------------------------- tensor maps ---

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// A 2-D bf16 tensor [outer, inner] with row stride `stride_elems`, read in
// boxes of box_inner (64 = 128 bytes, the swizzle span) x box_outer rows.
lsn_status make_map(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, int64_t stride_elems,
                    int box_inner, int box_outer, bool bytes = false) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(LSN_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const int esize = bytes ? 1 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
    cuuint64_t strides[1] = {(cuuint64_t)stride_elems * esize};
    cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
    cuuint32_t es[2] = {1, 1};
    // bf16 operand tiles use the 128-byte swizzle the MMA descriptors expect;
    // packed NF4 tiles (64-byte rows) use the 64-byte swizzle, which keeps the
    // converters' 16-byte reads free of bank conflicts.
    CUresult r = fn(m, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
                    dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    bytes ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(LSN_ERR_CUDA, "cuTensorMapEncodeTiled failed (code " + std::to_string((int)r) + ")");
    return LSN_OK;
}

template <bool PAIR, int BN, bool B_MN, bool MULTI = false>
lsn_status launch_cfg(const AMaps& a, const CUtensorMap& b, const CUtensorMap& la, const CUtensorMap& lb,
                      const GemmArgs& args, cudaStream_t st, const MultiParam<MULTI>& mpar = {}, int multi_units = 0) {
    using C = Cfg<PAIR, BN, B_MN>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(lsn_gemm_kernel<PAIR, BN, B_MN, MULTI>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    });
    if (attr_err != cudaSuccess) return fail_cuda(attr_err, "cudaFuncSetAttribute(gemm smem)");
    const int tiles = ((args.M + C::TILE_M - 1) / C::TILE_M) * ((args.N + BN - 1) / BN);
    const int units = MULTI ? multi_units
                            : args.sk ? (PAIR ? sm_count() / 2 : sm_count()) : gemm_units(tiles, PAIR);
    const int grid = (PAIR ? 2 : 1) * units;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (PAIR) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = 2;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    na += pdl_attr(&attr[na]);
    cfg.attrs = attr;
    cfg.numAttrs = na;
    LSN_CUDA_TRY(cudaLaunchKernelEx(&cfg, lsn_gemm_kernel<PAIR, BN, B_MN, MULTI>, a, b, la, lb, args, mpar));
    return LSN_OK;
}

}  // namespace

lsn_status make_tmap_2d(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, int64_t stride_elems,
                        int box_inner, int box_outer, bool bytes) {
    return make_map(m, base, inner, outer, stride_elems, box_inner, box_outer, bytes);
}

// Kernel choice from the shape alone: the 2-SM kernel (256 x 256 tiles on
// CTA pairs) when it has at least one full wave of pairs on a 148-SM part,
// else the 1-SM kernel with 128 x 128 tiles.
bool gemm_use_pairs(int64_t M, int64_t N) {
    const int64_t pair_tiles = ((M + 255) / 256) * ((N + 255) / 256);
    return pair_tiles >= 74;
}

// The fused NF4 variant: B is the NF4 weight w (W [wrows, wcols] row-major;
// forward: N = wrows, Kc = wcols; backward: N = wcols, Kc = wrows).  Runs on
// the pair kernel only; returns LSN_ERR_UNSUPPORTED for shapes that do not use
// it so the caller can fall back to dequantise + bf16 GEMM.
lsn_status launch_gemm_nf4(const uint16_t* A, int64_t lda, const lsn_nf4_weight* w, bool b_mn, const uint16_t* LA,
                           const uint16_t* LB, int r, int64_t M, int64_t N, int64_t Kc, uint16_t* D, int64_t ldd,
                           int* err, cudaStream_t st) {
    if (!gemm_use_pairs(M, N)) return LSN_ERR_UNSUPPORTED;
    const Nf4Tables& T = nf4_tables();
    CUtensorMap ma, mp, mla;
    lsn_status s;
    if ((s = make_map(&ma, A, Kc, M, lda, SUB, BM)) != LSN_OK) return s;
    // packed [wrows, wcols/2] bytes, boxes of 64 bytes x 128 rows
    if ((s = make_map(&mp, w->packed, w->cols / 2, w->rows, w->cols / 2, 64, 128, true)) != LSN_OK) return s;
    if (r > 0) {
        if ((s = make_map(&mla, LA, r, M, r, SUB, BM)) != LSN_OK) return s;
    } else {
        mla = ma;                                   // no LoRA term: never read
    }
    GemmArgs args{};
    args.M = (int)M;
    args.N = (int)N;
    args.num_kb = (int)((Kc + BK - 1) / BK);
    args.lora_k16 = (r + 15) / 16;
    args.D = D;
    args.ldd = ldd;
    args.err = err;
    args.absmax_q = w->absmax_q;
    args.absmax_s2 = w->absmax_s2;
    args.absmax_off = w->offset;
    args.wrows = (int)w->rows;
    args.wcols = (int)w->cols;
    std::memcpy(args.level, T.level, sizeof(args.level));
    std::memcpy(args.dq, T.dq, sizeof(args.dq));
    args.lora_b = LB;
    args.lora_r = r;
    auto launch = [&](auto kernel, int smem_bytes, int threads) -> lsn_status {
        const int tiles = ((args.M + 255) / 256) * ((args.N + 255) / 256);
        const int grid = 2 * gemm_units(tiles, true);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)grid);
        cfg.blockDim = dim3((unsigned)threads);
        cfg.dynamicSmemBytes = smem_bytes;
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1 + pdl_attr(&attr[1]);
        LSN_CUDA_TRY(cudaLaunchKernelEx(&cfg, kernel, ma, mp, mla, args));
        return LSN_OK;
    };
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(lsn_gemm_nf4_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        CfgN<false>::SMEM_BYTES);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(lsn_gemm_nf4_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            CfgN<true>::SMEM_BYTES);
    });
    if (attr_err != cudaSuccess) return fail_cuda(attr_err, "cudaFuncSetAttribute(gemm nf4 smem)");
    return b_mn ? launch(lsn_gemm_nf4_kernel<true>, CfgN<true>::SMEM_BYTES, CfgN<true>::THREADS)
                : launch(lsn_gemm_nf4_kernel<false>, CfgN<false>::SMEM_BYTES, CfgN<false>::THREADS);
}

// D = A . op(B) + LA . op(LB).
//   A  [M, Kc] bf16 row-major (lda), K-major.
//   b_mn == false: B is [N, Kc] (ldb), LB is [N, r]   (forward: W, B_lora)
//   b_mn == true : B is [Kc, N] (ldb), LB is [r, N]   (backward: W, A_lora)
//   LA [M, r] (bf16(s u) or bf16(s g)); r == 0 disables the LoRA term.
size_t gemm_split_ws_bytes() {
    const size_t pair = (size_t)(kSplitMaxUnits / 2 + 1) * 2 * 2 * 128 * 256 * sizeof(float);
    const size_t one = (size_t)(kSplitMaxUnits + 1) * 2 * 1 * 128 * 128 * sizeof(float);
    return kSplitCntBytes + (pair > one ? pair : one);
}

GemmSplitWs gemm_split_ws(void* base) {
    GemmSplitWs w;
    char* b = reinterpret_cast<char*>(base);
    w.cnt = reinterpret_cast<int*>(b);
    w.part = b ? reinterpret_cast<float*>(b + kSplitCntBytes) : nullptr;
    return w;
}

namespace {
std::atomic<int> g_stream_k{0};
std::atomic<int> g_min_units{0};
std::atomic<int> g_tail_split{0};
std::atomic<int> g_multi{1};
}

void gemm_set_stream_k(bool on) { g_stream_k.store(on ? 1 : 0); }
bool gemm_stream_k() { return g_stream_k.load() != 0; }
void gemm_set_min_units(bool on) { g_min_units.store(on ? 1 : 0); }
bool gemm_min_units() { return g_min_units.load() != 0; }
void gemm_set_tail_split(bool on) { g_tail_split.store(on ? 1 : 0); }
bool gemm_tail_split() { return g_tail_split.load() != 0; }
void gemm_set_multi(bool on) { g_multi.store(on ? 1 : 0); }
bool gemm_multi() { return g_multi.load() != 0; }

// Workers (CTA pairs, or CTAs) of a persistent GEMM over `tiles` whole tiles:
// with LSN_OPT_GEMM_MIN_UNITS the fewest that still finish in the same number
// of rounds of tiles as all the SMs would (the rest of the SMs stay free for
// work on other streams, at no cost to this GEMM); else one per SM (pair).
int gemm_units(int64_t tiles, bool pair) {
    const int64_t all = pair ? sm_count() / 2 : sm_count();
    if (tiles <= 0) return 1;
    if (!gemm_min_units()) return (int)(tiles < all ? tiles : all);
    const int64_t rounds = (tiles + all - 1) / all;
    return (int)((tiles + rounds - 1) / rounds);
}

lsn_status launch_gemm_grouped(const GemmGroup& g, const uint16_t* B, int64_t ldb, bool b_mn, const uint16_t* LA,
                               const uint16_t* LB, int r, int64_t M, int64_t N, int64_t Kc, uint16_t* D,
                               int64_t ldd, int* err, cudaStream_t st, const GemmSplitWs* split) {
    if (g.na < 1 || g.na > kMaxSeg || g.nseg < 0 || g.nseg > kMaxSeg)
        return fail(LSN_ERR_INVALID_ARG, "grouped GEMM: bad operand or segment count");
    const bool pair = gemm_use_pairs(M, N);
    const int b_rows = 128;                         // B rows staged per CTA: BN/2 = 128 (pair) or BN = 128
    AMaps ma;
    CUtensorMap mb, mla, mlb;
    lsn_status s;
    GemmArgs args{};
    int64_t kb_acc = 0;
    for (int i = 0; i < g.na; ++i) {
        if ((s = make_map(&ma.m[i], g.A[i], g.a_kc[i], M, g.lda[i], SUB, BM)) != LSN_OK) return s;
        args.a_kb[i] = (int)kb_acc;
        if (i + 1 < g.na && g.a_kc[i] % BK != 0)
            return fail(LSN_ERR_INVALID_ARG, "grouped GEMM: inner A extents must be multiples of 128");
        kb_acc += (g.a_kc[i] + BK - 1) / BK;
    }
    args.a_kb[g.na] = (int)kb_acc;
    args.na = g.na;
    for (int i = g.na; i < kMaxSeg; ++i) ma.m[i] = ma.m[0];
    if (!b_mn) {
        if ((s = make_map(&mb, B, Kc, N, ldb, SUB, b_rows)) != LSN_OK) return s;
    } else {
        if ((s = make_map(&mb, B, N, Kc, ldb, 64, BK)) != LSN_OK) return s;
    }
    if (r > 0) {
        if ((s = make_map(&mla, LA, r, M, r, SUB, BM)) != LSN_OK) return s;
        if (!b_mn) {
            if ((s = make_map(&mlb, LB, r, N, r, SUB, b_rows)) != LSN_OK) return s;
        } else {
            if ((s = make_map(&mlb, LB, N, r, N, 64, BK)) != LSN_OK) return s;
        }
    } else {                                        // no LoRA term: the maps are never read
        mla = ma.m[0];
        mlb = mb;
    }
    args.M = (int)M;
    args.N = (int)N;
    args.num_kb = (int)((Kc + BK - 1) / BK);
    if (args.num_kb != args.a_kb[g.na]) return fail(LSN_ERR_INVALID_ARG, "grouped GEMM: A extents do not add up to Kc");
    args.lora_k16 = (r + 15) / 16;
    args.D = D;
    args.ldd = ldd;
    args.err = err;
    args.nseg = g.nseg;
    int64_t c0 = 0;
    for (int i = 0; i < g.nseg; ++i) {
        args.seg_col[i] = (int)c0;
        args.seg_D[i] = g.seg_D[i];
        args.seg_ld[i] = g.seg_ld[i];
        c0 += g.seg_cols[i];
    }
    args.seg_col[g.nseg] = (int)c0;
    if (g.nseg > 0 && c0 != N) return fail(LSN_ERR_INVALID_ARG, "grouped GEMM: segments do not add up to N");
    // Stream-K when the tiles do not fill whole waves of workers (and there are
    // at least as many tiles as workers, so that a tile has at most two pieces).
    {
        const int64_t tile_m = pair ? 256 : 128, tile_n = pair ? 256 : 128;
        const int64_t tiles = ((M + tile_m - 1) / tile_m) * ((N + tile_n - 1) / tile_n);
        const int units = pair ? sm_count() / 2 : sm_count();
        if (split && split->cnt && gemm_stream_k() && units <= (pair ? kSplitMaxUnits / 2 : kSplitMaxUnits) &&
            tiles >= units && tiles % units != 0) {
            args.sk = 1;
            args.sk_per = (tiles * args.num_kb + units - 1) / units;     // base blocks only (see Items)
            args.sk_part = split->part;
            args.sk_cnt = split->cnt;
        }
    }
    // Tail split of the whole-tile schedule (see GemmArgs::tq): quanta of 64
    // columns (32 B rows per CTA of the pair) for a K-major B; 128 for an
    // MN-major B, whose per-CTA share must stay whole 64-column swizzle atoms.
    if (pair && !args.sk && gemm_tail_split()) {
        const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
        const int64_t units = gemm_units(tiles, true);
        const int tq = b_mn ? 128 : 64, qpt = 256 / tq;
        const int64_t rem = tiles % units;
        if (tiles > units && rem != 0 && (rem * qpt + units - 1) / units < qpt) args.tq = tq;
    }
    if (pair) return b_mn ? launch_cfg<true, 256, true>(ma, mb, mla, mlb, args, st)
                          : launch_cfg<true, 256, false>(ma, mb, mla, mlb, args, st);
    return b_mn ? launch_cfg<false, 128, true>(ma, mb, mla, mlb, args, st)
                : launch_cfg<false, 128, false>(ma, mb, mla, mlb, args, st);
}

// ------------------------------------------------------ several problems --

namespace {

// A balanced static schedule of whole tiles: tiles in decreasing cost
// (contraction blocks, the LoRA block included), each given to the worker with
// the least summed cost so far (lowest index on ties).  Depends on the shapes
// only, so it is computed once per shape family and kept.
struct MultiSched {
    std::vector<uint16_t> start, tile;
};

const MultiSched& multi_schedule(int units, int num_m, const int* ntiles, const int* cost, int n) {
    static std::mutex mu;
    static std::map<std::vector<int>, MultiSched> cache;
    std::vector<int> key{units, num_m, n};
    for (int i = 0; i < n; ++i) { key.push_back(ntiles[i]); key.push_back(cost[i]); }
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    std::vector<int> order(n), first(n + 1, 0);
    for (int i = 0; i < n; ++i) { order[i] = i; first[i + 1] = first[i] + ntiles[i]; }
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cost[a] > cost[b]; });
    std::vector<int64_t> load(units, 0);
    std::vector<std::vector<int>> lists(units);
    for (int i : order) {
        for (int t = 0; t < ntiles[i]; ++t) {
            int u = 0;
            for (int v = 1; v < units; ++v)
                if (load[v] < load[u]) u = v;
            load[u] += cost[i];
            lists[u].push_back(first[i] + t);
        }
    }
    MultiSched s;
    s.start.push_back(0);
    for (int u = 0; u < units; ++u) {
        for (int t : lists[u]) s.tile.push_back((uint16_t)t);
        s.start.push_back((uint16_t)s.tile.size());
    }
    return cache.emplace(std::move(key), std::move(s)).first->second;
}

}  // namespace

int gemm_multi_max_problems() { return kMultiMaxProb; }

lsn_status gemm_merged_schedule(int units, int n, const int* ntiles, const int* cost, int* start, int* tile,
                                int max_tiles) {
    if (units < 1 || n < 1 || n > 64 || !ntiles || !cost || !start || !tile || max_tiles < 0)
        return fail(LSN_ERR_INVALID_ARG, "lsn_gemm_merged_schedule: bad arguments");
    int64_t total = 0;
    for (int i = 0; i < n; ++i) {
        if (ntiles[i] < 0 || cost[i] < 1) return fail(LSN_ERR_INVALID_ARG, "lsn_gemm_merged_schedule: bad tile count or cost");
        total += ntiles[i];
    }
    if (total > max_tiles || total > 65535) return fail(LSN_ERR_INVALID_ARG, "lsn_gemm_merged_schedule: too many tiles");
    const MultiSched& sc = multi_schedule(units, 0, ntiles, cost, n);
    for (int u = 0; u <= units; ++u) start[u] = sc.start[u];
    for (size_t t = 0; t < sc.tile.size(); ++t) tile[t] = sc.tile[t];
    return LSN_OK;
}

bool gemm_multi_fits(const GemmProblem* pr, int n, int64_t M) {
    if (n < 1 || n > kMultiMaxProb || M <= 0 || sm_count() / 2 > kMultiMaxUnits) return false;
    int64_t tiles = 0;
    const int64_t num_m = (M + 255) / 256;
    for (int i = 0; i < n; ++i) tiles += num_m * ((pr[i].N + 255) / 256);
    return tiles <= kMultiMaxTiles;
}

lsn_status launch_gemm_multi(const GemmProblem* pr, int n, bool b_mn, int64_t M, int r, int* err,
                             cudaStream_t st) {
    if (!gemm_multi_fits(pr, n, M)) return fail(LSN_ERR_INVALID_ARG, "multi-problem GEMM: too many problems or tiles");
    MultiProbs mp{};
    mp.nprob = n;
    const int num_m = (int)((M + 255) / 256);
    int ntiles[kMultiMaxProb], cost[kMultiMaxProb];
    lsn_status s;
    for (int i = 0; i < n; ++i) {
        const GemmProblem& q = pr[i];
        const int ri = q.LA ? (q.lr > 0 ? q.lr : r) : 0;
        const int64_t ld_la = q.ld_la > 0 ? q.ld_la : ri;
        if (q.na < 1 || q.na > kMaxSeg) return fail(LSN_ERR_INVALID_ARG, "multi-problem GEMM: bad A part count");
        int64_t kb_acc = 0;
        for (int j = 0; j < q.na; ++j) {
            const int64_t akc = q.na == 1 ? q.Kc : q.a_kc[j];
            if ((s = make_map(&mp.a[i * kMaxSeg + j], q.A[j], akc, M, q.lda[j], SUB, BM)) != LSN_OK) return s;
            if (j + 1 < q.na && akc % BK != 0)
                return fail(LSN_ERR_INVALID_ARG, "multi-problem GEMM: inner A parts must be multiples of 128 wide");
            mp.a_kb[i][j] = (int)kb_acc;
            kb_acc += (akc + BK - 1) / BK;
        }
        mp.a_kb[i][q.na] = (int)kb_acc;
        mp.na[i] = q.na;
        for (int j = q.na; j < kMaxSeg; ++j) mp.a[i * kMaxSeg + j] = mp.a[i * kMaxSeg];
        if (!b_mn) {
            if ((s = make_map(&mp.b[i], q.B, q.Kc, q.N, q.ldb, SUB, 128)) != LSN_OK) return s;
        } else {
            if ((s = make_map(&mp.b[i], q.B, q.N, q.Kc, q.ldb, 64, BK)) != LSN_OK) return s;
        }
        if (ri > 0) {
            if ((s = make_map(&mp.la[i], q.LA, ri, M, ld_la, SUB, BM)) != LSN_OK) return s;
            if (!b_mn) {
                if ((s = make_map(&mp.lb[i], q.LB, ri, q.N, ri, SUB, 128)) != LSN_OK) return s;
            } else {
                if ((s = make_map(&mp.lb[i], q.LB, q.N, ri, q.N, 64, BK)) != LSN_OK) return s;
            }
        } else {                                        // no LoRA term: never read
            mp.la[i] = mp.a[i * kMaxSeg];
            mp.lb[i] = mp.b[i];
        }
        mp.N[i] = (int)q.N;
        mp.num_kb[i] = (int)((q.Kc + BK - 1) / BK);
        if (mp.num_kb[i] != mp.a_kb[i][q.na])
            return fail(LSN_ERR_INVALID_ARG, "multi-problem GEMM: A parts do not add up to Kc");
        mp.lora_k16[i] = (ri + 15) / 16;
        mp.D[i] = q.D;
        mp.ldd[i] = q.ldd;
        ntiles[i] = num_m * (int)((q.N + 255) / 256);
        cost[i] = mp.num_kb[i] + (ri > 0 ? 1 : 0);
        mp.tile0[i + 1] = mp.tile0[i] + ntiles[i];
    }
    int units = sm_count() / 2;
    if (mp.tile0[n] < units) units = mp.tile0[n];
    if (units < 1) return LSN_OK;
    const MultiSched& sc = multi_schedule(units, num_m, ntiles, cost, n);
    std::copy(sc.start.begin(), sc.start.end(), mp.start);
    std::copy(sc.tile.begin(), sc.tile.end(), mp.tile);
    GemmArgs args{};
    args.M = (int)M;
    args.N = 0;
    args.err = err;
    args.na = 1;
    AMaps ma;
    for (int i = 0; i < kMaxSeg; ++i) ma.m[i] = mp.a[0];
    return b_mn ? launch_cfg<true, 256, true, true>(ma, mp.b[0], mp.la[0], mp.lb[0], args, st, mp, units)
                : launch_cfg<true, 256, false, true>(ma, mp.b[0], mp.la[0], mp.lb[0], args, st, mp, units);
}

lsn_status launch_gemm(const uint16_t* A, int64_t lda, const uint16_t* B, int64_t ldb, bool b_mn, const uint16_t* LA,
                       const uint16_t* LB, int r, int64_t M, int64_t N, int64_t Kc, uint16_t* D, int64_t ldd,
                       int* err, cudaStream_t st, const GemmSplitWs* split) {
    GemmGroup g;
    g.na = 1;
    g.A[0] = A;
    g.lda[0] = lda;
    g.a_kc[0] = Kc;
    return launch_gemm_grouped(g, B, ldb, b_mn, LA, LB, r, M, N, Kc, D, ldd, err, st, split);
}

}  // namespace lsn
