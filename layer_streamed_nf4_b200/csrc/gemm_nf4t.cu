// Forward GEMM of the NF4 LoRA linear with the base converted straight into
// tensor memory (sm_100a: tcgen05 with the A operand in TMEM):
//
//   y^T[n, t] = sum_k W[n, k] x[t, k]  +  sum_j B[n, j] (s u)[t, j]
//
// "Can You Fine-Tune a 27B Model on a Laptop? (I Did the Math)", 2:19-2:29
// (a 4-bit base whose block constants are quantised a second time) and
// 1:47-1:58 (the adapter rides alongside the frozen weights): the NF4 codes of
// a weight tile are staged by TMA, unpacked, looked up and scaled in
// registers, and written into tensor memory as the A operand of the 2-SM MMA,
// so no bf16 copy of W exists in HBM or in shared memory.  With W as A the
// accumulator is y^T (lanes = output features, columns = tokens); the
// epilogue transposes it through a small shared-memory tile per warp.
//
// Tile: a CTA pair covers 256 rows of W (128 per CTA: its TMEM lanes) and 256
// tokens (each CTA stages 128 token rows of x; the MMA reads both halves).
// Tensor memory, 512 columns: the fp32 accumulator [128 lanes x 256 tokens]
// in columns 0-255, four 128-wide contraction stages of bf16 A in 256-511.
//
// Warps (640 threads):
//   0      x producer: TMA of this CTA's 128 token rows of x per stage (both
//          CTAs' loads complete on the pair leader's barrier);
//   1      TMEM allocation; one lane of the leader issues the MMAs;
//   2..17  converters, then epilogue.  Converter warp c = w - 2 owns TMEM
//          lane quadrant w % 4, NF4 block (c / 4) % 2 of the two in a
//          128-wide stage, and every other stage (c / 8 picks which): its
//          thread i converts row 32 (w % 4) + i of the CTA's W rows (32 bytes
//          of codes -> 64 bf16) and stores it with one tcgen05.st of 32
//          columns.  Two warp sets on alternate stages give each warp two
//          stages' time for one stage's conversion.  Once the first stages
//          of the next tile are converted, the same warps drain the
//          accumulator (a quadrant's four warps take 64 tokens each);
//   18     codes producer: TMA of this CTA's 128 W rows x 64 bytes per stage;
//   19     relay: once the eight converter warps writing a stage are done
//          (a CTA-local barrier), one arrival on the pair leader's barrier.
//          The cluster-scope release of that arrival is paid by this thread
//          alone, not by every converter warp for every stage.
// Every wait is bounded; a wait that runs out sets *err and the CTA winds
// down instead of hanging.
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "launch.cuh"

namespace lsn {
namespace {

constexpr int NT_STAGES = 4;
constexpr int NT_BK = 128;                     // contraction per stage
constexpr int NT_XSUB = 128 * 64 * 2;          // 128 token rows x 64 bf16 (one 128-byte swizzle atom wide)
constexpr int NT_XBYTES = 2 * NT_XSUB;         // 32 KB per stage
constexpr int NT_PBYTES = 128 * 64;            // 128 W rows x 64 bytes of codes: 8 KB per stage
// A warp's 32 x 32 bf16 transpose tile: 32 rows (tokens) of 80 bytes (32 bf16
// + 16 bytes of padding, so that 8 consecutive rows read as 16-byte chunks
// fall into distinct banks), rows 16..31 shifted by another 64 bytes (so that
// the two half-warps, writing rows j and 16 + j, hit distinct banks).
constexpr int NT_EPI_ROW = 80;
constexpr int NT_EPI_HALF = 16 * NT_EPI_ROW + 64;
constexpr int NT_EPI_BYTES = NT_EPI_HALF + 16 * NT_EPI_ROW;
constexpr int NT_PAR = 2;                      // converter warp sets, taking alternate stages
constexpr int NT_CONV_PER_STAGE = 8;           // converter warps writing one stage (2 per lane quadrant)
constexpr int NT_CONV_WARPS = NT_CONV_PER_STAGE * NT_PAR;
constexpr int NT_THREADS = 64 + 32 * NT_CONV_WARPS + 64;
constexpr int NT_PPRO_WARP = 2 + NT_CONV_WARPS;
constexpr int NT_RELAY_WARP = NT_PPRO_WARP + 1;
constexpr int NT_BAR_BYTES = 512;
constexpr int NT_SMEM_BYTES =
    NT_STAGES * (NT_XBYTES + NT_PBYTES) + NT_CONV_WARPS * NT_EPI_BYTES + NT_BAR_BYTES + 1024 + 1024;
constexpr uint32_t NT_TMEM_COLS = 512;
constexpr uint32_t NT_ACC_COL = 0, NT_A_COL = 256;
constexpr uint32_t NT_IDESC = idesc_bf16(256, 256, 0, 0);

struct Nf4tArgs {
    int M, N;                // tokens (rows of y), output features (rows of W)
    int num_kb;              // 128-wide contraction stages of the base term
    int lora_k16;            // K = 16 MMAs of the LoRA term (0: none)
    int kblk;                // 64-element NF4 blocks per row of W (Kc / 64)
    uint16_t* y;
    int64_t ldy;
    int* err;
    const uint8_t* absmax_q;
    const float* absmax_s2;
    const float* absmax_off;
    const uint16_t* lora_b;  // B [N, r] bf16
    int lora_r;
    float level[16];
    float dq[256];
};

__device__ __forceinline__ void nt_raise(volatile int* abort_flag, int* err, int code) {
    *abort_flag = 1;
    if (err) atomicExch(err, code);
}

__global__ void __launch_bounds__(NT_THREADS, 1)
    lsn_gemm_nf4t_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmP,
                         const __grid_constant__ CUtensorMap tmLA, const __grid_constant__ Nf4tArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ringX = smem;
    uint8_t* ringP = ringX + NT_STAGES * NT_XBYTES;
    uint8_t* epi = ringP + NT_STAGES * NT_PBYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(epi + NT_CONV_WARPS * NT_EPI_BYTES);
    uint64_t* fullX = bars;                       // x of a stage landed (both CTAs; leader's copy counts)
    uint64_t* emptyX = fullX + NT_STAGES;         // MMAs done reading x of a stage (both CTAs)
    uint64_t* fullP = emptyX + NT_STAGES;         // codes of a stage landed (this CTA)
    uint64_t* emptyP = fullP + NT_STAGES;         // converters done reading codes (this CTA)
    uint64_t* readyA = emptyP + NT_STAGES;        // A stage written in both CTAs (leader; one relay arrival each)
    uint64_t* emptyA = readyA + NT_STAGES;        // MMAs done reading an A stage (both CTAs)
    uint64_t* convDone = emptyA + NT_STAGES;      // this CTA's converters wrote an A stage (local)
    uint64_t* acc_full = convDone + NT_STAGES;
    uint64_t* acc_empty = acc_full + 1;           // accumulator drained by both CTAs' epilogues (leader)
    uint64_t* drain = acc_empty + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    float* dq_s = reinterpret_cast<float*>(bars + NT_BAR_BYTES / 8);   // 256 floats after the barrier block

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int unit = (int)(blockIdx.x >> 1), nunits = (int)(gridDim.x >> 1);
    const int num_w = (p.N + 255) / 256;          // tiles along W rows
    const int num_t = (p.M + 255) / 256;          // tiles along tokens
    const int num_tiles = num_w * num_t;
    const int nkb = p.num_kb + (p.lora_k16 > 0 ? 1 : 0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < NT_STAGES; ++s) {
            mbar_init(&fullX[s], 1);
            mbar_init(&emptyX[s], 1);
            mbar_init(&fullP[s], 1);
            mbar_init(&emptyP[s], NT_CONV_PER_STAGE);
            mbar_init(&readyA[s], 2);
            mbar_init(&emptyA[s], 1);
            mbar_init(&convDone[s], NT_CONV_PER_STAGE);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 2 * NT_CONV_WARPS);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    for (int i = threadIdx.x; i < 256; i += blockDim.x) dq_s[i] = p.dq[i];
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmP);
        if (p.lora_k16 > 0) tma_prefetch_desc(&tmLA);
    }
    if (warp == 1) { tmem_alloc_pair(tmem_holder, NT_TMEM_COLS); tmem_relinquish_pair(); }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_launch_dependents();
    pdl_wait();

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------- x producer --
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = unit; tile < num_tiles && ok; tile += nunits) {
                const int t_row = (tile / num_w) * 256 + (int)rank * 128;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&emptyX[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    uint8_t* sX = ringX + stage * NT_XBYTES;
                    const uint32_t fbar = mapa_shared(smem_u32(&fullX[stage]), 0);
                    if (leader) mbar_arrive_expect_tx(&fullX[stage], 2 * NT_XBYTES);
                    const bool lora = kb >= p.num_kb;
                    const CUtensorMap* m = lora ? &tmLA : &tmX;
                    const int kc = lora ? 0 : kb * NT_BK;
                    tma_load_2d_pair(sX, m, kc, t_row, fbar);
                    tma_load_2d_pair(sX + NT_XSUB, m, kc + 64, t_row, fbar);
                    if (++stage == NT_STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) nt_raise(abort_flag, p.err, 11);
        }
    } else if (warp == NT_PPRO_WARP) {
        if (lane == 0) {
            // --------------------------------------------- codes producer --
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = unit; tile < num_tiles && ok; tile += nunits) {
                const int w_row = (tile % num_w) * 256 + (int)rank * 128;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&emptyP[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    const bool lora = kb >= p.num_kb;
                    mbar_arrive_expect_tx(&fullP[stage], lora ? 0u : (uint32_t)NT_PBYTES);
                    if (!lora) tma_load_2d(ringP + stage * NT_PBYTES, &tmP, kb * 64, w_row, &fullP[stage]);
                    if (++stage == NT_STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) nt_raise(abort_flag, p.err, 12);
        }
    } else if (warp == NT_RELAY_WARP) {
        if (lane == 0) {
            // ------------------------------------------------------ relay --
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            const uint32_t ready0 = mapa_shared(smem_u32(&readyA[0]), 0);
            for (int tile = unit; tile < num_tiles && ok; tile += nunits) {
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&convDone[stage], phase, abort_flag)) { ok = false; break; }
                    mbar_arrive_cluster(ready0 + (uint32_t)(stage * 8));
                    if (++stage == NT_STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) nt_raise(abort_flag, p.err, 15);
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------------------------- MMA issuer --
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            const uint32_t d_tmem = tmem_base + NT_ACC_COL;
            for (int tile = unit; tile < num_tiles && ok; tile += nunits) {
                if (!mbar_wait(acc_empty, acc_phase ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&fullX[stage], phase, abort_flag)) { ok = false; break; }
                    if (!mbar_wait_cluster(&readyA[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t x0 = smem_u32(ringX + stage * NT_XBYTES);
                    const uint32_t a0 = tmem_base + NT_A_COL + (uint32_t)(stage * 64);
                    const int nk = kb < p.num_kb ? NT_BK / 16 : p.lora_k16;
                    for (int k = 0; k < nk; ++k) {
                        const int j = k >> 2, kk = k & 3;          // x sub-tile, step inside it
                        const uint64_t bd = smem_desc_sw128(x0 + j * NT_XSUB + kk * 32, 16, 1024);
                        umma_bf16_pair_ta(d_tmem, a0 + (uint32_t)(k * 8), bd, NT_IDESC, (kb | k) ? 1u : 0u);
                    }
                    umma_commit_pair(&emptyX[stage]);
                    umma_commit_pair(&emptyA[stage]);
                    if (++stage == NT_STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                umma_commit_pair(acc_full);
                acc_phase ^= 1;
            }
            if (!ok) nt_raise(abort_flag, p.err, 13);
            umma_commit_pair(drain);                        // every MMA completes before TMEM is freed
            mbar_wait(drain, 0, nullptr);
        }
    } else {
        // ------------------------------------------ converters + epilogue --
        const int cw = warp - 2;                             // converter warp 0 .. NT_CONV_WARPS - 1
        const int q = warp & 3;                              // TMEM lane quadrant
        const int h = (cw >> 2) & 1;                         // NF4 block of the stage
        const int par = cw >> 3;                             // stages g with g % NT_PAR == par
        const int rloc = q * 32 + lane;                      // W row of the CTA = TMEM lane
        const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
        const float off = *p.absmax_off;
        uint8_t* tp = epi + cw * NT_EPI_BYTES;               // this warp's transpose tile
        uint32_t acc_phase = 0;
        bool bad = false;
        const int first_conv = nkb < NT_STAGES ? nkb : NT_STAGES;   // stages converted before draining
        const int epi_chunk0 = (h + 2 * par) * (8 / (2 * NT_PAR));  // this warp's 32-token chunks
        constexpr int kEpiChunks = 8 / (2 * NT_PAR);

        // Drain the accumulator of `tile`: this warp's chunks of 32 of its 256
        // tokens for the 32 W rows of its quadrant, transposed to y[token, feature].
        auto epilogue = [&](int tile) -> bool {
            const bool got = mbar_wait(acc_full, acc_phase, abort_flag);
            if (!__all_sync(0xffffffffu, got)) return false;
            acc_phase ^= 1;
            tc_fence_after();
            const int n_base = (tile % num_w) * 256 + (int)rank * 128 + q * 32;
            const int t_tile = (tile / num_w) * 256;
            #pragma unroll 1
            for (int c = epi_chunk0; c < epi_chunk0 + kEpiChunks; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem_base + lane_addr + NT_ACC_COL + (uint32_t)(c * 32), v);
                tmem_ld_wait(v);
                // Lane i holds feature n_base + i for tokens 32c .. 32c+31.  Lanes 2m and
                // 2m+1 swap halves, so that the even lane holds features (2m, 2m+1) of
                // tokens 0..15 and the odd lane those of tokens 16..31, each pair one
                // 32-bit word of its token's row in the transpose tile.
                const bool odd = lane & 1;
                const uint32_t col = (uint32_t)(lane >> 1) * 4;
                const uint32_t half = odd ? NT_EPI_HALF : 0;
                #pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const uint32_t mine = odd ? v[16 + j] : v[j];
                    const uint32_t other = __shfl_xor_sync(0xffffffffu, odd ? v[j] : v[16 + j], 1);
                    const uint32_t w = odd ? pack_bf16x2(__uint_as_float(other), __uint_as_float(mine))
                                           : pack_bf16x2(__uint_as_float(mine), __uint_as_float(other));
                    asm volatile("st.shared.u32 [%0], %1;" ::"r"(smem_u32(tp + half + j * NT_EPI_ROW + col)), "r"(w)
                                 : "memory");
                }
                __syncwarp();
                const int t = t_tile + c * 32 + lane;        // row `lane`: one token, 32 features
                if (t < p.M && n_base < p.N) {
                    const uint4* src = reinterpret_cast<const uint4*>(
                        tp + (lane < 16 ? lane * NT_EPI_ROW : NT_EPI_HALF + (lane - 16) * NT_EPI_ROW));
                    uint4* dst = reinterpret_cast<uint4*>(p.y + (int64_t)t * p.ldy + n_base);
                    #pragma unroll
                    for (int i = 0; i < 4; ++i) dst[i] = src[i];
                }
                __syncwarp();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(acc_empty), 0));
            return true;
        };

        // Second-level constants of this thread's NF4 block at position g of the
        // worker's stage sequence (tile unit + (g / nkb) nunits, block g % nkb),
        // fetched one own stage (NT_PAR positions) ahead of their use.
        struct Meta { uint32_t code; float s2; bool ok; };
        auto fetch = [&](int64_t g) -> Meta {
            Meta m{0u, 0.0f, false};
            const int64_t tl = unit + (g / nkb) * nunits;
            const int kb = (int)(g % nkb);
            if (tl >= num_tiles || kb >= p.num_kb) return m;
            const int64_t n = (tl % num_w) * 256 + (int)rank * 128 + rloc;
            const int64_t b = (int64_t)kb * 2 + h;            // block of the row
            if (n < p.N && b < p.kblk) {
                const int64_t bi = n * p.kblk + b;
                m.code = __ldg(p.absmax_q + bi);
                m.s2 = __ldg(p.absmax_s2 + (bi >> 8));
                m.ok = true;
            }
            return m;
        };
        Meta nxt = fetch(par);

        int pending = -1;                                     // tile whose accumulator awaits draining
        int64_t g = 0;                                        // position in the worker's stage sequence
        for (int tile = unit; tile < num_tiles && !bad; tile += nunits) {
            const int64_t n_row = (int64_t)(tile % num_w) * 256 + (int)rank * 128 + rloc;
            for (int kb = 0; kb < nkb; ++kb, ++g) {
                const int stage = (int)(g % NT_STAGES);
                const uint32_t phase = (uint32_t)((g / NT_STAGES) & 1);
                if ((int)(g % NT_PAR) == par) {
                    const Meta cur = nxt;
                    nxt = fetch(g + NT_PAR);
                    const bool got = mbar_wait(&fullP[stage], phase, abort_flag) &&
                                     mbar_wait(&emptyA[stage], phase ^ 1, abort_flag);
                    if (!__all_sync(0xffffffffu, got)) { bad = true; break; }
                    uint32_t v[32];
                    if (kb < p.num_kb) {
                        // this thread's 32 bytes of codes: half h of its row's 64 bytes
                        // (64-byte swizzle: 16-byte chunk c of row r at c ^ ((r >> 1) & 3))
                        const uint8_t* prow = ringP + stage * NT_PBYTES + rloc * 64;
                        uint4 pk[2];
                        #pragma unroll
                        for (int e = 0; e < 2; ++e)
                            pk[e] = *reinterpret_cast<const uint4*>(prow + (((2 * h + e) ^ ((rloc >> 1) & 3)) << 4));
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&emptyP[stage]);
                        if (cur.ok) {
                            const float ah = __fadd_rn(__fmul_rn(dq_s[cur.code], cur.s2), off);
                            uint32_t lo[4], hi[4];
                            nf4_scaled_table(p.level, ah, lo, hi);
                            #pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const uint32_t w4[4] = {pk[e].x, pk[e].y, pk[e].z, pk[e].w};
                                #pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    const uint4 o = nf4x8_to_bf16(w4[i], lo, hi);
                                    v[16 * e + 4 * i + 0] = o.x;
                                    v[16 * e + 4 * i + 1] = o.y;
                                    v[16 * e + 4 * i + 2] = o.z;
                                    v[16 * e + 4 * i + 3] = o.w;
                                }
                            }
                        } else {
                            #pragma unroll
                            for (int i = 0; i < 32; ++i) v[i] = 0u;
                        }
                    } else {
                        // LoRA stage: row n of B_lora (r <= 64 bf16) as the A operand, zeros beyond r
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&emptyP[stage]);
                        #pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = 0u;
                        if (h == 0 && n_row < p.N) {
                            const uint32_t* src = reinterpret_cast<const uint32_t*>(p.lora_b + n_row * p.lora_r);
                            #pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (2 * i < p.lora_r) v[i] = __ldg(src + i);
                        }
                    }
                    tmem_st32(tmem_base + lane_addr + NT_A_COL + (uint32_t)(stage * 64 + h * 32), v);
                    tmem_st_wait(v);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&convDone[stage]);
                }
                if (kb == first_conv - 1 && pending >= 0) {
                    if (!epilogue(pending)) { bad = true; break; }
                    pending = -1;
                }
            }
            if (!bad) pending = tile;
        }
        if (!bad && pending >= 0 && !epilogue(pending)) bad = true;
        if (bad && lane == 0) nt_raise(abort_flag, p.err, 14);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                                       // no CTA leaves while its peer may still use it
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, NT_TMEM_COLS);
    }
}

}  // namespace

bool gemm_nf4t_supported(int64_t M, int64_t N, int64_t Kc) {
    const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
    return tiles >= sm_count() / 2 && Kc % 128 == 0 && N % 64 == 0;
}

lsn_status launch_gemm_nf4t(const uint16_t* x, int64_t ldx, const lsn_nf4_weight* w, const uint16_t* LA,
                            const uint16_t* LB, int r, int64_t M, int64_t N, int64_t Kc, uint16_t* y, int64_t ldy,
                            int* err, cudaStream_t st) {
    if (!gemm_nf4t_supported(M, N, Kc)) return LSN_ERR_UNSUPPORTED;
    if (r > 64) return fail(LSN_ERR_INVALID_ARG, "fused NF4 GEMM: rank above 64");
    CUtensorMap mx, mp, mla;
    lsn_status s;
    if ((s = make_tmap_2d(&mx, x, Kc, M, ldx, 64, 128, false)) != LSN_OK) return s;
    // codes [N, Kc/2] bytes, boxes of 64 bytes (128 weights) x 128 rows
    if ((s = make_tmap_2d(&mp, w->packed, Kc / 2, N, Kc / 2, 64, 128, true)) != LSN_OK) return s;
    if (r > 0) {
        if ((s = make_tmap_2d(&mla, LA, r, M, r, 64, 128, false)) != LSN_OK) return s;
    } else {
        mla = mx;                                     // no LoRA term: never read
    }
    const Nf4Tables& T = nf4_tables();
    Nf4tArgs a{};
    a.M = (int)M;
    a.N = (int)N;
    a.num_kb = (int)(Kc / 128);
    a.lora_k16 = (r + 15) / 16;
    a.kblk = (int)(Kc / 64);
    a.y = y;
    a.ldy = ldy;
    a.err = err;
    a.absmax_q = w->absmax_q;
    a.absmax_s2 = w->absmax_s2;
    a.absmax_off = w->offset;
    a.lora_b = LB;
    a.lora_r = r;
    std::memcpy(a.level, T.level, sizeof(a.level));
    std::memcpy(a.dq, T.dq, sizeof(a.dq));
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(lsn_gemm_nf4t_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        NT_SMEM_BYTES);
    });
    if (attr_err != cudaSuccess) return fail_cuda(attr_err, "cudaFuncSetAttribute(gemm nf4t smem)");
    const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
    const int grid = 2 * gemm_units(tiles, true);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(NT_THREADS);
    cfg.dynamicSmemBytes = NT_SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1 + pdl_attr(&attr[1]);
    LSN_CUDA_TRY(cudaLaunchKernelEx(&cfg, lsn_gemm_nf4t_kernel, mx, mp, mla, a));
    return LSN_OK;
}

}  // namespace lsn
