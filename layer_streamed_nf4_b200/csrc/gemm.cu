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
// Structure (one persistent CTA per SM, 192 threads):
//   warp 0     TMA producer: one elected lane streams 128x64 A tiles and
//              64xBN B tiles (128-byte swizzle) into a 4-stage ring;
//   warp 1     allocates 2*BN TMEM columns; one lane issues tcgen05.mma
//              (M=128, N=BN, K=16) and commits each stage back to the
//              producer and each finished accumulator to the epilogue;
//   warps 2-5  epilogue: tcgen05.ld 32 columns at a time from their TMEM lane
//              quadrant, round to bf16, store; the two accumulator buffers
//              let the epilogue of tile i overlap the main loop of tile i+1.
// Every wait is bounded; a wait that runs out sets *err and the CTA winds
// down (after letting its issued copies and MMAs finish) instead of hanging.
#include <cstring>
#include <mutex>

#include "common.cuh"

namespace lsn {

struct GemmArgs {
    int M, N;            // output rows (tokens) and columns
    int num_kb;          // 64-wide contraction blocks of the base term
    int lora_k16;        // K=16 MMAs of the LoRA term (0: none)
    uint16_t* D;         // bf16 output, row-major
    int64_t ldd;         // elements
    int* err;            // device error flag (set on a timed-out wait)
};

namespace {

constexpr int BM = 128, BK = 64, STAGES = 4;

template <int BN, bool B_MN>
struct Cfg {
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
    static constexpr uint32_t IDESC = idesc_bf16(BM, BN, 0, B_MN ? 1 : 0);
    static constexpr uint32_t TMEM_COLS = 2 * BN;
};

__device__ __forceinline__ void raise_error(volatile int* abort_flag, int* err, int code) {
    *abort_flag = 1;
    if (err) atomicExch(err, code);
}

template <int BN, bool B_MN>
__global__ void __launch_bounds__(192, 1)
    lsn_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmLA, const __grid_constant__ CUtensorMap tmLB,
                    const GemmArgs p) {
    using C = Cfg<BN, B_MN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* acc_full = bars + 2 * STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_m = (p.M + BM - 1) / BM;
    const int num_n = (p.N + BN - 1) / BN;
    const int num_tiles = num_m * num_n;
    const int nkb = p.num_kb + (p.lora_k16 > 0 ? 1 : 0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 128); }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA); tma_prefetch_desc(&tmB);
        if (p.lora_k16 > 0) { tma_prefetch_desc(&tmLA); tma_prefetch_desc(&tmLB); }
    }
    if (warp == 1) { tmem_alloc(tmem_holder, C::TMEM_COLS); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------- producer --
            int stage = 0;
            uint32_t phase = 0;
            int issued_parity[STAGES];
            for (int s = 0; s < STAGES; ++s) issued_parity[s] = -1;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int mb = tile % num_m, nb = tile / num_m;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
                    uint8_t* sA = smem + stage * C::STAGE_BYTES;
                    uint8_t* sB = sA + C::A_BYTES;
                    mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
                    issued_parity[stage] = (int)phase;
                    const bool lora = kb >= p.num_kb;
                    const CUtensorMap* ma = lora ? &tmLA : &tmA;
                    const CUtensorMap* mbp = lora ? &tmLB : &tmB;
                    const int kc = lora ? 0 : kb * BK;
                    tma_load_2d(sA, ma, kc, mb * BM, &full[stage]);
                    if (!B_MN) {
                        tma_load_2d(sB, mbp, kc, nb * BN, &full[stage]);
                    } else {
                        #pragma unroll
                        for (int a = 0; a < BN / 64; ++a)
                            tma_load_2d(sB + a * (64 * 128), mbp, nb * BN + a * 64, kc, &full[stage]);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) raise_error(abort_flag, p.err, 1);
            // Let every copy this CTA issued land before the CTA can exit.
            for (int s = 0; s < STAGES; ++s)
                if (issued_parity[s] >= 0) mbar_wait(&full[s], (uint32_t)issued_parity[s], nullptr);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // -------------------------------------------------- MMA issuer --
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(smem + stage * C::STAGE_BYTES);
                    const uint32_t b0 = a0 + C::A_BYTES;
                    const int nk = (kb < p.num_kb) ? BK / 16 : p.lora_k16;
                    for (int k = 0; k < nk; ++k) {
                        const uint64_t ad = smem_desc_sw128(a0 + k * 32, 16, 1024);
                        const uint64_t bd = B_MN ? smem_desc_sw128(b0 + k * 2048, 64 * 128, 1024)
                                                 : smem_desc_sw128(b0 + k * 32, 16, 1024);
                        umma_bf16(d_tmem, ad, bd, C::IDESC, (kb | k) ? 1u : 0u);
                    }
                    umma_commit(&empty[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                umma_commit(&acc_full[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
            if (!ok) raise_error(abort_flag, p.err, 2);
            // Every MMA issued by this thread completes before TMEM is freed.
            umma_commit(drain);
            mbar_wait(drain, 0, nullptr);
        }
    } else {
        // -------------------------------------------------------- epilogue --
        const int q = warp & 3;                    // TMEM lanes 32q .. 32q+31
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const int mb = tile % num_m, nb = tile / num_m;
            const bool got = mbar_wait(&acc_full[acc], acc_phase, abort_flag);
            if (!__all_sync(0xffffffffu, got)) { if (lane == 0) raise_error(abort_flag, p.err, 3); break; }
            tc_fence_after();
            const int row = mb * BM + q * 32 + lane;
            #pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                const int col = nb * BN + c * 32;
                if (col >= p.N) break;
                uint32_t v[32];
                tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + c * 32), v);
                tmem_ld_wait();
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
            mbar_arrive(&acc_empty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
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
                    int box_inner, int box_outer) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(LSN_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
    cuuint64_t strides[1] = {(cuuint64_t)stride_elems * 2};
    cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(LSN_ERR_CUDA, "cuTensorMapEncodeTiled failed (code " + std::to_string((int)r) + ")");
    return LSN_OK;
}

template <int BN, bool B_MN>
lsn_status launch_cfg(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& la, const CUtensorMap& lb,
                      const GemmArgs& args, cudaStream_t st) {
    using C = Cfg<BN, B_MN>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(lsn_gemm_kernel<BN, B_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        C::SMEM_BYTES);
    });
    if (attr_err != cudaSuccess) return fail_cuda(attr_err, "cudaFuncSetAttribute(gemm smem)");
    const int tiles = ((args.M + BM - 1) / BM) * ((args.N + BN - 1) / BN);
    const int grid = tiles < sm_count() ? tiles : sm_count();
    lsn_gemm_kernel<BN, B_MN><<<grid, 192, C::SMEM_BYTES, st>>>(a, b, la, lb, args);
    LSN_CUDA_TRY(cudaGetLastError());
    return LSN_OK;
}

}  // namespace

// N-tile width from the shape alone: 256 unless that leaves SMs idle.
int gemm_bn(int64_t M, int64_t N) {
    const int64_t tiles256 = ((M + BM - 1) / BM) * ((N + 255) / 256);
    return (tiles256 >= 148) ? 256 : 128;
}

// D = A . op(B) + LA . op(LB).
//   A  [M, Kc] bf16 row-major (lda), K-major.
//   b_mn == false: B is [N, Kc] (ldb), LB is [N, r]   (forward: W, B_lora)
//   b_mn == true : B is [Kc, N] (ldb), LB is [r, N]   (backward: W, A_lora)
//   LA [M, r] (bf16(s u) or bf16(s g)); r == 0 disables the LoRA term.
lsn_status launch_gemm(const uint16_t* A, int64_t lda, const uint16_t* B, int64_t ldb, bool b_mn, const uint16_t* LA,
                       const uint16_t* LB, int r, int64_t M, int64_t N, int64_t Kc, uint16_t* D, int64_t ldd,
                       int* err, cudaStream_t st) {
    const int bn = gemm_bn(M, N);
    CUtensorMap ma, mb, mla, mlb;
    lsn_status s;
    if ((s = make_map(&ma, A, Kc, M, lda, 64, BM)) != LSN_OK) return s;
    if (!b_mn) {
        if ((s = make_map(&mb, B, Kc, N, ldb, 64, bn)) != LSN_OK) return s;
    } else {
        if ((s = make_map(&mb, B, N, Kc, ldb, 64, 64)) != LSN_OK) return s;
    }
    if (r > 0) {
        if ((s = make_map(&mla, LA, r, M, r, 64, BM)) != LSN_OK) return s;
        if (!b_mn) {
            if ((s = make_map(&mlb, LB, r, N, r, 64, bn)) != LSN_OK) return s;
        } else {
            if ((s = make_map(&mlb, LB, N, r, N, 64, 64)) != LSN_OK) return s;
        }
    } else {
        mla = ma;
        mlb = mb;
    }
    GemmArgs args;
    args.M = (int)M;
    args.N = (int)N;
    args.num_kb = (int)(Kc / BK);
    args.lora_k16 = (r + 15) / 16;
    args.D = D;
    args.ldd = ldd;
    args.err = err;
    if (bn == 256) return b_mn ? launch_cfg<256, true>(ma, mb, mla, mlb, args, st)
                               : launch_cfg<256, false>(ma, mb, mla, mlb, args, st);
    return b_mn ? launch_cfg<128, true>(ma, mb, mla, mlb, args, st)
                : launch_cfg<128, false>(ma, mb, mla, mlb, args, st);
}

}  // namespace lsn
