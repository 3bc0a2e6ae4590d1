/*
 * lsnf4.h -- C ABI of liblsnf4.so: layer-streamed NF4 LoRA linears on B200 (sm_100a).
 *
 * The method ("Exact Layer Streaming: LoRA Fine-Tuning of an 8B Model on a 4 GB
 * Laptop GPU", abstract) keeps a frozen base model -- NF4 or bf16 -- in host
 * RAM, streams its decoder layers through a small pool of pre-allocated VRAM
 * buffers on a separate copy stream, and trains LoRA adapters on top.  This
 * library is its per-layer hot path:
 *
 *   nf4_quantize / nf4_dequant  the 4-bit base format and its double-quantised
 *                               constants ("Can You Fine-Tune a 27B Model on a
 *                               Laptop? (I Did the Math)", 2:19-2:29);
 *   lora_linear_fwd / _bwd      y = x W^T + s (x A^T) B^T and its gradients
 *                               for x, A, B (same video, 1:36-1:58);
 *   layer_pool_*                the VRAM layer pool fed from pinned host RAM,
 *                               prefetching the next layer on a side stream
 *                               (same video, 7:11-7:42; the sourcefeed article
 *                               "An 8B Fine-Tune Now Fits in 4 GB of VRAM",
 *                               section "The trick is that frozen weights are
 *                               just data").
 *
 * Conventions (all entry points):
 *  - Every call returns an lsn_status.  Argument errors are detected before
 *    anything is enqueued; lsn_last_error() then holds a message.  CUDA
 *    launch errors are reported as LSN_ERR_CUDA by the call that launched;
 *    asynchronous faults surface at the caller's next synchronisation.
 *  - Compute calls are asynchronous on the stream passed in; no call
 *    synchronises the device unless its comment says so.
 *  - All tensor pointers are DEVICE pointers owned by the caller, row-major and
 *    contiguous, unless stated otherwise.  bf16 tensors are passed as uint16_t
 *    bit patterns.  Pointers passed to a compute call must stay valid until
 *    the work enqueued on the stream has finished.
 *  - Every tensor pointer must be 16-byte aligned (the tensor-memory-access
 *    unit reads rows in 16-byte units).
 *  - Results are deterministic: the same inputs and shapes give the same bits,
 *    independent of pointers, streams or what ran before.
 */
#ifndef LSNF4_H
#define LSNF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle (cudaStream_t); NULL means the legacy default stream. */
typedef struct CUstream_st* lsn_stream_t;

typedef enum {
    LSN_OK = 0,
    LSN_ERR_INVALID_ARG = 1, /* bad shape, null or misaligned pointer, unpinned host memory */
    LSN_ERR_CUDA = 2,        /* a CUDA runtime/driver call failed */
    LSN_ERR_NO_MEMORY = 3,   /* device or host allocation failed */
    LSN_ERR_TIMEOUT = 4,     /* a bounded wait ran out */
    LSN_ERR_UNSUPPORTED = 5, /* no sm_100 device, or a shape outside the supported set */
    LSN_ERR_STATE = 6        /* call out of order (e.g. pool has no free slot) */
} lsn_status;

/* Thread-local message describing the last failure of this thread; never NULL. */
const char* lsn_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
int lsn_version(void);

/* ------------------------------------------------------------- NF4 codec --
 *
 * Format (the pages name NF4 and a second quantisation pass over its
 * constants but print neither; this follows QLoRA's construction, the paper
 * the sourcefeed article links):
 *  - levels: 16 fp32 values, index 0 = -1, index 7 = 0, index 15 = +1; the
 *    normalised N(0,1) quantiles of 7 negative and 8 positive equal steps up to
 *    p_max = 1 - (1/32 + 1/30)/2;
 *  - first level: blocks of 64 consecutive elements of the row-major weight
 *    (cols % 64 == 0, so a block never crosses a row); code = nearest level
 *    of w / absmax (smallest exact distance, lower index on a tie), computed in
 *    fp32; an all-zero block codes to index 7;
 *  - packing: byte j = (code[2j] << 4) | code[2j+1];
 *  - second level: offset = mean of all block absmax values (fp64 sums:
 *    sequential within each group of 256 blocks, then over groups in order;
 *    divided by the block count, rounded to fp32); per group of 256 blocks,
 *    s2 = max |fp32(absmax - offset)| and each block stores the 8-bit index of
 *    the nearest entry of the table k/127 (k = -127..127 at index k+127) to
 *    fp32((absmax - offset) / s2); s2 == 0 stores index 127;
 *  - dequantisation: absmax_hat = fp32(fp32(table[code8] * s2) + offset),
 *    w = bf16_rne(fp32(level[code4] * absmax_hat)), no fused multiply-add.
 */

/* Copies the 16 fp32 NF4 levels into out[16] (host memory). */
void lsn_nf4_codebook(float out[16]);
/* Copies the 256-entry fp32 second-level table into out[256] (host memory). */
void lsn_dq_codebook(float out[256]);

/* A quantised weight of rows x cols (N x K), cols % 64 == 0.  All pointers are
 * caller-owned device memory:
 *   packed     [rows*cols/2]      uint8, two 4-bit codes per byte (16-byte aligned)
 *   absmax_q   [rows*cols/64]     uint8 second-level codes
 *   absmax_s2  [ceil(nblk/256)]   fp32 per group of 256 blocks (4-byte aligned)
 *   offset     [1]                fp32 (device, so quantisation never syncs; 4-byte aligned)
 * The four arrays are independent: they may sit in one blob
 * (lsn_nf4_blob_layout) or apart, e.g. the codes in a layer-pool slot and the
 * constants in memory that stays resident. */
typedef struct {
    int64_t rows, cols;
    uint8_t* packed;
    uint8_t* absmax_q;
    float* absmax_s2;
    float* offset;
} lsn_nf4_weight;

/* Byte sizes of the four arrays of an rows x cols NF4 weight. */
size_t lsn_nf4_packed_bytes(int64_t rows, int64_t cols);
size_t lsn_nf4_absmax_bytes(int64_t rows, int64_t cols);
size_t lsn_nf4_s2_bytes(int64_t rows, int64_t cols);
/* Total bytes of the four arrays when each starts on a 1 KiB boundary (the
 * layout used for a layer blob, see lsn_nf4_blob_layout). */
size_t lsn_nf4_blob_bytes(int64_t rows, int64_t cols);
/* Offsets of packed, absmax_q, absmax_s2 and offset inside such a blob
 * (out[4], bytes from the blob start, each a multiple of 1024). */
void lsn_nf4_blob_layout(int64_t rows, int64_t cols, size_t out[4]);

/* Workspace bytes nf4_quantize needs for an rows x cols weight. */
size_t lsn_nf4_quantize_ws_bytes(int64_t rows, int64_t cols);

/* Quantise an fp32 weight W [rows, cols] (device) into *out.
 * ws: device scratch of at least lsn_nf4_quantize_ws_bytes(rows, cols).
 * Bit-exact with the format above.  A non-finite input element makes the
 * result undefined (the host does not scan W); rows*cols == 0 is a no-op. */
lsn_status nf4_quantize(const float* W, const lsn_nf4_weight* out, void* ws, size_t ws_bytes,
                        lsn_stream_t stream);

/* Largest rows*cols nf4_quantize_noalloc accepts (2^26 elements). */
#define LSN_NF4_NOALLOC_MAX_ELEMS 67108864LL

/* nf4_quantize without a caller workspace and without allocating anything.
 * (The pages have no counterpart: this exists for callers of the library.)
 *
 * For callers that cannot provide device memory when they quantise -- a host
 * whose allocator has reserved all device memory up front, a loop that must
 * not pay for cudaMalloc's implicit synchronisation, a plug-in without an
 * allocator.  The scratch it needs lives in a fixed array inside this
 * library's device image: 4 MiB + 32 KiB per device, present on every device
 * that loads the library until the process exits.  Limit: rows*cols <=
 * LSN_NF4_NOALLOC_MAX_ELEMS; larger weights are rejected with
 * LSN_ERR_INVALID_ARG before anything is enqueued.  Results are bit-identical
 * to nf4_quantize.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current) and keeps it for the life of the process;
 * make that first call before any stream capture.  A device reset
 * (cudaDeviceReset) after that first call is not supported: the kept address
 * would no longer name the array.  All calls share the one array: calls whose work overlaps on the
 * GPU (different streams without ordering between them) race and corrupt
 * each other's results -- order them on one stream or with events.  It calls
 * no cudaMalloc, cudaFree or allocating library routine. */
lsn_status nf4_quantize_noalloc(const float* W, const lsn_nf4_weight* out, lsn_stream_t stream);

/* Dequantise *w into bf16 W_out [rows, cols] (device).  HBM-bound. */
lsn_status nf4_dequant(const lsn_nf4_weight* w, uint16_t* W_out, lsn_stream_t stream);

/* Dequantise n weights with one launch (e.g. the projections of a layer):
 * w is a HOST array of n weights, W_out a HOST array of n device pointers
 * (bf16 [rows_i, cols_i] each, 16-byte aligned, not overlapping), both read
 * during the call only.  Same bits as n nf4_dequant calls.  Any n >= 0; more
 * than 16 weights take several launches.  blocks_per_sm: 0 = as many blocks
 * as the work has (fastest on an idle GPU); k > 0 = at most k blocks per SM,
 * looping over the work, for a dequantisation that runs beside other
 * kernels (e.g. the next layer's weights under the current layer's GEMMs). */
lsn_status nf4_dequant_batch(int n, const lsn_nf4_weight* w, uint16_t* const* W_out, int blocks_per_sm,
                             lsn_stream_t stream);

/* ------------------------------------------------------------ LoRA linear --
 *
 * y  = x W^T + s (x A^T) B^T                        (forward)
 * dX = dY W + s (dY B) A                            (input gradient)
 * dA = s (dY B)^T x,   dB = s dY^T (x A^T)          (adapter gradients, fp32)
 * x [T,K], W [N,K] (rows = N out features, cols = K in features), A [r,K],
 * B [N,r], y and dY [T,N], dX [T,K], dA [r,K], dB [N,r]; s = scale
 * (alpha / r).  The base W is frozen: there is no gradient for it.
 *
 * Shapes supported: K % 64 == 0, N % 64 == 0, 1 <= r <= 64 with r % 8 == 0,
 * T >= 0 (T == 0 is a no-op; any T, including a ragged last tile).
 * Precision: bf16 operands, fp32 accumulation in tensor memory; s*(x A^T) and
 * s*(dY B) enter the tensor-core contraction rounded to bf16; y and dX are
 * written as bf16; dA and dB are accumulated in fp32 in a fixed order.
 */
typedef enum { LSN_BASE_NF4 = 0, LSN_BASE_BF16 = 1 } lsn_base_kind;

typedef struct {
    int kind;            /* lsn_base_kind */
    int64_t rows, cols;  /* N, K */
    lsn_nf4_weight nf4;  /* used when kind == LSN_BASE_NF4 (its rows/cols must match) */
    const uint16_t* bf16;/* used when kind == LSN_BASE_BF16: bf16 W [rows, cols] */
} lsn_base;

/* Workspace bytes lora_linear_fwd / lora_linear_bwd need (the larger of the two).
 * The workspace starts with the kernels' status word, which must start at
 * zero: fill a new workspace with zeros once (lsn_ws_status clears it after
 * reporting a timeout). */
size_t lsn_lora_ws_bytes(int64_t T, int64_t K, int64_t N, int r, int kind);

/* Forward.  y may not alias x.  ws: device scratch of lsn_lora_ws_bytes bytes,
 * not touched by anyone else until the enqueued work finishes. */
lsn_status lora_linear_fwd(const lsn_base* W, const uint16_t* x, int64_t T, const uint16_t* A,
                           const uint16_t* B, int r, float scale, uint16_t* y, void* ws,
                           size_t ws_bytes, lsn_stream_t stream);

/* Backward.  dX may be NULL (input gradient not wanted).  accumulate != 0 adds
 * into dA and dB (gradient accumulation), otherwise they are overwritten. */
lsn_status lora_linear_bwd(const lsn_base* W, const uint16_t* x, const uint16_t* dY, int64_t T,
                           const uint16_t* A, const uint16_t* B, int r, float scale, uint16_t* dX,
                           float* dA, float* dB, int accumulate, void* ws, size_t ws_bytes,
                           lsn_stream_t stream);

/* ------------------------------------------------------- whole layer ---
 *
 * The LoRA linears of one decoder layer (q, k, v, o, gate, up, down, or any
 * n <= LSN_LAYER_MAX_PROJ) in one call, in the order the layer loop meets
 * them while the layer sits in its pool slot ("Can You Fine-Tune a 27B Model
 * on a Laptop? (I Did the Math)", 7:11-7:42).  Every projection's outputs are
 * bit for bit those of lora_linear_fwd / lora_linear_bwd on the same inputs;
 * only the launches differ: the NF4 dequantisation of all projections is one
 * kernel, their rank-r down projections one kernel, their dA/dB token
 * reductions one kernel, and (LSN_OPT_LAYER_MERGE, bf16 bases, no groups)
 * the GEMMs of projections 1..n-1 one launch after projection 0's own.  The
 * projections are independent of each other within a call (each reads only
 * its own x or dY): a caller whose projections depend on each other (o on
 * attention over q, k, v) makes one call per independent set.  The forward can keep u = x A^T, the low-rank
 * activation a LoRA layer saves for its backward pass, so the backward does
 * not read x again to rebuild it.  A projection whose A and B are NULL runs
 * with the adapter off: the streamed base alone, the reference model of
 * preference training ("An 8B Fine-Tune Now Fits in 4 GB of VRAM": the
 * streamed base with the adapters switched off is the reference); its
 * output is bit for bit the base term of the adapter-on call.
 *
 * Groups.  Projections that read the same input (q, k, v of attention; gate
 * and up of the MLP) can be marked as a group: consecutive entries with the
 * same positive `group`, at most 4, sharing the x pointer, K, base kind and
 * adapter state, with group size x r <= 64; bf16 bases of a group must lie
 * back to back in memory (as in a layer blob).  The forward computes the
 * group as one GEMM over the stacked weights (outputs routed to each y; the
 * same bits as ungrouped).  The backward computes the group's input gradient
 * sum_j (dY_j W_j + s (dY_j B_j) A_j) as one GEMM and writes it to the first
 * member's dX (the other members' dX must be NULL); dA and dB are per member
 * and the same bits as ungrouped.
 *
 * p is a HOST array of n descriptors, read during the call only; the
 * pointers inside are device pointers that must stay valid until the
 * enqueued work has finished.  Projections may have different K and N but
 * share T, r and scale.  The outputs of different projections may not
 * overlap each other or any input.
 */
#define LSN_LAYER_MAX_PROJ 16

typedef struct {
    lsn_base W;          /* frozen base [N, K] */
    const uint16_t* x;   /* [T, K] input */
    const uint16_t* A;   /* [r, K]; A and B both NULL: the adapter is off for this projection */
    const uint16_t* B;   /* [N, r]   (the frozen base alone: y = x W^T, dX = dY W; dA, dB, u unused) */
    uint16_t* y;         /* forward: output [T, N]; unused by the backward */
    const uint16_t* dY;  /* backward: output gradient [T, N]; unused by the forward */
    uint16_t* dX;        /* backward: input gradient [T, K], or NULL */
    float* dA;           /* backward: [r, K] fp32 */
    float* dB;           /* backward: [N, r] fp32 */
    float* u;            /* fp32 [T, r] = x A^T, or NULL.  Forward: written when non-NULL.
                            Backward: read when non-NULL (it must hold what the forward
                            wrote for the same x and A), recomputed when NULL. */
    int group;           /* 0, or a group id: consecutive projections with the same positive id
                            form a group (see below) */
} lsn_lora_proj;

/* Workspace bytes of lora_layer_fwd / lora_layer_bwd for these projections
 * (the larger of the two; 0 when an argument is invalid).  Like the
 * single-linear workspace it must be zero-filled once when allocated.  With
 * NF4 bases it holds the dequantised bf16 copy of every projection. */
size_t lsn_layer_ws_bytes(int n, const lsn_lora_proj* p, int64_t T, int r);

/* Forward of n projections: y_i = x_i W_i^T + s (x_i A_i^T) B_i^T. */
lsn_status lora_layer_fwd(int n, const lsn_lora_proj* p, int64_t T, int r, float scale, void* ws,
                          size_t ws_bytes, lsn_stream_t stream);

/* Backward of n projections: dX_i, dA_i, dB_i as lora_linear_bwd. */
lsn_status lora_layer_bwd(int n, const lsn_lora_proj* p, int64_t T, int r, float scale, int accumulate,
                          void* ws, size_t ws_bytes, lsn_stream_t stream);

/* Synchronise `stream`, then read the status word at the start of a LoRA
 * workspace: LSN_ERR_TIMEOUT if a tensor-core kernel gave up on a bounded
 * wait since the last check (the word is then cleared), LSN_OK otherwise.
 * The workspace must have been zero-filled once when it was allocated. */
lsn_status lsn_ws_status(void* ws, lsn_stream_t stream);

/* Self-test of the bounded wait the tensor-core kernels use: one thread waits
 * on an mbarrier that nothing arrives on, giving up after about limit_us
 * microseconds (1 .. 1e6) of SM clock.  Synchronises `stream`.  Returns
 * LSN_ERR_TIMEOUT when the wait gave up as designed (the expected outcome;
 * the context stays usable), LSN_ERR_STATE if it did not. */
lsn_status lsn_selftest_wait_timeout(int limit_us, lsn_stream_t stream);

/* ------------------------------------------------------- kernel timing --
 *
 * Optional per-launch timing of the library's own kernels: while enabled,
 * every launch is bracketed by two CUDA events on the stream it runs on, and
 * lsn_timing_read sums the event-measured device time per kernel kind with
 * the algorithmic work of each launch (flops for the GEMMs, bytes for the
 * memory-bound kernels).  Recording adds two event records per launch.
 */
typedef enum {
    LSN_K_GEMM_FWD = 0,   /* y = x W^T + s u B^T                 (flop) */
    LSN_K_GEMM_BWD = 1,   /* dX = dY W + s g A                   (flop) */
    LSN_K_DEQUANT = 2,    /* NF4 -> bf16                         (bytes) */
    LSN_K_LORA_DOWN = 3,  /* u = x A^T, g = dY B                 (bytes) */
    LSN_K_LORA_TGRAD = 4, /* dA, dB token reductions             (bytes) */
    LSN_K_QUANTIZE = 5,   /* fp32 -> NF4                         (bytes) */
    LSN_K_COUNT = 6
} lsn_kernel_kind;

typedef struct {
    uint64_t launches[LSN_K_COUNT];  /* timed launch groups (one per library call site) */
    uint64_t kernels[LSN_K_COUNT];   /* CUDA kernels inside those groups */
    double ms[LSN_K_COUNT];          /* summed device time */
    double work[LSN_K_COUNT];        /* summed algorithmic flop or bytes */
} lsn_kernel_timing;

/* Start (on != 0, clearing previous records) or stop recording.  At most
 * 65536 launches are kept; later ones are counted but not timed. */
lsn_status lsn_timing_enable(int on);
/* Wait for the recorded events, return the sums and clear the records. */
lsn_status lsn_timing_read(lsn_kernel_timing* out);

/* ------------------------------------------------------------- options --
 *
 * Process-wide switches between equivalent implementations.  Every setting
 * is deterministic: a given shape always gives the same bits.  LSN_OPT_STREAM_K
 * changes the last bits of some outputs (it decides where fp32 partial sums
 * meet); the other switches change only speed.
 *   LSN_OPT_FUSED_NF4  1: NF4 weights on the 2-SM GEMM are converted to bf16
 *                      inside the GEMM by converter warps (no bf16 copy of W;
 *                      whole tiles only: its bits equal the unfused path's
 *                      with LSN_OPT_STREAM_K 0);
 *                      0 (default): nf4_dequant into the workspace, then the
 *                      bf16 GEMM.  Narrow shapes always use the latter.
 *   LSN_OPT_STREAM_K   1: when a GEMM's output tiles do not fill whole
 *                      waves of the SMs, its contraction blocks are shared out
 *                      evenly over the SMs (stream-K): a tile cut between two
 *                      SMs is summed in two fp32 pieces that meet in the
 *                      workspace (in a fixed way, whatever the timing).
 *                      0 (default): whole tiles, round robin (the last wave
 *                      partly idle; measured faster on the 8B shapes).
 *   LSN_OPT_LAYER_LANES 2 (default): lora_layer_fwd / _bwd spread the work
 *                      of different projections that does not depend on each
 *                      other (their GEMMs; the backward's token reductions)
 *                      over the caller's stream and a library-owned second
 *                      stream of the same device, which forks from the
 *                      caller's stream and joins it again within the call;
 *                      1: everything on the caller's stream.
 *   LSN_OPT_PDL        1 (default): the hot-path kernels are launched with
 *                      programmatic dependent launch, so each kernel's set-up
 *                      (barriers, tensor memory, tensor-map prefetch) overlaps
 *                      the tail of the kernel before it on the same stream;
 *                      every kernel still waits for its predecessor to finish
 *                      before it reads or writes global memory.  0: ordinary
 *                      stream-ordered launches.
 *   LSN_OPT_GEMM_MIN_UNITS 1: a GEMM whose tiles take R rounds over all the
 *                      SMs runs on the fewest SMs that still finish in R
 *                      rounds (e.g. 128 tiles of 256 x 256: 64 SM pairs
 *                      instead of 74), leaving the rest free for work on other
 *                      streams; 0 (default): one CTA (pair) per SM.
 *   LSN_OPT_GEMM_TAIL_SPLIT 1: on the 2-SM GEMM, the output tiles of a last,
 *                      partly filled round are cut along N into quanta of 64
 *                      columns (128 for the backward's MN-major W) and shared
 *                      out evenly, so every SM pair gets about the same number
 *                      of columns; each output element is still summed over
 *                      the whole contraction by one SM pair, so the bits do
 *                      not change.  0 (default): whole tiles round robin.
 *   LSN_OPT_LAYER_MERGE 1 (default): in lora_layer_fwd / _bwd calls whose
 *                      bases are all bf16, the GEMMs run as one persistent
 *                      launch: whole 256 x 256 tiles of all of them, shared
 *                      out over the SM pairs by a schedule that balances the
 *                      pairs' summed contraction lengths, so the last round of
 *                      one projection's tiles no longer leaves SMs idle.
 *                      Without groups, projection 0's GEMM runs first on its
 *                      own (only its down projection then precedes a GEMM)
 *                      and projections 1..n-1 are merged; with groups (or the
 *                      adapter off on projection 0) every GEMM of the call is
 *                      merged, a group's backward as one problem over its
 *                      members' dY.  Up to 8 problems and 5120 tiles (beyond,
 *                      one launch each); none with LSN_OPT_STREAM_K 1.  Same
 *                      bits (each tile is computed as in its own launch).
 *                      0: one launch per projection or group.
 *   LSN_OPT_DEQUANT_SPARE_SMS 0 (default); n > 0: nf4_dequant_batch calls with
 *                      blocks_per_sm = k > 0 launch n * k blocks, each
 *                      reserving enough shared memory that it never shares an
 *                      SM with a GEMM CTA: a dequantisation beside GEMMs that
 *                      leave n SMs free runs on those SMs only.
 */
typedef enum {
    LSN_OPT_FUSED_NF4 = 1,
    LSN_OPT_LAYER_LANES = 2,
    LSN_OPT_PDL = 3,
    LSN_OPT_STREAM_K = 4,
    LSN_OPT_GEMM_MIN_UNITS = 5,
    LSN_OPT_DEQUANT_SPARE_SMS = 6,
    LSN_OPT_GEMM_TAIL_SPLIT = 7,
    LSN_OPT_LAYER_MERGE = 8
} lsn_option;
lsn_status lsn_set_option(int option, int value);
int lsn_get_option(int option);

/* The tile schedule of the merged GEMM launch (LSN_OPT_LAYER_MERGE), computed
 * on the host from the shapes alone (no device is touched): n problems of
 * ntiles[i] whole tiles costing cost[i] contraction blocks each, numbered
 * problem after problem, shared out over `units` workers (SM pairs): tiles in
 * decreasing cost (problem order among equal costs), each to the worker with
 * the least summed cost so far (the lowest index on ties).  Worker u takes
 * tile[start[u] .. start[u+1]).  start holds units + 1 entries (host memory),
 * tile max_tiles; LSN_ERR_INVALID_ARG when the tiles do not fit or an argument
 * is out of range.  Exposed for inspection and tests; the launch computes the
 * same schedule itself. */
lsn_status lsn_gemm_merged_schedule(int units, int n, const int* ntiles, const int* cost, int* start, int* tile,
                                    int max_tiles);

/* ------------------------------------------------------------ layer pool --
 *
 * n_slots VRAM buffers of slot_bytes each, allocated once at creation; the
 * pool copies registered host blobs (one per layer) into slots on its own copy
 * stream and orders copy and compute with events:
 *   ready[slot]     recorded on the copy stream after a layer's copy;
 *   released        one event per layer_pool_release, recorded on the
 *                   releasing stream.
 * A copy into a slot waits for every release event of that slot recorded
 * since its last fill, so a slot is never overwritten while any holder's
 * compute may still read it (a layer acquired on two streams stays intact
 * until both have released it, whichever releases first).  Forward sweeps prefetch
 * layer i+1 while layer i computes, backward sweeps layer i-1; with 2 slots a
 * fwd+bwd step reads 2L-4 layers in steady state (each layer twice, minus the
 * two still resident at each turn).  With S slots a sweep can keep S layers
 * in flight: prefetch the next S layers of the sweep at its start and one
 * more each time a layer is released; at each turn the S layers used last are
 * the S used first, so a step reads 2L-2S layers.
 */
typedef struct lsn_pool lsn_pool;

typedef struct {
    uint64_t copies;          /* host-to-device layer copies enqueued */
    uint64_t bytes_copied;    /* their bytes */
    uint64_t hits;            /* acquire/prefetch found the layer already resident */
    uint64_t misses;          /* acquire had to start the copy itself */
    double copy_ms;           /* summed device time of completed copies (events) */
} lsn_pool_stats;

/* Create a pool on `device` (the device is made current for the calls).
 * Slots are 1 KiB aligned.  Fails with LSN_ERR_NO_MEMORY if the slots do not fit. */
lsn_status layer_pool_create(int n_slots, size_t slot_bytes, int device, lsn_pool** out);

/* Register the host blob of `layer` (0 <= layer < 65536).  host_pinned must be
 * page-locked (cudaHostAlloc / cudaHostRegister) -- pageable memory is
 * rejected -- and stay alive and unchanged until layer_pool_destroy;
 * bytes <= slot_bytes.  Re-registering a layer replaces its blob and drops
 * any resident copy. */
lsn_status layer_pool_register(lsn_pool* pool, int layer, const void* host_pinned, size_t bytes);

/* Start copying `layer` into a free slot.  Takes the least recently released
 * slot that is neither acquired nor holding a prefetched, not yet acquired
 * layer; LSN_ERR_STATE if there is none.  If `layer` is resident or in flight
 * nothing is copied, and a resident layer that is not acquired counts as
 * prefetched again: its slot is not taken for another layer until it has been
 * acquired. */
lsn_status layer_pool_prefetch(lsn_pool* pool, int layer);

/* Make `compute` wait until `layer` is in VRAM (copying it first if needed)
 * and return its slot address in *dev_ptr.  The slot stays valid for kernels
 * enqueued on `compute` until layer_pool_release. */
lsn_status layer_pool_acquire(lsn_pool* pool, int layer, lsn_stream_t compute, void** dev_ptr);

/* Record a release event of the layer's slot on `compute`: this holder's
 * claim ends once the work enqueued on `compute` before this call has
 * finished; the slot may be reused when every holder's claim has ended. */
lsn_status layer_pool_release(lsn_pool* pool, int layer, lsn_stream_t compute);

/* Host-side bounded wait for every enqueued copy; LSN_ERR_TIMEOUT after
 * timeout_ms milliseconds (the copies keep running). */
lsn_status layer_pool_wait_idle(lsn_pool* pool, int timeout_ms);

/* Counters since creation or the last reset. */
lsn_status layer_pool_stats(lsn_pool* pool, lsn_pool_stats* out);

/* Forget which layers are resident (slots are refilled on the next acquire)
 * and zero the counters.  Waits for the pool's copies first (bounded, 10 s). */
lsn_status layer_pool_reset(lsn_pool* pool);

/* Test hooks that plant host-side faults (no GPU fault is ever produced):
 *   LSN_POOL_FAULT_NONE         normal operation;
 *   LSN_POOL_FAULT_STALE_SLOT   a copy into a slot that already held a layer
 *                               is skipped: the slot is relabelled but keeps
 *                               the previous layer's bytes -- the aliasing
 *                               defect the bit-exactness gate must catch
 *                               ("Exact Layer Streaming", abstract);
 *   LSN_POOL_FAULT_COPY_ERROR   the next copy fails with LSN_ERR_CUDA before
 *                               anything is enqueued. */
typedef enum {
    LSN_POOL_FAULT_NONE = 0,
    LSN_POOL_FAULT_STALE_SLOT = 1,
    LSN_POOL_FAULT_COPY_ERROR = 2
} lsn_pool_fault;
lsn_status layer_pool_inject_fault(lsn_pool* pool, int fault);

/* Debugging aids (flags, 0 = none):
 *   LSN_POOL_DEBUG_POISON  before every copy the slot is filled with 0xFF
 *                          bytes (on the copy stream, after the slot's
 *                          released event), so a read of a slot outside its
 *                          acquire..release window sees the sentinel instead
 *                          of plausible weights: NF4 codes of all 15s, bf16
 *                          NaNs.  Costs one device-side fill per copy.
 * LSN_ERR_INVALID_ARG for a NULL pool or unknown flag bits. */
typedef enum { LSN_POOL_DEBUG_POISON = 1 } lsn_pool_debug_flag;
lsn_status layer_pool_set_debug(lsn_pool* pool, int flags);

/* Free the slots, events and the copy stream (waits for pending copies). */
void layer_pool_destroy(lsn_pool* pool);

#ifdef __cplusplus
}
#endif
#endif /* LSNF4_H */
