/*
 * spear.h -- C ABI of the B200 (sm_100a) W4 linear layer with a per-token-gated
 * low-rank error compensator (EC).
 *
 * Source: "SPEAR: A System for Post-Quantization Error-Adaptive Recovery
 * Enabling Efficient Low-Bit LLM Serving".  The technical summary, section 2.1A
 * (input-adaptive error compensators), defines the effective weight
 * W + alpha * B diag(gamma(Ax)) A.  Section 3.1 quantises per output channel with
 * RTN to 4 bits.  Section 2.2A (phase-adaptive fused kernel dispatch) fuses the
 * EC into the low-bit GEMM's epilogue at decode and runs it as a separate
 * kernel at prefill.  The abstract names the per-token gates.  This library
 * computes, for every token row m of x:
 *
 *   y[m,n] = s[n] * sum_k x[m,k] (q[n,k] - z[n])  +  g[m] * sum_j t[m,j] B[j,n]
 *   t[m,j] = sum_k x[m,k] A[k,j]
 *   g[m]   = 1 / (1 + exp(-(sum_k x[m,k] w_g[k] + b_g)))
 *
 * with alpha = 1, gamma a scalar sigmoid gate, A stored [K, r], B stored [r, N].
 *
 * Conventions shared by every call:
 *   - Pointers marked "device" are CUDA device pointers that the caller
 *     allocates and owns.  The library keeps no pointer after a call returns.
 *     Apart from the one-time tensor-map and attribute set-up noted below, it
 *     allocates no device memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Every device call is asynchronous on that stream.
 *   - Argument errors are detected on the host, before anything is launched.
 *     A CUDA launch or runtime error returns SPEAR_ERR_CUDA.
 *   - Row-major layouts throughout.  bf16 = IEEE bfloat16 and fp16 = IEEE
 *     binary16, both stored as 16-bit patterns.
 *   - All device pointers must be 16-byte aligned (SPEAR_ERR_MISALIGNED).
 */
#ifndef SPEAR_H
#define SPEAR_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SPEAR_API __attribute__((visibility("default")))
#else
#define SPEAR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SPEAR_OK = 0,
    SPEAR_ERR_INVALID_ARG = 1,        /* NULL pointer, bad enum, negative size, ... */
    SPEAR_ERR_UNSUPPORTED_SHAPE = 2,  /* N % 128, K % 64, rank outside 16..256 or not % 16, K > 65536 with EC */
    SPEAR_ERR_MISALIGNED = 3,         /* a device pointer is not 16-byte aligned */
    SPEAR_ERR_WORKSPACE_TOO_SMALL = 4,
    SPEAR_ERR_CUDA = 5,               /* CUDA runtime / launch failure */
    SPEAR_ERR_TIMEOUT = 6             /* a bounded in-kernel wait gave up (see spear_get_device_status) */
} spear_status;

typedef enum { SPEAR_BF16 = 0, SPEAR_FP32 = 1 } spear_dtype;

/* Kernel families the dispatcher chooses from (section 2.2A's two phases). */
typedef enum {
    SPEAR_KERNEL_AUTO = 0,      /* let spear_gemm_plan decide */
    SPEAR_KERNEL_SPLITK = 1,    /* decode: split-K weight-streaming kernel (mma.sync on registers); EC
                                   CTAs of the same launch reduce x A through int64 accumulators */
    SPEAR_KERNEL_TC05 = 2,      /* prefill: TMA + tcgen05/TMEM kernel, EC applied in its epilogue.
                                   tile_n = 128 weight rows (or 256 with tile_m = 128), tile_m = 128,
                                   160, 192 or 256 tokens.  split_k = 1, or 2, 4 or 8 with 128 weight
                                   rows, tile_m 128 or 256 and (K / 64) divisible by it: the tile's K
                                   range is split over a thread-block cluster of split_k CTAs whose
                                   partial tiles are summed in shared memory in rank order (for small
                                   grids with long K); not with SPEAR_PLAN_SEPARATE_EC. */
    SPEAR_KERNEL_STREAM = 3,    /* decode and small batches (M <= 64): persistent stream-K TMA + tcgen05
                                   kernel; every SM streams an equal share of the weight tiles' K chunks,
                                   partial tiles meet through the workspace in a fixed order, and the
                                   compensator is fused (its x A split over the CTAs, u B on the tensor
                                   cores).  Plan fields: tile_n = 128 (weight rows per tile), tile_m =
                                   16, 32 or 64 (token tile, >= M), split_k = K codes per pipeline stage
                                   (128 or 256, dividing K).  The scalar gate only. */
    SPEAR_KERNEL_STREAM_RK = 4  /* decode (M <= 64): the same stream-K schedule, workspace and fused
                                   compensator as SPEAR_KERNEL_STREAM, with the int4 codes converted
                                   into registers and fed to mma.sync (no TMEM staging).  Reads the
                                   codes in the tile order of spear_tile_w4 (plan flag
                                   SPEAR_PLAN_W4_TILES, required).  tile_n = 128, tile_m = 8, 16, 32
                                   or 64 (>= M; 64 needs SPEAR_PLAN_DEEP_RING), split_k = 128 or 256
                                   (dividing K), rank <= 128, scalar gate only. */
} spear_kernel;

/* spear_plan.flags bits. */
enum {
    /* The compensator leaves the GEMM's epilogue (section 2.2A); ignored without a compensator.
     * Split-K decode kernel: the weight-streaming CTAs write their fp32 main term to the
     * workspace and a second kernel, chained by programmatic dependent launch, applies the
     * compensator (the "split-K kernel with a separate EC pass").  It spares the weight-streaming
     * CTAs the wait for the compensator, which matters when their grid takes several waves.
     * Prefill kernel: the semi-fused path.  The EC tiles run alone on a side stream of the
     * library (highest priority; one per device, created on first use) beside the main tiles on
     * the caller's stream, which write the fp32 main term [M][N] to the workspace; after both, a
     * third kernel adds u B and rounds y.  The call forks and joins through events, so a CUDA
     * graph captured from the caller's stream holds the two as parallel branches (a static DAG).
     * Concurrent calls from several host threads are ordered by a lock around the enqueue. */
    SPEAR_PLAN_SEPARATE_EC = 1,
    /* SPEAR_KERNEL_STREAM and _STREAM_RK: one CTA per SM with a deep weight ring (up to 227 KB of shared
     * memory, 512 TMEM columns) instead of a ring small enough for two CTAs per SM.  The deep ring
     * keeps more weight bytes in flight (large layers); the small one lets the next call's CTAs
     * start their weight stream on the same SMs while this call finishes (small layers). */
    SPEAR_PLAN_DEEP_RING = 2,
    /* `packed` holds the codes in the tile order written by spear_tile_w4, not spear_pack_w4's
     * row order.  Required by SPEAR_KERNEL_STREAM_RK and rejected by every other kernel. */
    SPEAR_PLAN_W4_TILES = 4
};

/* Error compensator of one layer.  Pass NULL for a layer without EC (section
 * 2.1B: compensators sit only at the selected, error-sensitive modules). */
typedef struct {
    const void* A;    /* device, bf16 [K, rank]   down-projection */
    const void* B;    /* device, bf16 [rank, N]   up-projection */
    const void* w_g;  /* device, bf16 [K]         gate weights */
    float b_g;        /* gate bias (host value); -INFINITY gives g = 0 exactly */
    int32_t rank;     /* r: 16..256, a multiple of 16 */
    /* Optional: the pages' gate form (section 2.1A), effective weight W + alpha B diag(gamma(Ax)) A
     * with gamma a bottleneck MLP over t = x A:
     *   gamma(t) = sigmoid(W2 relu(W1 t + b1) + b2),   u = alpha * gamma(t) * t  (elementwise).
     * gate_w1 == NULL keeps the scalar gate above; otherwise w_g and b_g do not enter the result
     * (w_g must still be a readable [K] array).  All four arrays are fp32 on the device. */
    const void* gate_w1;   /* [gate_hidden, rank] */
    const void* gate_b1;   /* [gate_hidden] */
    const void* gate_w2;   /* [rank, gate_hidden] */
    const void* gate_b2;   /* [rank] */
    int32_t gate_hidden;   /* H: 1..64 */
    float alpha;           /* compensator scale (MLP gate only) */
} spear_ec;

/* A launch plan.  Produced by spear_gemm_plan and read by spear_w4ec_gemm.  A
 * caller may override kernel_id/split_k.  Invalid fields are rejected with
 * SPEAR_ERR_INVALID_ARG. */
typedef struct {
    int32_t kernel_id;        /* spear_kernel */
    int32_t tile_n;           /* weight rows per CTA (per tile for SPEAR_KERNEL_STREAM) */
    int32_t split_k;          /* number of K slices (1 = none), reduced in a thread-block cluster;
                                 SPEAR_KERNEL_STREAM: K codes per pipeline stage */
    int32_t tile_m;           /* token rows per CTA (or per launch chunk) */
    int32_t flags;            /* SPEAR_PLAN_* bits; 0 = none */
    int32_t reserved;
    size_t workspace_bytes;   /* minimum workspace for this (M, N, K, rank) */
} spear_plan;

/*
 * spear_pack_w4 -- RTN per-output-channel asymmetric int4 quantisation
 * (technical summary section 3.1: per-channel W4, RTN backend).
 *
 *   W       device, [N, K] fp32 (w_dtype = SPEAR_FP32) or bf16 (SPEAR_BF16)
 *   packed  device, uint8 [N, K/2]: byte b of row n holds q[n,2b] in bits 0..3
 *           and q[n,2b+1] in bits 4..7
 *   scale   device, fp16 [N]    s[n]
 *   zero    device, fp16 [N]    z[n], an integer in [0, 15]
 *
 * Per row, in IEEE fp32 operations, each correctly rounded:
 *   lo = min(min_k W, 0), hi = max(max_k W, 0); hi == lo -> lo = -1, hi = 1;
 *   s = fp16_rne((hi - lo) / 15); s == 0 -> row treated as all-zero;
 *   z = clamp(rint(-lo / s), 0, 15); q = clamp(rint(W / s) + z, 0, 15)
 *   (rint = round half to even).
 * Requires N >= 1 and K >= 2 with K even.  Deterministic: the output is
 * bit-identical on every run.
 */
SPEAR_API spear_status spear_pack_w4(const void* W, spear_dtype w_dtype, int64_t N, int64_t K,
                           void* packed, void* scale, void* zero, void* stream);

/*
 * spear_debug_unpack_w4 -- test hook: the codes and the exact (q - z) values
 * that the GEMM kernels feed their tensor-core operands.
 *
 *   packed     device, uint8 [N, K/2] (layout of spear_pack_w4)
 *   zero       device, fp16 [N]
 *   q_out      device, uint8 [N, K] or NULL
 *   qz_out     device, bf16 [N, K] holding (q - z), exact in bf16; or NULL
 */
SPEAR_API spear_status spear_debug_unpack_w4(const void* packed, const void* zero, int64_t N, int64_t K,
                                   void* q_out, void* qz_out, void* stream);

/*
 * spear_tile_w4 -- copy packed codes (spear_pack_w4's row order) into the tile order that
 * SPEAR_KERNEL_STREAM_RK streams (section 2.2A: decode is bound by the weight stream, so the codes
 * are laid out for it once, at load time).
 *
 *   packed  device, uint8 [N, K/2] (layout of spear_pack_w4)
 *   tiled   device, N * K / 2 bytes, 16-byte aligned, not overlapping `packed`
 *
 * Tile order: blocks of 128 rows x 128 codes (8192 bytes); block (T, B) holds rows 128T ..
 * 128T + 127 and codes 128B .. 128B + 127 and starts at byte (T * K/128 + B) * 8192.  Inside a
 * block, row r's 64 bytes start at r * 64 as 16 little-endian 32-bit words; word i = 4c + w
 * (c, w = 0..3) holds codes 8s .. 8s + 7 of the block row with s = 2c + w for w < 2 and
 * s = 8 + 2c + (w - 2) for w >= 2, code 8s + j in bits 4p .. 4p + 3 with p = (j / 2) + 4 (j % 2)
 * (codes 2i' and 2i' + 1 sit in nibbles i' and i' + 4).  The scales and zero-points are unchanged.
 * Requires N % 128 == 0 and K % 128 == 0.  A pure permutation of the 4-bit codes: bit-exact.
 */
SPEAR_API spear_status spear_tile_w4(const void* packed, int64_t N, int64_t K, void* tiled, void* stream);

/*
 * spear_gemm_plan -- host-only choice of kernel and tiling for one
 * (M, N, K, rank) problem (section 2.2A: the phase decides between the fused
 * epilogue and a separate EC kernel; section 2.2C: decisions come from
 * precomputed latency tables).  rank = 0 means no compensator.  `device` picks
 * the SM count used for sizing; pass -1 for the current device.  Launches
 * nothing.
 */
SPEAR_API spear_status spear_gemm_plan(int64_t M, int64_t N, int64_t K, int32_t rank, int device,
                             spear_plan* out);

/*
 * spear_gemm_plan_tiled -- as spear_gemm_plan, for codes in spear_tile_w4's tile order: a
 * SPEAR_KERNEL_STREAM_RK plan (flags include SPEAR_PLAN_W4_TILES).  Requires M <= 64,
 * N % 128 == 0, K % 128 == 0 and rank <= 128; SPEAR_ERR_UNSUPPORTED_SHAPE otherwise (such
 * problems need the row-order codes).  The plan serves the scalar gate only.
 */
SPEAR_API spear_status spear_gemm_plan_tiled(int64_t M, int64_t N, int64_t K, int32_t rank, int device,
                                   spear_plan* out);

/* Code orders a caller holds, for spear_gemm_plan_formats. */
enum { SPEAR_W4_ROWS = 1, SPEAR_W4_TILES = 2 };

/*
 * spear_gemm_plan_formats -- as spear_gemm_plan, choosing among the code orders the caller holds
 * (SPEAR_W4_ROWS: spear_pack_w4's; SPEAR_W4_TILES: spear_tile_w4's; either or both).  With both,
 * the plan reads the tile order (flags include SPEAR_PLAN_W4_TILES) when the measured latency
 * table has that order faster for this shape, and the row order otherwise.  The caller passes
 * the matching codes to spear_w4ec_gemm.  SPEAR_ERR_INVALID_ARG for an empty or unknown set.
 */
SPEAR_API spear_status spear_gemm_plan_formats(int64_t M, int64_t N, int64_t K, int32_t rank, int device,
                                     int32_t formats, spear_plan* out);

/*
 * spear_plan_update -- check a plan whose fields the caller has changed (kernel, tiling, flags)
 * for this shape and recompute plan->workspace_bytes in place.  The semi-fused prefill path
 * (SPEAR_KERNEL_TC05 with SPEAR_PLAN_SEPARATE_EC and a compensator), for one, needs M * N * 4
 * more bytes than the fused one.  Host only; launches nothing.
 *
 *   plan       host, in/out
 * Returns SPEAR_ERR_INVALID_ARG for a NULL plan or a field the kernels do not support, and
 * SPEAR_ERR_UNSUPPORTED_SHAPE as spear_gemm_plan does; the plan is unchanged then.
 */
SPEAR_API spear_status spear_plan_update(spear_plan* plan, int64_t M, int64_t N, int64_t K, int32_t rank);

/*
 * spear_w4ec_gemm -- y = x dequant(Wq)^T + g(x) * ((x A) B)  (section 2.1A).
 *
 *   plan       host, from spear_gemm_plan, or NULL (planned on the fly)
 *   x          device, bf16 [M, K]
 *   packed, scale, zero   from spear_pack_w4 for W [N, K]; with SPEAR_PLAN_W4_TILES in the
 *              plan's flags, packed from spear_tile_w4 (a NULL plan means row order)
 *   ec         host struct with device pointers, or NULL for a plain W4 layer
 *   y          device, [M, N], bf16 (y_dtype = SPEAR_BF16, one rounding at the
 *              end) or fp32 (SPEAR_FP32, unrounded: a test/debug output)
 *   workspace  device, >= plan->workspace_bytes.  Zero-fill it once before its
 *              first use.  Every call leaves its control words zeroed again.
 *              Calls that share a workspace must be ordered on one stream.
 *
 * Requires N % 128 == 0, K % 64 == 0 (and K <= 65536 with a compensator),
 * M >= 0 (M = 0 launches nothing).  The accumulation is fp32 throughout (the
 * EC factors u = g t enter the prefill tensor cores rounded to bf16).  The
 * output is deterministic for a given plan: no atomics take part in any
 * floating-point sum.
 */
SPEAR_API spear_status spear_w4ec_gemm(const spear_plan* plan, const void* x, int64_t M, int64_t N, int64_t K,
                             const void* packed, const void* scale, const void* zero,
                             const spear_ec* ec, void* y, spear_dtype y_dtype,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * spear_w4ec_gemm_noalloc -- the same layer as spear_w4ec_gemm for decode-sized batches, without a
 * workspace.  The SPEAR pages have no counterpart to this call; it exists for callers that cannot
 * allocate device memory: code whose device memory belongs to another allocator or framework
 * that hands out no scratch buffers, and latency-critical paths where an allocation could block
 * or fail at an unpredictable moment.
 *
 * The layer's scratch (an error word, per-token-chunk counters and the compensator's int64
 * accumulators) lives in one library-owned device array of 256 KiB.  Every GPU that loads the
 * library holds that array until the process exits.  Nothing is allocated, by this call or by
 * anything it calls.
 *
 *   Arguments as for spear_w4ec_gemm, minus the workspace.  plan may be NULL; a given plan must
 *   select SPEAR_KERNEL_SPLITK.
 *   Limits: 1 <= M <= 64 (larger M returns SPEAR_ERR_UNSUPPORTED_SHAPE), rank 0 or 16..256, the
 *   scalar gate only (ec->gate_w1 != NULL returns SPEAR_ERR_INVALID_ARG).
 *   plan == NULL plans the split-K decode kernel for the shape (never another kernel).
 *   The first call on a device looks up that device's scratch address (once per device, with the
 *   device current); make that first call before any stream capture.  The array starts zeroed
 *   and each completed call leaves its counters and accumulators zeroed again, so a call clears
 *   nothing before its launch.
 *   All calls share the one array and it keeps the last call's contents: calls that can overlap
 *   on the GPU (different streams, or different host threads) race and must be serialised by the
 *   caller.  Timeouts of bounded in-kernel waits are read (and the array reset after one) with
 *   spear_noalloc_get_device_status.
 */
SPEAR_API spear_status spear_w4ec_gemm_noalloc(const spear_plan* plan, const void* x, int64_t M, int64_t N,
                                               int64_t K, const void* packed, const void* scale, const void* zero,
                                               const spear_ec* ec, void* y, spear_dtype y_dtype, void* stream);

/*
 * spear_noalloc_get_device_status -- the error word of spear_w4ec_gemm_noalloc's array (the
 * timeouts of its bounded in-kernel waits), as spear_get_device_status reads a workspace's.  With
 * clear != 0 and a nonzero word, the whole array is zeroed, so that the next call starts clean.
 * Synchronises `stream`; order it after the calls it should observe.  Allocates nothing.
 * Returns SPEAR_OK, SPEAR_ERR_TIMEOUT, or SPEAR_ERR_CUDA.
 */
SPEAR_API spear_status spear_noalloc_get_device_status(int clear, void* stream);

/*
 * Group-wise scales (section 3.1: the method sits on GPTQ, AWQ and OmniQuant backends as well as
 * on RTN).  Every `group` consecutive k of a row have their own binary16 scale and zero-point,
 * found by the same RTN steps as spear_pack_w4 applied to that group alone:
 *   What[n,k] = (q[n,k] - z[n, k/group]) * s[n, k/group]
 *
 * spear_pack_w4_grouped -- as spear_pack_w4, with scale and zero [N, K/group] (row-major).
 *   group      even and dividing K; spear_w4ec_gemm_grouped needs a multiple of 128
 *   packed     [N, K/2], the same layout as spear_pack_w4's
 * Returns SPEAR_ERR_UNSUPPORTED_SHAPE for a group that is odd or does not divide K.
 */
SPEAR_API spear_status spear_pack_w4_grouped(const void* W, spear_dtype w_dtype, int64_t N, int64_t K,
                                             int64_t group, void* packed, void* scale, void* zero, void* stream);

/*
 * spear_grouped_workspace_bytes -- workspace of spear_w4ec_gemm_grouped for this shape: the
 * zeroed control block, plus, with a compensator, u (bf16 [M, rank]) and the fp32 main term
 * [M, N].  Host only.
 */
SPEAR_API spear_status spear_grouped_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t group,
                                                     int32_t rank, size_t* out);

/*
 * spear_w4ec_gemm_grouped -- y = x What^T + g(x) * ((x A) B) with group-wise scales.
 *
 * Arguments as for spear_w4ec_gemm, without a plan, with `group` and the [N, K/group] scale and
 * zero from spear_pack_w4_grouped.  Requires N % 128 == 0, group a multiple of 128 dividing K, and a
 * compensator rank of at most 128 (16..128, step 16); the scalar and the MLP gate are both taken.
 * A weight-streaming tensor-core kernel computes the main term, applying each group's scale to its
 * 128-code windows.  With a compensator the main term goes to the workspace (fp32) and the
 * compensator runs beside it on the library's side stream (as SPEAR_PLAN_SEPARATE_EC does for the
 * prefill kernel), joined by a kernel that adds u B and rounds y once.  Deterministic.
 */
SPEAR_API spear_status spear_w4ec_gemm_grouped(const void* x, int64_t M, int64_t N, int64_t K, int64_t group,
                                               const void* packed, const void* scale, const void* zero,
                                               const spear_ec* ec, void* y, spear_dtype y_dtype, void* workspace,
                                               size_t workspace_bytes, void* stream);

/*
 * spear_get_device_status -- read (and optionally clear) the error word that
 * bounded in-kernel waits set when they give up.  Synchronises `stream`.
 * Returns SPEAR_OK, SPEAR_ERR_TIMEOUT, or SPEAR_ERR_CUDA.
 */
SPEAR_API spear_status spear_get_device_status(void* workspace, int clear, void* stream);

/*
 * EC-aware, SLO-constrained prefill chunk picker (section 2.2C): the largest prefill chunk whose
 * predicted step latency meets the inter-token-latency target, from tables of measured kernel
 * latencies.  Host only; nothing here touches a GPU.
 *
 * A step runs every linear of the model once on M = decode_tokens + chunk tokens.  Predicted step
 * latency = fixed_us + sum_i count_i * T(M, N_i, K_i, rank_i > 0), where T reads the latency table:
 * for one (N, K, compensator or not) its samples are made nondecreasing in M, then interpolated
 * linearly between measured M, held at the smallest measured M below it, and scaled by
 * M / M_max above the largest.  The step latency is therefore nondecreasing in M.
 */
typedef struct {
    int64_t N, K;       /* the linear's W [N, K] */
    int32_t rank;       /* its compensator's rank; 0 = none (where compensators sit is what the
                           picker adapts to) */
    int32_t count;      /* how many linears of this shape and rank one step runs (>= 0) */
} spear_linear_desc;

typedef struct {
    int64_t M, N, K;    /* tokens and weight shape of one call */
    int32_t has_ec;     /* nonzero: with a compensator */
    int32_t reserved;
    double us;          /* device time of one call, microseconds */
} spear_latency_entry;

/*
 * spear_latency_table -- copy the library's built-in latency table: for each shape measured on
 * a B200, the device time per call of its fastest plan in a chained CUDA graph (the dispatcher's
 * table; one row per (M, N, K, compensator or not), the faster code order where the table holds
 * both).  out may be NULL to query *len_out only; otherwise capacity must be >= *len_out.
 */
SPEAR_API spear_status spear_latency_table(spear_latency_entry* out, int32_t capacity, int32_t* len_out);

/*
 * spear_predict_step_us -- predicted latency of one step on M tokens (0 <= M <= 65536).
 *   linears, n_linears   host array (n_linears >= 1)
 *   fixed_us             time of the step outside these linears (>= 0), added as is
 *   lut, lut_len         host latency table, or NULL to use the built-in one
 * Returns SPEAR_ERR_UNSUPPORTED_SHAPE if a linear with count > 0 has no row of its (N, K,
 * compensator or not) in the table, SPEAR_ERR_INVALID_ARG for bad arguments or table rows.
 */
SPEAR_API spear_status spear_predict_step_us(const spear_linear_desc* linears, int32_t n_linears, int64_t M,
                                             double fixed_us, const spear_latency_entry* lut, int32_t lut_len,
                                             double* us_out);

/*
 * spear_pick_prefill_chunk -- the largest chunk = c * granule (c >= 0, chunk <= max_chunk and
 * decode_tokens + chunk <= 65536) whose predicted step latency on decode_tokens + chunk tokens
 * is <= slo_us; *predicted_us_out is that step's predicted latency.  If the decode tokens alone
 * already miss the target, *chunk_out = 0 and *predicted_us_out > slo_us.  Other arguments and
 * errors as for spear_predict_step_us; slo_us > 0, granule >= 1.
 */
SPEAR_API spear_status spear_pick_prefill_chunk(const spear_linear_desc* linears, int32_t n_linears,
                                                int64_t decode_tokens, int64_t max_chunk, int64_t granule,
                                                double slo_us, double fixed_us, const spear_latency_entry* lut,
                                                int32_t lut_len, int64_t* chunk_out, double* predicted_us_out);

/* Static string for a status code (never NULL). */
SPEAR_API const char* spear_status_string(spear_status status);

/* Library version, as MAJOR * 10000 + MINOR * 100 + PATCH. */
SPEAR_API int spear_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SPEAR_H */
