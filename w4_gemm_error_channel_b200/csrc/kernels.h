// kernels.h -- internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

#include "../../include/spear.h"

namespace spear {

// Host helpers shared by the kernels' launchers (tc05.cu).
constexpr int kMaxDevices = 64;
// 2-D tensor map over a row-major [rows][cols] array of `elem`-byte elements, box {box_cols, box_rows}.
bool make_map_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem, uint64_t cols,
                 uint64_t rows, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz);
// 3-D tensor map: dims[0] innermost, strides of dims 1 and 2 in bytes.
bool make_map_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, const uint64_t dims[3],
                 const uint64_t strides_bytes[2], const uint32_t box[3], CUtensorMapSwizzle swz);
// Raise `func`'s dynamic shared-memory limit to `bytes` once per device (thread-safe); `once` and
// `status` are per-function arrays of kMaxDevices entries.
cudaError_t opt_in_smem(const void* func, size_t bytes, std::once_flag* once, cudaError_t* status);
// For kernels whose dynamic size varies per launch (and that may also use static shared memory):
// raise the limit to `bytes` if it is below, under `mu`; opted[] holds the limit set per device.
cudaError_t opt_in_smem_at_least(const void* func, size_t bytes, std::mutex& mu, size_t* opted);
// Largest dynamic shared memory of a block on sm_100.
constexpr size_t SMEM_OPTIN_MAX = 227 * 1024;

// Zeroed part of every workspace: it must start zeroed and every call leaves it zeroed again
// (unless a bounded wait timed out).
//   control block, CTRL_BYTES, in 32-bit words:
//     [0]                     device error word (bit 0: a wait for the EC accumulators gave up;
//                             bit 1: an EC partial sum was outside the fixed-point range;
//                             bits 2, 3: prefill kernel waits)
//     [64, +CHUNKS)           reserved (cleared by the decode kernel; no longer counted)
//     [.., +CHUNKS)           consumer counters (level 2: finished groups), one per token chunk;
//                             word 0 also counts the CTAs of the separate EC pass
//     [.., +CHUNKS*GROUPS)    consumer counters (level 1: CTAs of a group of 64 GEMM CTAs)
//     [.., +TC_BLOCKS)        prefill kernel: u-ready flags, one per token block
//     [.., +TC_BLOCKS)        prefill kernel: flag consumer counters
//   EC accumulators, TACC_BYTES: int64 [tokens of a launch][r + 1] (t, then the gate
//   pre-activation), fixed point with 32 fraction bits above an 8-bit count of the K slices added.
// After the zeroed part: the prefill kernel's u (bf16 [M][r], padded to 256 bytes), then, on
// the semi-fused prefill path, its fp32 main term ([M][N]); or the decode kernel's separate EC
// pass's fp32 main term ([tokens of a launch][N]).
constexpr size_t CTRL_BYTES = 128 * 1024;
constexpr size_t CTRL_HEADER_WORDS = 64;
constexpr size_t CHUNKS_MAX = 32;                          // token chunks per launch (>= 8 tokens each)
constexpr int CONSUMER_GROUP = 64;                         // GEMM CTAs per level-1 consumer counter
constexpr size_t GROUPS_MAX = 256;                         // level-1 counters per token chunk
constexpr size_t TACC_BYTES = 1024 * 1024;
constexpr size_t ZEROED_BYTES = CTRL_BYTES + TACC_BYTES;
constexpr int64_t LAUNCH_TOKENS_MAX = 256;                 // tokens per decode launch
constexpr size_t TC_BLOCKS_MAX = 512;                      // token blocks of the prefill kernel (M <= 65536)
constexpr int64_t M_MAX = 65536;
constexpr size_t TC_FLAGS_WORD = CTRL_HEADER_WORDS + 2 * CHUNKS_MAX + CHUNKS_MAX * GROUPS_MAX;
static_assert(TC_FLAGS_WORD + 2 * TC_BLOCKS_MAX <= CTRL_BYTES / 4, "control block");

// The pages' bottleneck-MLP gate over t = x A: gamma = sigmoid(w2 relu(w1 t + b1) + b2),
// u = alpha gamma t.  w1 == null selects the scalar gate sigmoid(x w_g + b_g).
constexpr int GATE_HIDDEN_MAX = 64;
struct GateMlp {
    const float* w1;        // [H][r]
    const float* b1;        // [H]
    const float* w2;        // [r][H]
    const float* b2;        // [r]
    int hidden;             // H
    float alpha;
};

struct DecodeArgs {
    const uint16_t* x;      // bf16 [M, K]
    const uint8_t* packed;  // [N, K/2]
    const __half* scale;    // [N]
    const __half* zero;     // [N]
    const uint16_t* A;      // bf16 [K, r]   (EC; rank == 0 means no EC)
    const uint16_t* B;      // bf16 [r, N]
    const uint16_t* wg;     // bf16 [K]
    float b_g;
    int rank;
    void* y;
    int y_fp32;
    int64_t M, N, K;
    int64_t k_slice;        // GEMM K slice per CTA, a multiple of 64
    int split;              // S: GEMM K slices = thread-block cluster size (1, 2, 4 or 8)
    int ec_jr;              // EC columns added per K slice (multiple of 4)
    int ec_splits;          // EC CTAs per token chunk (decode_ec_ctas_per_chunk)
    int ec_ctas;            // EC CTAs in the grid (ec_splits * mchunks, padded to whole clusters)
    int row_tiles;          // N / (16 G)
    int mchunks;            // ceil(M / (8 NB))
    long long* tacc;        // [M][r + 1] EC accumulators (zeroed part of the workspace)
    unsigned* err;          // error word
    unsigned* arrivals;     // [mchunks] reserved words, cleared with the accumulators
    unsigned* consumed;     // [mchunks] level-2 consumer counters
    unsigned* consumed1;    // [mchunks][GROUPS_MAX] level-1 consumer counters
    float* ymain;           // separate EC pass: fp32 main term [M][N] (workspace); null when fused
    GateMlp mlp;            // bottleneck-MLP gate (w1 == null: the scalar gate)
    int64_t group;          // 0: per-channel scale/zero [N]; else group-wise [N][K / group], group a
                            // multiple of 128 and k_slice a multiple of 128
};

// Prefill (tcgen05) kernel arguments.
struct TcArgs {
    const uint16_t* x;      // bf16 [M, K]
    const uint8_t* packed;  // [N, K/2]
    const __half* scale;    // [N]
    const __half* zero;     // [N]
    const uint16_t* A;      // bf16 [K, r]  (EC; rank == 0 means none)
    const uint16_t* B;      // bf16 [r, N]
    const uint16_t* wg;     // bf16 [K]
    float b_g;
    int rank;               // 0 or 16..128
    __nv_bfloat16* u;       // [M][r] bf16 u = g t (workspace, written by the EC tiles)
    void* y;
    int y_fp32;
    int64_t M, N, K;
    unsigned* err;          // error word (bit 2: an mbarrier wait gave up; bit 3: an EC-ready wait gave up)
    unsigned* ec_ready;     // [token blocks] u of the block is ready
    unsigned* ec_consumed;  // [token blocks] main tiles that have seen the flag
    GateMlp mlp;            // bottleneck-MLP gate (w1 == null: the scalar gate)
    int ec_only;            // 1: launch the EC tiles alone (u only, no ready flags); 0: the whole layer
    int split;              // K splits per weight tile, one cluster of `split` CTAs (set by launch_tc05)
};

// Small-batch stream-K kernel (stream.cu).  The host fills the problem fields and `grid`, then
// stream_configure() fills the tiling, shared-memory layout and compensator slicing.
constexpr size_t STREAM_GRID_MAX = 1024;                   // CTAs (one partial-sum flag each)
constexpr size_t STREAM_FLAGS_WORD = TC_FLAGS_WORD + 2 * TC_BLOCKS_MAX;
static_assert(STREAM_FLAGS_WORD + STREAM_GRID_MAX + 1 <= CTRL_BYTES / 4, "control block");
struct StreamArgs {
    const uint16_t* x;      // bf16 [M, K]
    const uint8_t* packed;  // [N, K/2]
    const __half* scale;    // [N]
    const __half* zero;     // [N]
    const uint16_t* A;      // bf16 [K, r]   (rank == 0: no compensator)
    const uint16_t* B;      // bf16 [r, N]
    const uint16_t* wg;     // bf16 [K]
    float b_g;
    int rank;
    void* y;
    int y_fp32;
    int64_t M, N, K;
    int grid;               // CTAs (<= SMs, <= units)
    // filled by stream_configure
    int kc, nch, ntiles, units;     // K codes per unit, units per tile, tiles, units in all
    int nst, na;                    // shared-memory stages, TMEM sub-chunk slots
    int jb, nbu;                    // B rows per B unit, B units per finalised tile
    int stage_bytes, off_u, off_a, off_wg, off_g, off_bar, smem_bytes;
    int off_b, off_red, nfin;       // register path: B-slice buffer, K-half exchange buffer, finalised EC tiles
    uint32_t tmem_cols;
    int ec_kr, ec_slices;           // rows of A per compensator slice, slices (<= grid)
    int ec_groups;                  // register path: 16-column groups of A (+ the gate) per slice;
                                    // one (slice, group) item per CTA
    int finalizers;                 // CTAs that finalise at least one tile
    // workspace
    long long* tacc;        // [M][r + 1] int64 fixed-point accumulators (zeroed part)
    unsigned* err;          // error word
    unsigned* flags;        // [grid] partial-sum ready flags (zeroed part)
    unsigned* ec_readers;   // CTAs that have read the accumulators (zeroed part)
    float* partial;         // [grid][BN][128] fp32 partial sums (register path: 64-bit words,
                            // ready tag in the high half; the reader zeroes them)
};
int stream_grid(int64_t N, int64_t K, int kc, int sms, bool deep);
// The register-path variant (stream_rk.cu): same schedule and workspace, converted weights in
// registers feeding mma.sync.  bn = 8, 16, 32 or 64 tokens; kc = 128 or 256; rank <= 128.
bool stream_rk_configure(StreamArgs& a, int bn, int kc, bool deep);
cudaError_t launch_stream_rk(const StreamArgs& a, int bn, cudaStream_t stream);
// A fused split-K decode plan for this shape (api.cu).
spear_status plan_split_k_decode(int64_t M, int64_t N, int64_t K, int32_t rank, spear_plan* out);
bool stream_configure(StreamArgs& a, int bn, int kc, bool deep);
cudaError_t launch_stream(const StreamArgs& a, int bn, cudaStream_t stream);

// bn = tokens per tile; rows = weight rows per tile (128, or 256 with bn = 128).  pdl: launch as a
// programmatic dependent of the previous kernel in the stream; priority: 0 or a launch priority.
cudaError_t launch_tc05(const TcArgs& a, int bn, int rows, cudaStream_t stream, bool pdl = true, int priority = 0,
                        int split = 1);
// Whether launch_tc05 takes this K split for a tile of bn tokens and `rows` weight rows.
bool tc05_split_supported(int bn, int rows, int split, int64_t K);

// The compensator beside a main-term launch: the tcgen05 kernel's EC tiles alone (u = g t) on a
// side stream of the library, `main` (which writes the fp32 main term to ymain [M][N]) on the
// caller's stream, joined by ec_up_add (y = ymain + u B).  `ctx` is read during the call only.
using MainLaunch = cudaError_t (*)(const void* ctx, cudaStream_t stream);
cudaError_t launch_ec_beside(const TcArgs& a, MainLaunch main, const void* ctx, float* ymain, cudaStream_t stream);
// Semi-fused prefill: launch_ec_beside with the tcgen05 kernel's main tiles as the main term.
cudaError_t launch_semifused(const TcArgs& a, int bn, int rows, float* ymain, cudaStream_t stream);

// Group-wise scales: s, z [N, K / group], group a multiple of 128 dividing K.  Writes the main
// term to ymain (fp32 [M][N]) when it is set, else y.
struct GroupedArgs {
    const uint16_t* x;      // bf16 [M, K]
    const uint8_t* packed;  // [N, K/2]
    const __half* scale;    // [N, K/group]
    const __half* zero;     // [N, K/group]
    int64_t M, N, K, group;
    float* ymain;
    void* y;
    int y_fp32;
};
cudaError_t launch_w4g_gemm(const GroupedArgs& a, cudaStream_t stream);

cudaError_t launch_pack_w4(const void* W, bool w_is_bf16, int64_t N, int64_t K, void* packed, void* scale,
                           void* zero, cudaStream_t stream);
cudaError_t launch_tile_w4(const void* packed, int64_t N, int64_t K, void* tiled, cudaStream_t stream);
cudaError_t launch_unpack_w4(const void* packed, const void* zero, int64_t N, int64_t K, void* q_out,
                             void* qz_out, cudaStream_t stream);

// nb: tokens per CTA = 8*nb (1, 2, 4); g: weight rows per CTA = 16*g; wpw: 128-wide K windows per
// warp (K slice of a CTA <= 512*wpw).  decode_config_supported() lists the compiled combinations.
bool decode_config_supported(int nb, int g, int wpw);
// Largest K with a compensator: the decode kernel counts K slices of 512 rows in 8 bits.
constexpr int64_t EC_K_MAX = 65536;
int decode_ec_ctas_per_chunk(int64_t K, int rank);
// Separate EC pass after the decode kernel (it reads DecodeArgs::ymain, tacc, B).
cudaError_t launch_apply(const DecodeArgs& a, cudaStream_t stream);
size_t apply_dyn_smem_bytes(int rank, int gate_hidden);
size_t decode_dyn_smem_bytes(int nb, int g, int ec_jr, int rank, int gate_hidden);
cudaError_t launch_decode(const DecodeArgs& a, int nb, int g, int wpw, cudaStream_t stream);

}  // namespace spear
