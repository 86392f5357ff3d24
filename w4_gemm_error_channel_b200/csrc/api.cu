// api.cu -- the C ABI declared in include/spear.h: argument checks, planning, workspace layout
// and kernel dispatch.  Host code only; the kernels live in pack.cu and decode.cu.
#include <math.h>
#include <cmath>
#include <cstdlib>

#include "common.cuh"
#include "kernels.h"

using namespace spear;

namespace {

constexpr int MAX_DEVICES = 64;
constexpr int DEFAULT_SMS = 148;  // B200, used when no device can be queried (host-only planning)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int device_sms(int device) {
    static int cache[MAX_DEVICES] = {0};
    if (device < 0 && cudaGetDevice(&device) != cudaSuccess) return DEFAULT_SMS;
    if (device < 0 || device >= MAX_DEVICES) return DEFAULT_SMS;
    if (cache[device] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || v <= 0) {
            cudaGetLastError();
            return DEFAULT_SMS;
        }
        cache[device] = v;
    }
    return cache[device];
}

spear_status check_shape(int64_t M, int64_t N, int64_t K, int32_t rank) {
    if (M < 0 || N <= 0 || K <= 0 || rank < 0) return SPEAR_ERR_INVALID_ARG;
    if (N % 128 != 0 || K % 64 != 0) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    if (M > M_MAX) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    if (rank != 0 && (rank < 16 || rank > 256 || rank % 16 != 0)) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    if (rank != 0 && K > EC_K_MAX) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    return SPEAR_OK;
}

// The optional bottleneck-MLP gate: all four arrays or none, H in 1..GATE_HIDDEN_MAX.
spear_status check_gate_mlp(const spear_ec* ec) {
    if (!ec || !ec->gate_w1) return SPEAR_OK;
    if (!ec->gate_b1 || !ec->gate_w2 || !ec->gate_b2) return SPEAR_ERR_INVALID_ARG;
    if (ec->gate_hidden < 1 || ec->gate_hidden > GATE_HIDDEN_MAX || isnan(ec->alpha)) return SPEAR_ERR_INVALID_ARG;
    if (!aligned16(ec->gate_w1) || !aligned16(ec->gate_b1) || !aligned16(ec->gate_w2) || !aligned16(ec->gate_b2))
        return SPEAR_ERR_MISALIGNED;
    return SPEAR_OK;
}

GateMlp gate_mlp_of(const spear_ec* ec) {
    GateMlp g = {};
    if (ec && ec->gate_w1) {
        g.w1 = (const float*)ec->gate_w1;
        g.b1 = (const float*)ec->gate_b1;
        g.w2 = (const float*)ec->gate_w2;
        g.b2 = (const float*)ec->gate_b2;
        g.hidden = ec->gate_hidden;
        g.alpha = ec->alpha;
    }
    return g;
}

int nb_for_tile_m(int tile_m) { return tile_m <= 8 ? 1 : (tile_m <= 16 ? 2 : 4); }

// K codes per slice for S slices: a multiple of 64, so every lane's 32-code piece is whole.
int64_t k_slice_for(int64_t K, int64_t S) { return ((K + S - 1) / S + 63) / 64 * 64; }
int wpw_for(int64_t k_slice) { return (int)((k_slice + 511) / 512); }
int ec_jr_for(int32_t rank, int64_t S) {
    if (rank <= 0) return 0;
    return (int)(((rank + S - 1) / S + 3) / 4 * 4);
}
// u of the prefill kernel, bf16 [M][r], padded to 256 bytes.
size_t tc05_u_bytes(int64_t M, int32_t rank) { return ((size_t)M * rank * 2 + 255) / 256 * 256; }

// Workspace: the zeroed prefix (control block + EC accumulators); split-K partial sums meet in
// distributed shared memory.  The prefill kernel with a compensator also keeps u (bf16 [M][r]).
size_t workspace_bytes_for(const spear_plan& p, int64_t M, int64_t N_for_ws, int64_t K, int32_t rank, int sms) {
    size_t b = ZEROED_BYTES;
    if (p.kernel_id == SPEAR_KERNEL_STREAM || p.kernel_id == SPEAR_KERNEL_STREAM_RK) {
        // fp32 partial sums of the tiles that straddle two CTAs: [grid][tile_m][128].
        const int grid = p.split_k > 0 && K % p.split_k == 0 ? stream_grid(N_for_ws, K, p.split_k, sms, (p.flags & SPEAR_PLAN_DEEP_RING) != 0) : 0;
        const size_t word = p.kernel_id == SPEAR_KERNEL_STREAM_RK ? 8 : 4;   // tagged 64-bit words there
        return b + (size_t)grid * p.tile_m * 128 * word;
    }
    if (p.kernel_id == SPEAR_KERNEL_TC05 && rank > 0) b += tc05_u_bytes(M, rank);
    if (p.kernel_id == SPEAR_KERNEL_TC05 && (p.flags & SPEAR_PLAN_SEPARATE_EC) && rank > 0)
        b += (size_t)M * N_for_ws * 4;                                              // fp32 main term
    if (p.kernel_id == SPEAR_KERNEL_SPLITK && (p.flags & SPEAR_PLAN_SEPARATE_EC) && rank > 0)
        b += (size_t)(M < LAUNCH_TOKENS_MAX ? M : LAUNCH_TOKENS_MAX) * N_for_ws * 4;   // fp32 main term
    return b;
}

// Decode plan.  Every weight byte of a CTA (16*g rows x K/S codes, 128 threads) is requested up
// front; the S K slices of a row tile form a cluster (S in {1, 2, 4, 8}).  The cost model prefers
// tilings that spread the weight bytes evenly over all SMs (many small CTAs stream best), then
// the least re-reading of activations from L2, then fewer slices.
// Measured plans (plans/gen_table.py): the fastest tiling per swept shape on one B200.
struct MeasuredPlan {
    int64_t M, N, K;
    int has_ec, kernel_id, tile_n, split_k, tile_m, flags;
    double us;
};
spear_status plan_tc05(int64_t M, int64_t N, int sms, spear_plan* p);

const MeasuredPlan kMeasured[] = {
#include "plan_table.inc"
};

spear_status validate_plan(const spear_plan& p, int64_t M, int64_t N, int64_t K, int32_t rank);

// tiles: only the register-path stream kernel's entries (codes in tile order); otherwise every
// other kernel's.
bool lookup_measured(int64_t M, int64_t N, int64_t K, int32_t rank, int sms, spear_plan* p, bool tiles = false,
                     double* us = nullptr) {
    const int has_ec = rank > 0 ? 1 : 0;
    const int nb = M <= 8 ? 1 : (M <= 16 ? 2 : 4);
    const MeasuredPlan* best = nullptr;
    for (const MeasuredPlan& e : kMeasured) {
        const int enb = e.M <= 8 ? 1 : (e.M <= 16 ? 2 : 4);
        if ((e.kernel_id == SPEAR_KERNEL_STREAM_RK) != tiles) continue;
        if (e.N != N || e.K != K || e.has_ec != has_ec || enb != nb) continue;
        if (e.M > 2 * M || 2 * e.M < M) continue;        // measured within a factor of two of M
        // Same token-tile size; prefer the measured batch closest to M.
        if (!best || std::llabs(e.M - M) < std::llabs(best->M - M)) best = &e;
    }
    if (!best) return false;
    if (us) *us = best->us;
    if (best->kernel_id == SPEAR_KERNEL_STREAM || best->kernel_id == SPEAR_KERNEL_STREAM_RK) {
        // The measured stage width and ring mode; the token tile must hold M.
        const int bn = (best->kernel_id == SPEAR_KERNEL_STREAM_RK && M <= 8) ? 8 : M <= 16 ? 16 : (M <= 32 ? 32 : 64);
        if (M > 64 || K % best->split_k != 0) return false;
        p->kernel_id = best->kernel_id;
        p->tile_n = 128;
        p->split_k = best->split_k;
        p->tile_m = best->tile_m > bn ? best->tile_m : bn;
        p->flags = (best->flags & SPEAR_PLAN_DEEP_RING) | (tiles ? SPEAR_PLAN_W4_TILES : 0);
        p->reserved = 0;
        if (validate_plan(*p, M, N, K, rank) != SPEAR_OK) return false;
        return true;
    }
    if (best->kernel_id == SPEAR_KERNEL_TC05) {
        if (plan_tc05(M, N, sms, p) != SPEAR_OK) return false;
        if (best->tile_m == 128 || best->tile_m == 256) p->tile_m = best->tile_m;   // the measured width
        if (tc05_split_supported(p->tile_m, p->tile_n, best->split_k, K)) p->split_k = best->split_k;
        return true;
    }
    p->kernel_id = SPEAR_KERNEL_SPLITK;
    p->tile_n = best->tile_n;
    p->split_k = best->split_k;
    p->tile_m = 8 * nb;
    p->flags = has_ec ? (best->flags & SPEAR_PLAN_SEPARATE_EC) : 0;
    p->reserved = 0;
    return true;
}

spear_status plan_decode_rules(int64_t M, int64_t N, int64_t K, int32_t rank, int sms, spear_plan* p);
spear_status plan_decode(int64_t M, int64_t N, int64_t K, int32_t rank, int sms, spear_plan* p) {
    if (lookup_measured(M, N, K, rank, sms, p)) return SPEAR_OK;
    return plan_decode_rules(M, N, K, rank, sms, p);
}

// The split-K decode kernel's tiling from the cost model alone.
spear_status plan_decode_rules(int64_t M, int64_t N, int64_t K, int32_t rank, int sms, spear_plan* p) {
    (void)rank;
    const int nb = M <= 8 ? 1 : (M <= 16 ? 2 : 4);
    const int64_t tm = 8 * nb;
    const int64_t ml = M < LAUNCH_TOKENS_MAX ? M : LAUNCH_TOKENS_MAX;
    const int64_t mchunks = (ml + tm - 1) / tm;
    const double wbytes = (double)N * K / 2;
    const double hbm = 6.5e12, l2 = 20e12;
    double best = 1e300;
    int best_g = 1, best_s = 1;
    const int gs[4] = {1, 2, 4, 8};
    const int ss[4] = {1, 2, 4, 8};
    for (int gi = 0; gi < 4; ++gi) {
        const int g = gs[gi];
        const int64_t rt = 16 * g;
        if (N % rt != 0) continue;
        const int64_t tiles = (N / rt) * mchunks;
        for (int si = 0; si < 4; ++si) {
            const int64_t S = ss[si];
            const int64_t ksl = k_slice_for(K, S);
            if ((S - 1) * ksl >= K) continue;               // no empty slices
            if (!decode_config_supported(nb, g, wpw_for(ksl))) continue;
            const double ctas = (double)tiles * S;
            // Work per SM in whole CTAs (4 CTAs of 128 threads resident per SM).
            const double rounds = std::ceil(ctas / (4.0 * sms));
            const double balance = rounds * 4.0 * sms / ctas;   // >= 1; 1 = even
            const double spread = ctas < sms ? (double)sms / ctas : 1.0;
            const double xbytes = (double)(N / rt) * M * K * 2;
            const double cost = wbytes / hbm * balance * spread + xbytes / l2 + (S > 1 ? 0.2e-6 : 0.0);
            if (cost < best * 0.999) { best = cost; best_g = g; best_s = (int)S; }
        }
    }
    p->kernel_id = SPEAR_KERNEL_SPLITK;
    p->tile_n = 16 * best_g;
    p->split_k = best_s;
    p->tile_m = (int32_t)tm;
    p->flags = 0;
    p->reserved = 0;
    return SPEAR_OK;
}

// Prefill (tcgen05) plan: 128 weight rows x tile_m tokens per CTA, no K split.  Every weight
// tile of a token block reads that block's x from L2, so the L2-to-SM traffic is led by x times
// N / 128 whatever the token width; wider token tiles cut the weight re-reads.  Measured on the
// 2048 x 4096 x 14336 layer (with EC): 253 us at 256 tokens, 306 at 160, 348 at 192, 382 at 128.
// 160 and 192 stay available to explicit plans.
spear_status plan_tc05(int64_t M, int64_t N, int sms, spear_plan* p) {
    (void)N;
    (void)sms;
    p->kernel_id = SPEAR_KERNEL_TC05;
    p->tile_n = 128;
    p->split_k = 1;
    p->tile_m = M >= 2048 ? 256 : 128;
    p->flags = 0;
    p->reserved = 0;
    return SPEAR_OK;
}

// Group-wise layer: groups of a multiple of 128 codes dividing K; with a compensator, its EC
// tiles run on the tcgen05 kernel (rank <= TC05_MAX_RANK).
spear_status check_grouped_shape(int64_t M, int64_t N, int64_t K, int64_t group, int32_t rank);

// Token count from which the tensor-core kernel replaces the weight-streaming kernel, and the
// largest compensator rank it takes (one 128-row EC tile per token block).
constexpr int64_t TC05_MIN_M = 128;
constexpr int32_t TC05_MAX_RANK = 128;
bool use_tc05(int64_t M, int32_t rank) { return M >= TC05_MIN_M && rank <= TC05_MAX_RANK; }

spear_status check_grouped_shape(int64_t M, int64_t N, int64_t K, int64_t group, int32_t rank) {
    spear_status st = check_shape(M, N, K, rank);
    if (st != SPEAR_OK) return st;
    if (group <= 0 || group % 128 != 0 || K % group != 0) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    if (rank > TC05_MAX_RANK) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    return SPEAR_OK;
}

spear_status validate_plan(const spear_plan& p, int64_t M, int64_t N, int64_t K, int32_t rank) {
    if (p.kernel_id == SPEAR_KERNEL_STREAM_RK) {
        if ((p.flags & ~(SPEAR_PLAN_DEEP_RING | SPEAR_PLAN_W4_TILES)) || !(p.flags & SPEAR_PLAN_W4_TILES))
            return SPEAR_ERR_INVALID_ARG;
        if (N % 128 != 0 || K % 128 != 0) return SPEAR_ERR_INVALID_ARG;
        if (p.tile_n != 128 || !(p.tile_m == 8 || p.tile_m == 16 || p.tile_m == 32 || p.tile_m == 64) || M > p.tile_m)
            return SPEAR_ERR_INVALID_ARG;
        if (!(p.split_k == 128 || p.split_k == 256) || K % p.split_k != 0) return SPEAR_ERR_INVALID_ARG;
        StreamArgs a = {};
        a.M = M > 0 ? M : 1;
        a.N = N;
        a.K = K;
        a.rank = rank;
        a.grid = stream_grid(N, K, p.split_k, device_sms(-1), (p.flags & SPEAR_PLAN_DEEP_RING) != 0);
        if (!stream_rk_configure(a, p.tile_m, p.split_k, (p.flags & SPEAR_PLAN_DEEP_RING) != 0)) return SPEAR_ERR_INVALID_ARG;
        return SPEAR_OK;
    }
    if (p.kernel_id == SPEAR_KERNEL_STREAM) {
        if (p.flags & ~SPEAR_PLAN_DEEP_RING) return SPEAR_ERR_INVALID_ARG;
        if (p.tile_n != 128 || !(p.tile_m == 16 || p.tile_m == 32 || p.tile_m == 64) || M > p.tile_m)
            return SPEAR_ERR_INVALID_ARG;
        if (!(p.split_k == 128 || p.split_k == 256) || K % p.split_k != 0) return SPEAR_ERR_INVALID_ARG;
        // The tiling must fit the ring mode's shared memory and TMEM (checked as the launch will).
        StreamArgs a = {};
        a.M = M > 0 ? M : 1;
        a.N = N;
        a.K = K;
        a.rank = rank;
        a.grid = stream_grid(N, K, p.split_k, device_sms(-1), (p.flags & SPEAR_PLAN_DEEP_RING) != 0);
        if (!stream_configure(a, p.tile_m, p.split_k, (p.flags & SPEAR_PLAN_DEEP_RING) != 0)) return SPEAR_ERR_INVALID_ARG;
        return SPEAR_OK;
    }
    if (p.kernel_id == SPEAR_KERNEL_TC05) {
        if (rank > TC05_MAX_RANK || (p.flags & ~SPEAR_PLAN_SEPARATE_EC)) return SPEAR_ERR_INVALID_ARG;
        if ((M + p.tile_m - 1) / p.tile_m > (int64_t)TC_BLOCKS_MAX) return SPEAR_ERR_INVALID_ARG;
        if (!(p.tile_m == 128 || p.tile_m == 160 || p.tile_m == 192 || p.tile_m == 256)) return SPEAR_ERR_INVALID_ARG;
        // 128 weight rows per tile, or 256 (two sub-tiles sharing x) with 128 tokens.
        if (!(p.tile_n == 128 || (p.tile_n == 256 && p.tile_m == 128 && N % 256 == 0))) return SPEAR_ERR_INVALID_ARG;
        // K split over a cluster of split_k CTAs (fused compensator only).
        if (!tc05_split_supported(p.tile_m, p.tile_n, p.split_k, K)) return SPEAR_ERR_INVALID_ARG;
        if (p.split_k > 1 && (p.flags & SPEAR_PLAN_SEPARATE_EC)) return SPEAR_ERR_INVALID_ARG;
        return SPEAR_OK;
    }
    if (p.kernel_id != SPEAR_KERNEL_SPLITK) return SPEAR_ERR_INVALID_ARG;
    if (p.flags & ~SPEAR_PLAN_SEPARATE_EC) return SPEAR_ERR_INVALID_ARG;
    if (!(p.split_k == 1 || p.split_k == 2 || p.split_k == 4 || p.split_k == 8)) return SPEAR_ERR_INVALID_ARG;
    const int nb = nb_for_tile_m(p.tile_m);
    if (p.tile_m != 8 * nb) return SPEAR_ERR_INVALID_ARG;
    if (p.tile_n % 16 != 0 || p.tile_n <= 0) return SPEAR_ERR_INVALID_ARG;
    const int g = p.tile_n / 16;
    const int64_t ksl = k_slice_for(K, p.split_k);
    if ((p.split_k - 1) * ksl >= K) return SPEAR_ERR_INVALID_ARG;
    if (!decode_config_supported(nb, g, wpw_for(ksl))) return SPEAR_ERR_INVALID_ARG;
    if (N % p.tile_n != 0) return SPEAR_ERR_INVALID_ARG;
    // Consumer counters: at most GROUPS_MAX groups of GEMM CTAs per token chunk.
    if ((N / p.tile_n) * p.split_k > (int64_t)GROUPS_MAX * CONSUMER_GROUP) return SPEAR_ERR_INVALID_ARG;
    return SPEAR_OK;
}

// The split-K decode kernel over launches of at most LAUNCH_TOKENS_MAX tokens.  group > 0: scale
// and zero [N][K / group] with K slices of k_slice codes (a multiple of 128); else per-channel.
spear_status run_decode(const spear_plan& p, const void* x, int64_t M, int64_t N, int64_t K, const void* packed,
                        const void* scale, const void* zero, const spear_ec* ec, void* y, spear_dtype y_dtype,
                        unsigned char* ws, int64_t group, int64_t k_slice, cudaStream_t s) {
    const int32_t rank = ec ? ec->rank : 0;
    unsigned* ctrl = (unsigned*)ws;
    const int nb = nb_for_tile_m(p.tile_m);
    const int g = p.tile_n / 16;

    DecodeArgs a;
    a.packed = (const uint8_t*)packed;
    a.scale = (const __half*)scale;
    a.zero = (const __half*)zero;
    a.A = ec ? (const uint16_t*)ec->A : nullptr;
    a.B = ec ? (const uint16_t*)ec->B : nullptr;
    a.wg = ec ? (const uint16_t*)ec->w_g : nullptr;
    a.b_g = ec ? ec->b_g : 0.0f;
    a.mlp = gate_mlp_of(ec);
    a.rank = rank;
    a.y_fp32 = (y_dtype == SPEAR_FP32);
    a.N = N;
    a.K = K;
    a.k_slice = group > 0 ? k_slice : k_slice_for(K, p.split_k);
    a.group = group;
    a.split = p.split_k;
    a.ec_jr = ec_jr_for(rank, p.split_k);
    a.ec_splits = decode_ec_ctas_per_chunk(K, rank);
    a.row_tiles = (int)(N / p.tile_n);
    a.tacc = (long long*)(ws + CTRL_BYTES);
    a.err = ctrl;
    a.arrivals = ctrl + CTRL_HEADER_WORDS;
    a.consumed = a.arrivals + CHUNKS_MAX;
    a.consumed1 = a.consumed + CHUNKS_MAX;
    const bool separate = rank > 0 && (p.flags & SPEAR_PLAN_SEPARATE_EC);
    a.ymain = separate ? (float*)(ws + ZEROED_BYTES) : nullptr;
    const size_t ysz = y_dtype == SPEAR_FP32 ? 4 : 2;
    // Launches of at most LAUNCH_TOKENS_MAX tokens, in token order on one stream.
    for (int64_t m0 = 0; m0 < M; m0 += LAUNCH_TOKENS_MAX) {
        const int64_t ml = (M - m0) < LAUNCH_TOKENS_MAX ? (M - m0) : LAUNCH_TOKENS_MAX;
        a.x = (const uint16_t*)x + m0 * K;
        a.y = (unsigned char*)y + (size_t)m0 * N * ysz;
        a.M = ml;
        a.mchunks = (int)((ml + p.tile_m - 1) / p.tile_m);
        const int e = a.ec_splits * a.mchunks;
        a.ec_ctas = (e + p.split_k - 1) / p.split_k * p.split_k;
        if (launch_decode(a, nb, g, wpw_for(a.k_slice), s) != cudaSuccess) return SPEAR_ERR_CUDA;
        if (separate && launch_apply(a, s) != cudaSuccess) return SPEAR_ERR_CUDA;
    }
    return SPEAR_OK;
}

}  // namespace

namespace spear {
// A fused split-K decode plan (SPEAR_KERNEL_SPLITK, no separate EC pass): the measured table's
// entry for this shape when it is one, else the cost model.  Used where only that kernel can run.
spear_status plan_split_k_decode(int64_t M, int64_t N, int64_t K, int32_t rank, spear_plan* out) {
    spear_status st = check_shape(M, N, K, rank);
    if (st != SPEAR_OK) return st;
    const int sms = device_sms(-1);
    spear_plan p = {};
    if (!lookup_measured(M, N, K, rank, sms, &p) || p.kernel_id != SPEAR_KERNEL_SPLITK ||
        (p.flags & SPEAR_PLAN_SEPARATE_EC)) {
        st = plan_decode_rules(M, N, K, rank, sms, &p);
        if (st != SPEAR_OK) return st;
    }
    p.workspace_bytes = workspace_bytes_for(p, M, N, K, rank, sms);
    *out = p;
    return SPEAR_OK;
}
}  // namespace spear

extern "C" {

const char* spear_status_string(spear_status status) {
    switch (status) {
        case SPEAR_OK: return "ok";
        case SPEAR_ERR_INVALID_ARG: return "invalid argument";
        case SPEAR_ERR_UNSUPPORTED_SHAPE: return "unsupported shape (need N % 128 == 0, K % 64 == 0, rank 0 or 16..256 step 16, M <= 65536)";
        case SPEAR_ERR_MISALIGNED: return "device pointer not 16-byte aligned";
        case SPEAR_ERR_WORKSPACE_TOO_SMALL: return "workspace smaller than plan.workspace_bytes";
        case SPEAR_ERR_CUDA: return "CUDA runtime or launch error";
        case SPEAR_ERR_TIMEOUT: return "a bounded in-kernel wait timed out";
    }
    return "unknown status";
}

int spear_version(void) { return 100; }

spear_status spear_pack_w4(const void* W, spear_dtype w_dtype, int64_t N, int64_t K, void* packed, void* scale,
                           void* zero, void* stream) {
    if (!W || !packed || !scale || !zero) return SPEAR_ERR_INVALID_ARG;
    if (w_dtype != SPEAR_BF16 && w_dtype != SPEAR_FP32) return SPEAR_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0) return SPEAR_ERR_INVALID_ARG;
    if (K % 2 != 0) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(W) || !aligned16(packed) || !aligned16(scale) || !aligned16(zero)) return SPEAR_ERR_MISALIGNED;
    cudaError_t e = launch_pack_w4(W, w_dtype == SPEAR_BF16, N, K, packed, scale, zero, (cudaStream_t)stream);
    return e == cudaSuccess ? SPEAR_OK : SPEAR_ERR_CUDA;
}

spear_status spear_debug_unpack_w4(const void* packed, const void* zero, int64_t N, int64_t K, void* q_out,
                                   void* qz_out, void* stream) {
    if (!packed || !zero || (!q_out && !qz_out)) return SPEAR_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0) return SPEAR_ERR_INVALID_ARG;
    if (K % 2 != 0) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(packed) || !aligned16(zero) || (q_out && !aligned16(q_out)) || (qz_out && !aligned16(qz_out)))
        return SPEAR_ERR_MISALIGNED;
    cudaError_t e = launch_unpack_w4(packed, zero, N, K, q_out, qz_out, (cudaStream_t)stream);
    return e == cudaSuccess ? SPEAR_OK : SPEAR_ERR_CUDA;
}

spear_status spear_gemm_plan(int64_t M, int64_t N, int64_t K, int32_t rank, int device, spear_plan* out) {
    if (!out) return SPEAR_ERR_INVALID_ARG;
    spear_status st = check_shape(M, N, K, rank);
    if (st != SPEAR_OK) return st;
    const int sms = device_sms(device);
    spear_plan p = {};
    // A measured plan for this shape (either kernel) first, then the rules.
    if (lookup_measured(M > 0 ? M : 1, N, K, rank, sms, &p)) st = SPEAR_OK;
    else if (use_tc05(M, rank)) st = plan_tc05(M, N, sms, &p);
    else st = plan_decode(M > 0 ? M : 1, N, K, rank, sms, &p);
    if (st != SPEAR_OK) return st;
    p.workspace_bytes = workspace_bytes_for(p, M, N, K, rank, sms);
    *out = p;
    return SPEAR_OK;
}

spear_status spear_gemm_plan_tiled(int64_t M, int64_t N, int64_t K, int32_t rank, int device, spear_plan* out) {
    if (!out) return SPEAR_ERR_INVALID_ARG;
    spear_status st = check_shape(M, N, K, rank);
    if (st != SPEAR_OK) return st;
    if (M > 64 || N % 128 != 0 || K % 128 != 0 || rank > 128) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    const int sms = device_sms(device);
    const int64_t m = M > 0 ? M : 1;
    spear_plan p = {};
    if (!lookup_measured(m, N, K, rank, sms, &p, true)) {
        // Rules: the smallest token tile that holds M, 256-code stages where K allows, the deep
        // ring for 64 tokens (the only ring with their registers), else the two-per-SM ring.
        p.kernel_id = SPEAR_KERNEL_STREAM_RK;
        p.tile_n = 128;
        p.tile_m = m <= 8 ? 8 : (m <= 16 ? 16 : (m <= 32 ? 32 : 64));
        p.split_k = (K % 256 == 0 && p.tile_m <= 16) ? 256 : 128;   // 32+ tokens: registers for 128
        p.flags = SPEAR_PLAN_W4_TILES | (p.tile_m == 64 ? SPEAR_PLAN_DEEP_RING : 0);
        p.reserved = 0;
        if (validate_plan(p, m, N, K, rank) != SPEAR_OK) {
            p.split_k = 128;
            if (K % 128 != 0 || validate_plan(p, m, N, K, rank) != SPEAR_OK) return SPEAR_ERR_UNSUPPORTED_SHAPE;
        }
    }
    p.workspace_bytes = workspace_bytes_for(p, M, N, K, rank, sms);
    *out = p;
    return SPEAR_OK;
}

spear_status spear_gemm_plan_formats(int64_t M, int64_t N, int64_t K, int32_t rank, int device, int32_t formats,
                                    spear_plan* out) {
    if (!out || formats <= 0 || (formats & ~(SPEAR_W4_ROWS | SPEAR_W4_TILES))) return SPEAR_ERR_INVALID_ARG;
    if (!(formats & SPEAR_W4_TILES)) return spear_gemm_plan(M, N, K, rank, device, out);
    if (!(formats & SPEAR_W4_ROWS)) return spear_gemm_plan_tiled(M, N, K, rank, device, out);
    spear_status st = check_shape(M, N, K, rank);
    if (st != SPEAR_OK) return st;
    // Both orders at hand: the tile order where this shape was measured faster with it.
    const int sms = device_sms(device);
    const int64_t m = M > 0 ? M : 1;
    spear_plan rows = {}, tiles = {};
    double us_rows = 0.0, us_tiles = 0.0;
    const bool have_rows = lookup_measured(m, N, K, rank, sms, &rows, false, &us_rows);
    const bool have_tiles = M <= 64 && lookup_measured(m, N, K, rank, sms, &tiles, true, &us_tiles);
    if (have_tiles && (!have_rows || us_tiles < us_rows)) return spear_gemm_plan_tiled(M, N, K, rank, device, out);
    return spear_gemm_plan(M, N, K, rank, device, out);
}

spear_status spear_tile_w4(const void* packed, int64_t N, int64_t K, void* tiled, void* stream) {
    if (!packed || !tiled) return SPEAR_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0) return SPEAR_ERR_INVALID_ARG;
    if (N % 128 != 0 || K % 128 != 0) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(packed) || !aligned16(tiled)) return SPEAR_ERR_MISALIGNED;
    const uintptr_t a0 = (uintptr_t)packed, b0 = (uintptr_t)tiled, bytes = (uintptr_t)(N * K / 2);
    if (a0 < b0 + bytes && b0 < a0 + bytes) return SPEAR_ERR_INVALID_ARG;   // overlapping buffers
    cudaError_t e = launch_tile_w4(packed, N, K, tiled, (cudaStream_t)stream);
    return e == cudaSuccess ? SPEAR_OK : SPEAR_ERR_CUDA;
}

spear_status spear_plan_update(spear_plan* plan, int64_t M, int64_t N, int64_t K, int32_t rank) {
    if (!plan) return SPEAR_ERR_INVALID_ARG;
    spear_status st = check_shape(M, N, K, rank);
    if (st != SPEAR_OK) return st;
    st = validate_plan(*plan, M, N, K, rank);
    if (st != SPEAR_OK) return st;
    plan->workspace_bytes = workspace_bytes_for(*plan, M, N, K, rank, device_sms(-1));
    return SPEAR_OK;
}

spear_status spear_w4ec_gemm(const spear_plan* plan, const void* x, int64_t M, int64_t N, int64_t K,
                             const void* packed, const void* scale, const void* zero, const spear_ec* ec, void* y,
                             spear_dtype y_dtype, void* workspace, size_t workspace_bytes, void* stream) {
    // An empty batch may come with NULL activation/output pointers (M = 0 launches nothing).
    if (!packed || !scale || !zero || !workspace) return SPEAR_ERR_INVALID_ARG;
    if (M != 0 && (!x || !y)) return SPEAR_ERR_INVALID_ARG;
    if (y_dtype != SPEAR_BF16 && y_dtype != SPEAR_FP32) return SPEAR_ERR_INVALID_ARG;
    const int32_t rank = ec ? ec->rank : 0;
    if (ec && (!ec->A || !ec->B || !ec->w_g)) return SPEAR_ERR_INVALID_ARG;
    if (ec && isnan(ec->b_g)) return SPEAR_ERR_INVALID_ARG;
    spear_status st = check_shape(M, N, K, rank);
    if (st != SPEAR_OK) return st;
    if (ec && rank == 0) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    if ((M != 0 && (!aligned16(x) || !aligned16(y))) || !aligned16(packed) || !aligned16(scale) ||
        !aligned16(zero) || !aligned16(workspace))
        return SPEAR_ERR_MISALIGNED;
    if (ec && (!aligned16(ec->A) || !aligned16(ec->B) || !aligned16(ec->w_g))) return SPEAR_ERR_MISALIGNED;
    st = check_gate_mlp(ec);
    if (st != SPEAR_OK) return st;
    if (M == 0) return SPEAR_OK;

    const int sms = device_sms(-1);
    const bool mlp_gate = ec && ec->gate_w1;
    spear_plan p;
    if (plan) {
        p = *plan;
        if (mlp_gate && (p.kernel_id == SPEAR_KERNEL_STREAM || p.kernel_id == SPEAR_KERNEL_STREAM_RK))
            return SPEAR_ERR_INVALID_ARG;   // scalar gate only
    } else {
        if (lookup_measured(M, N, K, rank, sms, &p)) st = SPEAR_OK;
        else if (use_tc05(M, rank)) st = plan_tc05(M, N, sms, &p);
        else st = plan_decode(M, N, K, rank, sms, &p);
        if (st != SPEAR_OK) return st;
        // The stream kernel takes the scalar gate only: the bottleneck-MLP gate runs on the
        // split-K decode kernel.
        if (mlp_gate && (p.kernel_id == SPEAR_KERNEL_STREAM || p.kernel_id == SPEAR_KERNEL_STREAM_RK))
            st = plan_decode_rules(M, N, K, rank, sms, &p);
        if (st != SPEAR_OK) return st;
    }
    st = validate_plan(p, M, N, K, rank);
    if (st != SPEAR_OK) return st;
    if (workspace_bytes < workspace_bytes_for(p, M, N, K, rank, sms)) return SPEAR_ERR_WORKSPACE_TOO_SMALL;

    cudaStream_t s = (cudaStream_t)stream;
    unsigned char* ws = (unsigned char*)workspace;
    unsigned* ctrl = (unsigned*)ws;
    if (p.kernel_id == SPEAR_KERNEL_TC05) {
        TcArgs t;
        t.x = (const uint16_t*)x;
        t.packed = (const uint8_t*)packed;
        t.scale = (const __half*)scale;
        t.zero = (const __half*)zero;
        t.A = ec ? (const uint16_t*)ec->A : nullptr;
        t.B = ec ? (const uint16_t*)ec->B : nullptr;
        t.wg = ec ? (const uint16_t*)ec->w_g : nullptr;
        t.b_g = ec ? ec->b_g : 0.0f;
        t.mlp = gate_mlp_of(ec);
        t.rank = rank;
        t.u = rank > 0 ? (__nv_bfloat16*)(ws + ZEROED_BYTES) : nullptr;
        t.y = y;
        t.y_fp32 = (y_dtype == SPEAR_FP32);
        t.M = M;
        t.N = N;
        t.K = K;
        t.err = ctrl;
        t.ec_ready = ctrl + TC_FLAGS_WORD;
        t.ec_consumed = t.ec_ready + TC_BLOCKS_MAX;
        t.ec_only = 0;
        cudaError_t e;
        if (rank > 0 && (p.flags & SPEAR_PLAN_SEPARATE_EC))
            e = launch_semifused(t, p.tile_m, p.tile_n, (float*)(ws + ZEROED_BYTES + tc05_u_bytes(M, rank)), s);
        else
            e = launch_tc05(t, p.tile_m, p.tile_n, s, true, 0, p.split_k);
        return e == cudaSuccess ? SPEAR_OK : SPEAR_ERR_CUDA;
    }
    if (p.kernel_id == SPEAR_KERNEL_STREAM || p.kernel_id == SPEAR_KERNEL_STREAM_RK) {
        const bool rk = p.kernel_id == SPEAR_KERNEL_STREAM_RK;
        StreamArgs a = {};
        a.x = (const uint16_t*)x;
        a.packed = (const uint8_t*)packed;
        a.scale = (const __half*)scale;
        a.zero = (const __half*)zero;
        a.A = ec ? (const uint16_t*)ec->A : nullptr;
        a.B = ec ? (const uint16_t*)ec->B : nullptr;
        a.wg = ec ? (const uint16_t*)ec->w_g : nullptr;
        a.b_g = ec ? ec->b_g : 0.0f;
        a.rank = rank;
        a.y = y;
        a.y_fp32 = (y_dtype == SPEAR_FP32);
        a.M = M;
        a.N = N;
        a.K = K;
        const bool deep = (p.flags & SPEAR_PLAN_DEEP_RING) != 0;
        a.grid = stream_grid(N, K, p.split_k, sms, deep);
        if (!(rk ? stream_rk_configure(a, p.tile_m, p.split_k, deep) : stream_configure(a, p.tile_m, p.split_k, deep)))
            return SPEAR_ERR_INVALID_ARG;
        a.tacc = (long long*)(ws + CTRL_BYTES);
        a.err = ctrl;
        a.flags = ctrl + STREAM_FLAGS_WORD;
        a.ec_readers = ctrl + STREAM_FLAGS_WORD + STREAM_GRID_MAX;
        a.partial = (float*)(ws + ZEROED_BYTES);
        const cudaError_t e = rk ? launch_stream_rk(a, p.tile_m, s) : launch_stream(a, p.tile_m, s);
        return e == cudaSuccess ? SPEAR_OK : SPEAR_ERR_CUDA;
    }
    return run_decode(p, x, M, N, K, packed, scale, zero, ec, y, y_dtype, ws, 0, 0, s);
}

spear_status spear_pack_w4_grouped(const void* W, spear_dtype w_dtype, int64_t N, int64_t K, int64_t group,
                                   void* packed, void* scale, void* zero, void* stream) {
    if (!W || !packed || !scale || !zero) return SPEAR_ERR_INVALID_ARG;
    if (w_dtype != SPEAR_BF16 && w_dtype != SPEAR_FP32) return SPEAR_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0 || group <= 0) return SPEAR_ERR_INVALID_ARG;
    if (group % 2 != 0 || K % group != 0) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(W) || !aligned16(packed) || !aligned16(scale) || !aligned16(zero)) return SPEAR_ERR_MISALIGNED;
    // Each group is quantised as a row of its own: the per-channel packer over W viewed as
    // [N * K / group, group], whose outputs are laid out as [N, K/2] and [N, K/group].
    cudaError_t e = launch_pack_w4(W, w_dtype == SPEAR_BF16, N * (K / group), group, packed, scale, zero,
                                   (cudaStream_t)stream);
    return e == cudaSuccess ? SPEAR_OK : SPEAR_ERR_CUDA;
}

spear_status spear_grouped_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t group, int32_t rank,
                                           size_t* out) {
    if (!out) return SPEAR_ERR_INVALID_ARG;
    spear_status st = check_grouped_shape(M, N, K, group, rank);
    if (st != SPEAR_OK) return st;
    size_t b = ZEROED_BYTES;
    if (rank > 0) b += tc05_u_bytes(M, rank) + (size_t)M * N * 4;     // u, then the fp32 main term
    *out = b;
    return SPEAR_OK;
}

spear_status spear_w4ec_gemm_grouped(const void* x, int64_t M, int64_t N, int64_t K, int64_t group,
                                     const void* packed, const void* scale, const void* zero, const spear_ec* ec,
                                     void* y, spear_dtype y_dtype, void* workspace, size_t workspace_bytes,
                                     void* stream) {
    if (!packed || !scale || !zero || !workspace) return SPEAR_ERR_INVALID_ARG;
    if (M != 0 && (!x || !y)) return SPEAR_ERR_INVALID_ARG;
    if (y_dtype != SPEAR_BF16 && y_dtype != SPEAR_FP32) return SPEAR_ERR_INVALID_ARG;
    const int32_t rank = ec ? ec->rank : 0;
    if (ec && (!ec->A || !ec->B || !ec->w_g)) return SPEAR_ERR_INVALID_ARG;
    if (ec && isnan(ec->b_g)) return SPEAR_ERR_INVALID_ARG;
    if (ec && rank == 0) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    spear_status st = check_grouped_shape(M, N, K, group, rank);
    if (st != SPEAR_OK) return st;
    if ((M != 0 && (!aligned16(x) || !aligned16(y))) || !aligned16(packed) || !aligned16(scale) ||
        !aligned16(zero) || !aligned16(workspace))
        return SPEAR_ERR_MISALIGNED;
    if (ec && (!aligned16(ec->A) || !aligned16(ec->B) || !aligned16(ec->w_g))) return SPEAR_ERR_MISALIGNED;
    st = check_gate_mlp(ec);
    if (st != SPEAR_OK) return st;
    size_t need = 0;
    spear_grouped_workspace_bytes(M, N, K, group, rank, &need);
    if (workspace_bytes < need) return SPEAR_ERR_WORKSPACE_TOO_SMALL;
    if (M == 0) return SPEAR_OK;

    cudaStream_t s = (cudaStream_t)stream;
    unsigned char* ws = (unsigned char*)workspace;
    GroupedArgs ga;
    ga.x = (const uint16_t*)x;
    ga.packed = (const uint8_t*)packed;
    ga.scale = (const __half*)scale;
    ga.zero = (const __half*)zero;
    ga.M = M;
    ga.N = N;
    ga.K = K;
    ga.group = group;
    ga.y = y;
    ga.y_fp32 = (y_dtype == SPEAR_FP32);
    ga.ymain = nullptr;
    // Decode batches: the fused decode kernel with the group scale applied per 128-code window,
    // its K slices rounded to whole windows; otherwise the grouped kernel (below).
    if (M <= LAUNCH_TOKENS_MAX) {
        spear_plan p;
        const int sms = device_sms(-1);
        if (!lookup_measured(M, N, K, rank > 0 ? 1 : 0, sms, &p) || p.kernel_id != SPEAR_KERNEL_SPLITK)
            st = plan_decode(M, N, K, rank, sms, &p);
        if (st == SPEAR_OK && p.kernel_id == SPEAR_KERNEL_SPLITK) {
            p.flags = 0;
            for (; p.split_k >= 1; p.split_k /= 2) {
                const int64_t ksl = (K + p.split_k - 1) / p.split_k;
                const int64_t k_slice = (ksl + 127) / 128 * 128;
                if ((p.split_k - 1) * k_slice >= K) continue;
                if (!decode_config_supported(nb_for_tile_m(p.tile_m), p.tile_n / 16, wpw_for(k_slice))) continue;
                return run_decode(p, x, M, N, K, packed, scale, zero, ec, y, y_dtype, ws, group, k_slice, s);
            }
        }
    }
    if (rank == 0) return launch_w4g_gemm(ga, s) == cudaSuccess ? SPEAR_OK : SPEAR_ERR_CUDA;

    // The compensator beside the grouped GEMM, as on the semi-fused prefill path.
    unsigned* ctrl = (unsigned*)ws;
    TcArgs t;
    t.x = (const uint16_t*)x;
    t.packed = (const uint8_t*)packed;
    t.scale = (const __half*)scale;
    t.zero = (const __half*)zero;
    t.A = (const uint16_t*)ec->A;
    t.B = (const uint16_t*)ec->B;
    t.wg = (const uint16_t*)ec->w_g;
    t.b_g = ec->b_g;
    t.mlp = gate_mlp_of(ec);
    t.rank = rank;
    t.u = (__nv_bfloat16*)(ws + ZEROED_BYTES);
    t.y = y;
    t.y_fp32 = (y_dtype == SPEAR_FP32);
    t.M = M;
    t.N = N;
    t.K = K;
    t.err = ctrl;
    t.ec_ready = ctrl + TC_FLAGS_WORD;
    t.ec_consumed = t.ec_ready + TC_BLOCKS_MAX;
    t.ec_only = 0;
    ga.ymain = (float*)(ws + ZEROED_BYTES + tc05_u_bytes(M, rank));
    auto grouped_main = [](const void* ctx, cudaStream_t st) { return launch_w4g_gemm(*(const GroupedArgs*)ctx, st); };
    return launch_ec_beside(t, grouped_main, &ga, ga.ymain, s) == cudaSuccess ? SPEAR_OK : SPEAR_ERR_CUDA;
}

spear_status spear_get_device_status(void* workspace, int clear, void* stream) {
    if (!workspace) return SPEAR_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return SPEAR_ERR_MISALIGNED;
    unsigned word = 0;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return SPEAR_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SPEAR_ERR_CUDA;
    if (clear && word != 0) {
        if (cudaMemsetAsync(workspace, 0, sizeof(word), s) != cudaSuccess) return SPEAR_ERR_CUDA;
        if (cudaStreamSynchronize(s) != cudaSuccess) return SPEAR_ERR_CUDA;
    }
    return word == 0 ? SPEAR_OK : SPEAR_ERR_TIMEOUT;
}

}  // extern "C"
