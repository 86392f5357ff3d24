// api.cu -- the C ABI declared in include/spear.h: argument checks, planning, workspace layout
// and kernel dispatch.  Host code only; the kernels live in pack.cu, splitk.cu and tc05.cu.
#include <math.h>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

using namespace spear;

namespace {

constexpr int MAX_DEVICES = 64;
constexpr int DEFAULT_SMS = 148;  // B200, used when no device can be queried (host-only planning)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

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

// One-time, per-device function attributes (dynamic shared memory above 48 KB).
cudaError_t ensure_attributes() {
    static std::once_flag flags[MAX_DEVICES];
    static cudaError_t results[MAX_DEVICES];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
    std::call_once(flags[dev], [dev]() {
        results[dev] = cudaFuncSetAttribute(ec_prepass_kernel_ptr(), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            (int)ec_prepass_max_smem_bytes());
    });
    return results[dev];
}

spear_status check_shape(int64_t M, int64_t N, int64_t K, int32_t rank) {
    if (M < 0 || N <= 0 || K <= 0 || rank < 0) return SPEAR_ERR_INVALID_ARG;
    if (N % 128 != 0 || K % 64 != 0) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    if (M > M_MAX) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    if (rank != 0 && (rank < 16 || rank > 256 || rank % 16 != 0)) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    return SPEAR_OK;
}

// Workspace layout for a given problem and plan.
struct Layout {
    size_t u_off = 0, ec_part_off = 0, part_off = 0, total = 0;
    int64_t ec_k_per_cta = 0, ec_splits = 0;
};

Layout layout_for(int64_t M, int64_t N, int64_t K, int32_t rank, const spear_plan& p, int sms) {
    Layout L;
    size_t off = CTRL_BYTES;
    if (rank > 0 && M > 0) {
        L.ec_k_per_cta = ec_prepass_k_per_cta(M, K, sms);
        L.ec_splits = ec_prepass_splits(K, L.ec_k_per_cta);
        L.u_off = off;
        off = align_up(off + sizeof(float) * (size_t)M * rank, 256);
        L.ec_part_off = off;
        off = align_up(off + sizeof(float) * (size_t)L.ec_splits * M * (rank + 1), 256);
    }
    if (p.split_k > 1) {
        L.part_off = off;
        off = align_up(off + sizeof(float) * (size_t)p.split_k * M * N, 256);
    }
    L.total = off;
    return L;
}

int nb_for_tile_m(int tile_m) { return tile_m <= 8 ? 1 : (tile_m <= 16 ? 2 : 4); }

spear_status plan_splitk(int64_t M, int64_t N, int64_t K, int sms, spear_plan* p) {
    const int nb = M <= 8 ? 1 : (M <= 16 ? 2 : 4);
    const int64_t tm = 8 * nb;
    const int64_t mchunks = (M + tm - 1) / tm;
    int g = 4;
    if (nb <= 2 && (N / 64) * mchunks > 4 * (int64_t)sms && N % 128 == 0) g = 8;
    const int64_t rt = 16 * g;
    const int64_t tiles = (N / rt) * mchunks;
    int64_t want = (2 * (int64_t)sms + tiles - 1) / tiles;
    int64_t smax = K / 512;
    if (smax < 1) smax = 1;
    int64_t s = want < smax ? want : smax;
    if (s < 1) s = 1;
    while (s > 1 && (K % (s * 64) != 0 || (size_t)tiles > GEMM_TICKETS_MAX)) --s;
    p->kernel_id = SPEAR_KERNEL_SPLITK;
    p->tile_n = (int32_t)rt;
    p->split_k = (int32_t)s;
    p->tile_m = (int32_t)tm;
    p->flags = 0;
    p->reserved = 0;
    return SPEAR_OK;
}

spear_status validate_plan(const spear_plan& p, int64_t M, int64_t N, int64_t K) {
    if (p.kernel_id != SPEAR_KERNEL_SPLITK) return SPEAR_ERR_INVALID_ARG;
    if (p.split_k < 1 || K % ((int64_t)p.split_k * 64) != 0) return SPEAR_ERR_INVALID_ARG;
    const int nb = nb_for_tile_m(p.tile_m);
    if (p.tile_m != 8 * nb) return SPEAR_ERR_INVALID_ARG;
    const int g = p.tile_n / 16;
    if (p.tile_n % 16 != 0 || !(g == 1 || g == 2 || g == 4 || g == 8) || (g == 8 && nb > 2))
        return SPEAR_ERR_INVALID_ARG;
    if (N % p.tile_n != 0) return SPEAR_ERR_INVALID_ARG;
    const int64_t tiles = (N / p.tile_n) * ((M + p.tile_m - 1) / p.tile_m);
    if (p.split_k > 1 && (size_t)tiles > GEMM_TICKETS_MAX) return SPEAR_ERR_INVALID_ARG;
    return SPEAR_OK;
}

}  // namespace

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
    st = plan_splitk(M > 0 ? M : 1, N, K, sms, &p);
    if (st != SPEAR_OK) return st;
    p.workspace_bytes = layout_for(M, N, K, rank, p, sms).total;
    *out = p;
    return SPEAR_OK;
}

spear_status spear_w4ec_gemm(const spear_plan* plan, const void* x, int64_t M, int64_t N, int64_t K,
                             const void* packed, const void* scale, const void* zero, const spear_ec* ec, void* y,
                             spear_dtype y_dtype, void* workspace, size_t workspace_bytes, void* stream) {
    if (!x || !packed || !scale || !zero || !y || !workspace) return SPEAR_ERR_INVALID_ARG;
    if (y_dtype != SPEAR_BF16 && y_dtype != SPEAR_FP32) return SPEAR_ERR_INVALID_ARG;
    const int32_t rank = ec ? ec->rank : 0;
    if (ec && (!ec->A || !ec->B || !ec->w_g)) return SPEAR_ERR_INVALID_ARG;
    if (ec && isnan(ec->b_g)) return SPEAR_ERR_INVALID_ARG;
    spear_status st = check_shape(M, N, K, rank);
    if (st != SPEAR_OK) return st;
    if (ec && rank == 0) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || !aligned16(packed) || !aligned16(scale) || !aligned16(zero) || !aligned16(y) ||
        !aligned16(workspace))
        return SPEAR_ERR_MISALIGNED;
    if (ec && (!aligned16(ec->A) || !aligned16(ec->B) || !aligned16(ec->w_g))) return SPEAR_ERR_MISALIGNED;
    if (M == 0) return SPEAR_OK;

    const int sms = device_sms(-1);
    spear_plan p;
    if (plan) {
        p = *plan;
    } else {
        st = plan_splitk(M, N, K, sms, &p);
        if (st != SPEAR_OK) return st;
    }
    st = validate_plan(p, M, N, K);
    if (st != SPEAR_OK) return st;
    const Layout L = layout_for(M, N, K, rank, p, sms);
    if (workspace_bytes < L.total) return SPEAR_ERR_WORKSPACE_TOO_SMALL;

    if (ensure_attributes() != cudaSuccess) return SPEAR_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned char* ws = (unsigned char*)workspace;
    unsigned* ec_tickets = (unsigned*)(ws + CTRL_HEADER_BYTES);
    unsigned* gemm_tickets = ec_tickets + EC_TICKETS_MAX;

    float* u = nullptr;
    if (ec) {
        EcPrepassArgs ea;
        ea.x = (const uint16_t*)x;
        ea.A = (const uint16_t*)ec->A;
        ea.wg = (const uint16_t*)ec->w_g;
        ea.b_g = ec->b_g;
        ea.M = M;
        ea.K = K;
        ea.rank = rank;
        ea.k_per_cta = L.ec_k_per_cta;
        ea.ec_part = (float*)(ws + L.ec_part_off);
        ea.u = (float*)(ws + L.u_off);
        ea.tickets = ec_tickets;
        if (launch_ec_prepass(ea, s) != cudaSuccess) return SPEAR_ERR_CUDA;
        u = ea.u;
    }

    SplitKArgs a;
    a.x = (const uint16_t*)x;
    a.packed = (const uint8_t*)packed;
    a.scale = (const __half*)scale;
    a.zero = (const __half*)zero;
    a.B = ec ? (const uint16_t*)ec->B : nullptr;
    a.u = u;
    a.rank = rank;
    a.y = y;
    a.y_fp32 = (y_dtype == SPEAR_FP32);
    a.M = M;
    a.N = N;
    a.K = K;
    a.k_slice = K / p.split_k;
    a.part = p.split_k > 1 ? (float*)(ws + L.part_off) : nullptr;
    a.tickets = gemm_tickets;
    cudaError_t e = launch_splitk(a, nb_for_tile_m(p.tile_m), p.tile_n / 16, p.split_k, s, ec != nullptr);
    return e == cudaSuccess ? SPEAR_OK : SPEAR_ERR_CUDA;
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
