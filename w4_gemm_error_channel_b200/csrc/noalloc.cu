// noalloc.cu -- spear_w4ec_gemm_noalloc: the decode-phase layer without a caller workspace.
//
// The fused decode kernel needs a little device scratch: an error word, per-token-chunk counters
// and the int64 compensator accumulators.  spear_w4ec_gemm takes that scratch from the caller's
// workspace.  This entry point keeps it instead in one file-scope device array, so a caller that
// cannot allocate device memory can still run the layer.  Each device that loads this library
// holds the array for the life of its context.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace spear {

// Scratch layout: control words in the first NOALLOC_CTRL_BYTES (same word layout as the workspace
// control block), then the accumulators, int64 [M][r + 1].
constexpr size_t NOALLOC_SCRATCH_BYTES = 256 * 1024;
constexpr size_t NOALLOC_CTRL_BYTES = 64 * 1024;
constexpr int64_t NOALLOC_M_MAX = 64;
static_assert(CTRL_HEADER_WORDS + 2 * CHUNKS_MAX + CHUNKS_MAX * GROUPS_MAX <= NOALLOC_CTRL_BYTES / 4,
              "control words must fit");
static_assert(NOALLOC_CTRL_BYTES + (size_t)NOALLOC_M_MAX * 257 * 8 <= NOALLOC_SCRATCH_BYTES,
              "accumulators for the largest batch and rank must fit");

static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int MAX_DEVICES = 64;

// Device address of the scratch on the current device, looked up once per device.  In host code
// g_noalloc_scratch names a host-side stand-in, never a device address.
cudaError_t scratch_address(unsigned char** out) {
    static std::once_flag once[MAX_DEVICES];
    static cudaError_t status[MAX_DEVICES];
    static unsigned char* addr[MAX_DEVICES];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [dev]() {
        void* p = nullptr;
        status[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        addr[dev] = static_cast<unsigned char*>(p);
    });
    *out = addr[dev];
    return status[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int nb_of(int tile_m) { return tile_m <= 8 ? 1 : (tile_m <= 16 ? 2 : 4); }
int64_t k_slice_of(int64_t K, int64_t S) { return ((K + S - 1) / S + 63) / 64 * 64; }
int wpw_of(int64_t k_slice) { return (int)((k_slice + 511) / 512); }

}  // namespace
}  // namespace spear

using namespace spear;

extern "C" spear_status spear_w4ec_gemm_noalloc(const spear_plan* plan, const void* x, int64_t M, int64_t N,
                                                int64_t K, const void* packed, const void* scale, const void* zero,
                                                const spear_ec* ec, void* y, spear_dtype y_dtype, void* stream) {
    if (!x || !packed || !scale || !zero || !y) return SPEAR_ERR_INVALID_ARG;
    if (y_dtype != SPEAR_BF16 && y_dtype != SPEAR_FP32) return SPEAR_ERR_INVALID_ARG;
    const int32_t rank = ec ? ec->rank : 0;
    if (ec && (!ec->A || !ec->B || !ec->w_g || isnan(ec->b_g))) return SPEAR_ERR_INVALID_ARG;
    if (ec && ec->gate_w1) return SPEAR_ERR_INVALID_ARG;   // the scalar gate only here
    if (M <= 0 || N <= 0 || K <= 0) return SPEAR_ERR_INVALID_ARG;
    if (M > NOALLOC_M_MAX) return SPEAR_ERR_UNSUPPORTED_SHAPE;       // the scratch is sized for 64 tokens
    if (N % 128 != 0 || K % 64 != 0) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    if (ec && (rank < 16 || rank > 256 || rank % 16 != 0 || K > EC_K_MAX)) return SPEAR_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || !aligned16(packed) || !aligned16(scale) || !aligned16(zero) || !aligned16(y))
        return SPEAR_ERR_MISALIGNED;
    if (ec && (!aligned16(ec->A) || !aligned16(ec->B) || !aligned16(ec->w_g))) return SPEAR_ERR_MISALIGNED;

    // Without a plan, the split-K decode kernel's own plan for this shape (the dispatcher may
    // prefer another kernel, which needs a workspace).
    spear_plan p;
    if (plan) {
        p = *plan;
    } else {
        const spear_status st = plan_split_k_decode(M, N, K, rank, &p);
        if (st != SPEAR_OK) return st;
    }
    // Only the weight-streaming decode kernel runs here.
    if (p.kernel_id != SPEAR_KERNEL_SPLITK || p.flags != 0) return SPEAR_ERR_INVALID_ARG;
    if (!(p.split_k == 1 || p.split_k == 2 || p.split_k == 4 || p.split_k == 8)) return SPEAR_ERR_INVALID_ARG;
    const int nb = nb_of(p.tile_m);
    if (p.tile_m != 8 * nb || p.tile_n <= 0 || p.tile_n % 16 != 0 || N % p.tile_n != 0) return SPEAR_ERR_INVALID_ARG;
    const int64_t ksl = k_slice_of(K, p.split_k);
    if ((p.split_k - 1) * ksl >= K || !decode_config_supported(nb, p.tile_n / 16, wpw_of(ksl)))
        return SPEAR_ERR_INVALID_ARG;
    if ((N / p.tile_n) * p.split_k > (int64_t)GROUPS_MAX * CONSUMER_GROUP) return SPEAR_ERR_INVALID_ARG;

    unsigned char* scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess || scratch == nullptr) return SPEAR_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    // The array starts zeroed and every completed call leaves its counters and accumulators
    // zeroed again, so nothing is cleared here (a clear would also sit between the previous
    // kernel and this one and stop their overlap).  After a call that stopped on a timed-out
    // wait, spear_noalloc_get_device_status(clear = 1) zeroes the array.

    unsigned* ctrl = reinterpret_cast<unsigned*>(scratch);
    DecodeArgs a;
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
    a.k_slice = ksl;
    a.split = p.split_k;
    a.ec_jr = rank > 0 ? (int)(((rank + p.split_k - 1) / p.split_k + 3) / 4 * 4) : 0;
    a.ec_splits = decode_ec_ctas_per_chunk(K, rank);
    a.row_tiles = (int)(N / p.tile_n);
    a.mchunks = (int)((M + p.tile_m - 1) / p.tile_m);
    a.ec_ctas = (a.ec_splits * a.mchunks + p.split_k - 1) / p.split_k * p.split_k;
    a.tacc = reinterpret_cast<long long*>(scratch + NOALLOC_CTRL_BYTES);
    a.err = ctrl;
    a.arrivals = ctrl + CTRL_HEADER_WORDS;
    a.consumed = a.arrivals + CHUNKS_MAX;
    a.consumed1 = a.consumed + CHUNKS_MAX;
    a.ymain = nullptr;                                    // the compensator stays fused here
    a.mlp = GateMlp{};                                    // the scalar gate
    a.group = 0;                                          // per-channel scales
    return launch_decode(a, nb, p.tile_n / 16, wpw_of(ksl), s) == cudaSuccess ? SPEAR_OK : SPEAR_ERR_CUDA;
}

extern "C" spear_status spear_noalloc_get_device_status(int clear, void* stream) {
    unsigned char* scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess || scratch == nullptr) return SPEAR_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned word = 0;
    if (cudaMemcpyAsync(&word, scratch, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess) return SPEAR_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SPEAR_ERR_CUDA;
    if (clear && word != 0) {
        // A call that gave up may have left counters and accumulators set: zero the whole array.
        if (cudaMemsetAsync(scratch, 0, NOALLOC_SCRATCH_BYTES, s) != cudaSuccess) return SPEAR_ERR_CUDA;
        if (cudaStreamSynchronize(s) != cudaSuccess) return SPEAR_ERR_CUDA;
    }
    return word == 0 ? SPEAR_OK : SPEAR_ERR_TIMEOUT;
}
