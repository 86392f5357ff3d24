// semifused.cu -- the semi-fused prefill path: the compensator as kernels of its own beside the GEMM.
//
// SPEAR technical summary, section 2.2A: at prefill a compensator fused into the GEMM's epilogue
// competes with the GEMM for the SMs, so the pages' second form runs the compensator as a separate
// kernel that overlaps the GEMM, the two tied together in a static CUDA-graph DAG so that no CPU
// launch sits between them.  One call enqueues a fork and a join:
//
//   side stream (the library's, highest priority)   tcgen05 kernel, EC tiles alone:   u = g t, bf16 [M][r]
//   caller's stream                                 tcgen05 kernel, main tiles alone: ymain = s[n] D, fp32 [M][N]
//   caller's stream, after both                     ec_up_add_kernel:                 y = ymain + u B
//
// When the caller captures its stream into a CUDA graph, the first two launches become parallel
// branches and the third joins them.  launch_ec_beside is the fork/join with any main-term launch;
// the group-wise-scale layer (grouped.cu) uses it too.  The arithmetic is the fused path's (the same bf16 u, the same
// fp32 main term); only the last sum takes two fp32 roundings (s[n] D, then + u B) where the fused
// epilogue takes one multiply-add, before the single rounding to y's type.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace spear {

constexpr int UA_BM = 64;                // tokens per CTA
constexpr int UA_BN = 128;               // output columns per CTA
constexpr int UA_THREADS = 256;          // 8 warps: 4 (tokens) x 2 (columns), 16 x 64 each
constexpr int UA_BPAD = UA_BN + 8;       // smem row stride of B: rows start 4 banks apart
constexpr int UA_RANK_MAX = 128;         // the EC tiles' largest rank

SPEAR_DEVI void ldsm_x4(uint32_t r[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"((uint32_t)__cvta_generic_to_shared(p)));
}
SPEAR_DEVI void ldsm_x4_trans(uint32_t r[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"((uint32_t)__cvta_generic_to_shared(p)));
}

static size_t up_add_smem_bytes(int r) { return ((size_t)UA_BM * (r + 8) + (size_t)r * UA_BPAD) * 2; }

// y[m, n] = ymain[m, n] + sum_j u[m, j] B[j, n] for a 64-token x 128-column tile.  u rows and the
// B slice are staged in shared memory (u rows past M as zeros); each warp runs m16n8k16 MMAs with
// both operands fetched by ldmatrix (B transposed on the fly from its [r, N] rows).
__global__ void __launch_bounds__(UA_THREADS) ec_up_add_kernel(const uint16_t* __restrict__ u,
                                                                const uint16_t* __restrict__ B,
                                                                const float* __restrict__ ymain, void* __restrict__ y,
                                                                int y_fp32, int64_t M, int64_t N, int r) {
    extern __shared__ __align__(16) unsigned char ua_smem[];
    const int upad = r + 8;                              // u row stride: rows start 4 banks apart
    uint16_t* us = reinterpret_cast<uint16_t*>(ua_smem); // [UA_BM][r + 8]
    uint16_t* bs = us + UA_BM * upad;                    // [r][UA_BN + 8]
    const int64_t m0 = (int64_t)blockIdx.y * UA_BM;
    const int64_t n0 = (int64_t)blockIdx.x * UA_BN;
    const int tid = threadIdx.x;

    const int upr = r / 8;                               // 16-byte pieces per u row
    for (int i = tid; i < UA_BM * upr; i += UA_THREADS) {
        const int mm = i / upr, c = i - mm * upr;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (m0 + mm < M) v = ldg_u4(u + (m0 + mm) * r + c * 8);
        *reinterpret_cast<uint4*>(us + mm * upad + c * 8) = v;
    }
    constexpr int BPR = UA_BN / 8;                       // 16-byte pieces per B row slice
    for (int i = tid; i < r * BPR; i += UA_THREADS) {
        const int j = i / BPR, c = i - j * BPR;
        *reinterpret_cast<uint4*>(bs + j * UA_BPAD + c * 8) = ldg_u4(B + (int64_t)j * N + n0 + c * 8);
    }
    __syncthreads();

    const int warp = tid >> 5, lane = tid & 31;
    const int wm = warp & 3, wn = warp >> 2;
    // ldmatrix x4: lanes 8i .. 8i+7 give the rows of matrix i; matrices 0, 1 are rows 0-7 and 8-15
    // of the first 8 columns, matrices 2, 3 the same rows of the next 8.
    const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8, lcol = (lane >> 4) * 8;
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;
    for (int k0 = 0; k0 < r; k0 += 16) {
        uint32_t a[4];
        ldsm_x4(a, us + (wm * 16 + lrow) * upad + k0 + lcol);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
            uint32_t b[4];                               // b[0], b[1]: columns +0..7; b[2], b[3]: +8..15
            ldsm_x4_trans(b, bs + (k0 + lrow) * UA_BPAD + wn * 64 + np * 16 + lcol);
            mma_bf16_16816(acc[2 * np], a, b[0], b[1]);
            mma_bf16_16816(acc[2 * np + 1], a, b[2], b[3]);
        }
    }
    // Accumulator of an n8 tile: [0], [1] at token g, columns 2q, 2q + 1; [2], [3] at token g + 8.
    const int g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int64_t m = m0 + wm * 16 + g + h * 8;
        if (m >= M) continue;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const int64_t o = m * N + n0 + wn * 64 + nt * 8 + 2 * q;
            const float2 ym = __ldcs(reinterpret_cast<const float2*>(ymain + o));
            const float v0 = ym.x + acc[nt][2 * h], v1 = ym.y + acc[nt][2 * h + 1];
            if (y_fp32)
                *reinterpret_cast<float2*>(reinterpret_cast<float*>(y) + o) = make_float2(v0, v1);
            else
                *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(y) + o) =
                    __floats2bfloat162_rn(v0, v1);
        }
    }
}

static cudaError_t launch_ec_up_add(const TcArgs& a, const float* ymain, cudaStream_t stream) {
    if (a.rank < 16 || a.rank > UA_RANK_MAX || a.rank % 16 != 0 || a.N % UA_BN != 0) return cudaErrorInvalidValue;
    static std::once_flag once[kMaxDevices];
    static cudaError_t opt_status[kMaxDevices];
    cudaError_t e = opt_in_smem((const void*)ec_up_add_kernel, up_add_smem_bytes(UA_RANK_MAX), once, opt_status);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)(a.N / UA_BN), (unsigned)((a.M + UA_BM - 1) / UA_BM));
    cudaGetLastError();   // report this launch only, not an earlier call's error
    ec_up_add_kernel<<<grid, UA_THREADS, up_add_smem_bytes(a.rank), stream>>>(
        reinterpret_cast<const uint16_t*>(a.u), a.B, ymain, a.y, a.y_fp32, a.M, a.N, a.rank);
    return cudaGetLastError();
}

// One side stream and a fork/join pair of events per device, created on first use.  The mutex
// covers only the host-side enqueue: recording an event and the wait that reads it must not
// interleave with another thread's record of the same event.
struct SideLane {
    std::mutex mu;
    bool ready = false;
    cudaStream_t stream = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    int priority = 0;
};
constexpr int SIDE_DEVICES = 64;
static SideLane g_lanes[SIDE_DEVICES];

static cudaError_t lane_init(SideLane& L) {
    // Creating a stream or an event is not stream work; with this thread's capture mode relaxed it
    // is allowed even while the caller's stream is being captured into a graph.
    cudaStreamCaptureMode mode = cudaStreamCaptureModeRelaxed;
    cudaError_t e = cudaThreadExchangeStreamCaptureMode(&mode);
    if (e != cudaSuccess) return e;
    int least = 0, greatest = 0;
    e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
    if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&L.stream, cudaStreamNonBlocking, greatest);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&L.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&L.join, cudaEventDisableTiming);
    cudaStreamCaptureMode back = mode;
    cudaThreadExchangeStreamCaptureMode(&back);
    if (e != cudaSuccess) {
        if (L.join) cudaEventDestroy(L.join);
        if (L.fork) cudaEventDestroy(L.fork);
        if (L.stream) cudaStreamDestroy(L.stream);
        L.join = L.fork = nullptr;
        L.stream = nullptr;
        return e;
    }
    L.priority = greatest;
    L.ready = true;
    return cudaSuccess;
}

cudaError_t launch_ec_beside(const TcArgs& a, MainLaunch main, const void* ctx, float* ymain, cudaStream_t stream) {
    if (a.rank <= 0 || a.u == nullptr || ymain == nullptr || main == nullptr) return cudaErrorInvalidValue;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= SIDE_DEVICES) return cudaErrorInvalidDevice;
    SideLane& L = g_lanes[dev];
    std::lock_guard<std::mutex> lock(L.mu);
    if (!L.ready && (e = lane_init(L)) != cudaSuccess) return e;

    TcArgs ec = a;                        // EC tiles alone: u = g t
    ec.ec_only = 1;
    ec.y = nullptr;
    ec.y_fp32 = 1;

    // Fork: the side stream starts after all the work already in the caller's stream (the previous
    // call's join read u).  Once forked, the join is always recorded and waited for, so that a
    // stream capture stays joined whatever fails in between.
    if ((e = cudaEventRecord(L.fork, stream)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(L.stream, L.fork, 0)) != cudaSuccess) return e;
    cudaError_t first = launch_tc05(ec, 128, 128, L.stream, false, L.priority);
    e = cudaEventRecord(L.join, L.stream);
    if (e != cudaSuccess) return first != cudaSuccess ? first : e;
    const cudaError_t m = main(ctx, stream);
    if (first == cudaSuccess) first = m;
    e = cudaStreamWaitEvent(stream, L.join, 0);
    if (first == cudaSuccess) first = e;
    if (first != cudaSuccess) return first;
    return launch_ec_up_add(a, ymain, stream);
}

}  // namespace spear

namespace spear {

// The semi-fused prefill path: the tcgen05 kernel's main tiles alone write the main term.
struct Tc05Main {
    TcArgs a;
    int bn, rows;
};
static cudaError_t tc05_main(const void* ctx, cudaStream_t stream) {
    const Tc05Main* c = static_cast<const Tc05Main*>(ctx);
    return launch_tc05(c->a, c->bn, c->rows, stream, false, 0);
}

cudaError_t launch_semifused(const TcArgs& a, int bn, int rows, float* ymain, cudaStream_t stream) {
    Tc05Main c;
    c.a = a;                              // main tiles alone, no compensator: ymain = s[n] D
    c.a.rank = 0;
    c.a.A = c.a.B = c.a.wg = nullptr;
    c.a.u = nullptr;
    c.a.mlp = GateMlp{};
    c.a.y = ymain;
    c.a.y_fp32 = 1;
    c.a.ec_only = 0;
    c.bn = bn;
    c.rows = rows;
    return launch_ec_beside(a, tc05_main, &c, ymain, stream);
}

}  // namespace spear
