// splitk.cu -- decode-phase kernels: the EC pre-pass and the split-K weight-streaming W4 GEMM.
//
// SPEAR (Post-Quantization Error-Adaptive Recovery), technical summary section 2.2A: decode is
// memory-bound, so the cost to beat is the time to stream the packed weights once.  Here the EC
// runs as its own small kernel (t = x A, gate, u = g t), overlapped with the weight stream by
// programmatic dependent launch, and u B is added in the GEMM's split-K reduction epilogue:
//
//   y[m,n] = s[n] * sum_k x[m,k] (q[n,k] - z[n]) + sum_j u[m,j] B[j,n],   u = g t
//
// Weight-streaming kernel layout (one CTA = 4 warps):
//   * the CTA owns RT = 16*G weight rows, a K slice, and a chunk of 8*NB tokens;
//   * warp w takes 128-wide K windows w, w+4, ... of the slice; inside a window, lane
//     (g = lane/4, t = lane%4) loads 16 bytes (32 codes) of rows g and g+8 of every 16-row
//     group straight from HBM into registers: no shared-memory staging of weights;
//   * codes become exact bf16 (q - z) in registers and feed mma.sync m16n8k16 with the weights as
//     the M=16 operand and the tokens as N=8 ("swap AB"); the K order inside each MMA is permuted
//     (pairs k, k+4), and x is loaded with the same permutation, which leaves the dot product
//     unchanged;
//   * the four warps' partial sums meet in shared memory in a fixed order; K slices meet in the
//     workspace, where the last CTA of a tile (atomic ticket, no spinning) sums the slices in
//     slice order, applies s[n], adds the EC term and rounds once to bf16.
// No floating-point atomics: results are deterministic for a given plan.
#include "common.cuh"
#include "kernels.h"

namespace spear {

// ---------------------------------------------------------------------------------------------
// EC pre-pass: partial t = x A and gate pre-activation over a K chunk, then the last CTA of a
// token chunk finishes u = sigmoid(p) * t.
// ---------------------------------------------------------------------------------------------
constexpr int EC_KC = 64;   // K rows of A staged per step
constexpr int EC_TM = 16;   // tokens per CTA
constexpr int EC_THREADS = 256;
constexpr int EC_OUT_PER_THREAD = (EC_TM * 257 + EC_THREADS - 1) / EC_THREADS;  // rank <= 256

__global__ void __launch_bounds__(EC_THREADS) ec_prepass_kernel(EcPrepassArgs a) {
    // Let the dependent GEMM start streaming weights right away; it waits for this grid only
    // before reading u.
    pdl_launch_dependents();
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float* xs = reinterpret_cast<float*>(smem_raw);            // [EC_TM][EC_KC]
    float* As = xs + EC_TM * EC_KC;                            // [EC_KC][r + 1] (col r = w_g)
    __shared__ unsigned s_last;
    __shared__ float s_gate[EC_TM];

    const int r = a.rank, r1 = a.rank + 1;
    const int64_t kbeg = (int64_t)blockIdx.x * a.k_per_cta;
    const int64_t kend = imin64(kbeg + a.k_per_cta, a.K);
    const int64_t m0 = (int64_t)blockIdx.y * EC_TM;
    const int tm = (int)imin64(EC_TM, a.M - m0);

    float acc[EC_OUT_PER_THREAD];
#pragma unroll
    for (int q = 0; q < EC_OUT_PER_THREAD; ++q) acc[q] = 0.0f;

    for (int64_t k0 = kbeg; k0 < kend; k0 += EC_KC) {
        const int kc = (int)imin64(EC_KC, kend - k0);
        __syncthreads();
        for (int i = threadIdx.x; i < EC_TM * EC_KC; i += EC_THREADS) {
            const int m = i / EC_KC, k = i % EC_KC;
            xs[i] = (m < tm && k < kc) ? bf16_bits_to_f32(a.x[(m0 + m) * a.K + k0 + k]) : 0.0f;
        }
        for (int i = threadIdx.x; i < EC_KC * r1; i += EC_THREADS) {
            const int k = i / r1, j = i % r1;
            float v = 0.0f;
            if (k < kc) v = (j < r) ? bf16_bits_to_f32(a.A[(k0 + k) * r + j]) : bf16_bits_to_f32(a.wg[k0 + k]);
            As[i] = v;
        }
        __syncthreads();
#pragma unroll
        for (int q = 0; q < EC_OUT_PER_THREAD; ++q) {
            const int o = threadIdx.x + q * EC_THREADS;
            if (o < tm * r1) {
                const int m = o / r1, j = o % r1;
                float v = acc[q];
#pragma unroll 8
                for (int k = 0; k < EC_KC; ++k) v = fmaf(xs[m * EC_KC + k], As[k * r1 + j], v);
                acc[q] = v;
            }
        }
    }

    float* part = a.ec_part + (int64_t)blockIdx.x * a.M * r1;   // [S][M][r+1]
#pragma unroll
    for (int q = 0; q < EC_OUT_PER_THREAD; ++q) {
        const int o = threadIdx.x + q * EC_THREADS;
        if (o < tm * r1) part[(m0 + o / r1) * r1 + o % r1] = acc[q];
    }

    // The last CTA along K for this token chunk sums the slices in slice order.
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned prev = atomicAdd(&a.tickets[blockIdx.y], 1u);
        s_last = (prev == gridDim.x - 1) ? 1u : 0u;
        if (s_last) a.tickets[blockIdx.y] = 0u;  // every slice has arrived: re-arm for the next call
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if ((int)threadIdx.x < tm) {
        const int m = threadIdx.x;
        float p = 0.0f;
        for (unsigned s = 0; s < gridDim.x; ++s) p += __ldcg(a.ec_part + ((int64_t)s * a.M + m0 + m) * r1 + r);
        p += a.b_g;
        s_gate[m] = 1.0f / (1.0f + expf(-p));
    }
    __syncthreads();
    for (int o = threadIdx.x; o < tm * r; o += EC_THREADS) {
        const int m = o / r, j = o % r;
        float t = 0.0f;
        for (unsigned s = 0; s < gridDim.x; ++s) t += __ldcg(a.ec_part + ((int64_t)s * a.M + m0 + m) * r1 + j);
        a.u[(m0 + m) * r + j] = s_gate[m] * t;
    }
}

int64_t ec_prepass_token_chunks(int64_t M) { return (M + EC_TM - 1) / EC_TM; }

// K rows per CTA: enough CTAs to cover the SMs about twice, in whole EC_KC steps.
int64_t ec_prepass_k_per_cta(int64_t M, int64_t K, int num_sms) {
    const int64_t steps = (K + EC_KC - 1) / EC_KC;
    int64_t want = (2 * (int64_t)num_sms) / ec_prepass_token_chunks(M);
    want = want < 1 ? 1 : (want > steps ? steps : want);
    const int64_t steps_per_cta = (steps + want - 1) / want;
    return steps_per_cta * EC_KC;
}

int64_t ec_prepass_splits(int64_t K, int64_t k_per_cta) { return (K + k_per_cta - 1) / k_per_cta; }

size_t ec_prepass_smem_bytes(int rank) { return sizeof(float) * (EC_TM * EC_KC + EC_KC * (rank + 1)); }
size_t ec_prepass_max_smem_bytes() { return ec_prepass_smem_bytes(256); }

cudaError_t launch_ec_prepass(const EcPrepassArgs& a, cudaStream_t stream) {
    const dim3 grid((unsigned)ec_prepass_splits(a.K, a.k_per_cta), (unsigned)ec_prepass_token_chunks(a.M));
    ec_prepass_kernel<<<grid, EC_THREADS, ec_prepass_smem_bytes(a.rank), stream>>>(a);
    return cudaGetLastError();
}

const void* ec_prepass_kernel_ptr() { return (const void*)ec_prepass_kernel; }

// ---------------------------------------------------------------------------------------------
// Split-K weight-streaming GEMM.
// ---------------------------------------------------------------------------------------------
constexpr int SK_WARPS = 4;
constexpr int SK_WIN = 128;   // K per warp window

template <int NB, int G>
__global__ void __launch_bounds__(SK_WARPS * 32) splitk_w4_kernel(SplitKArgs a) {
    constexpr int RT = 16 * G;        // weight rows per CTA
    constexpr int TM = 8 * NB;        // tokens per CTA
    __shared__ float red[SK_WARPS][RT][TM + 1];
    __shared__ unsigned s_last;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t n0 = (int64_t)blockIdx.x * RT;
    const int ks = blockIdx.y;
    const int64_t m0 = (int64_t)blockIdx.z * TM;
    const int64_t kbeg = (int64_t)ks * a.k_slice;
    const int64_t kend = imin64(kbeg + a.k_slice, a.K);
    const int64_t row_bytes = a.K / 2;

    // Zero-point bias per row held by this thread (rows n0 + 16i + g and + 8).
    uint32_t zb[G][2];
#pragma unroll
    for (int i = 0; i < G; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t z = (uint32_t)__half2float(a.zero[n0 + 16 * i + g + 8 * h]);
            zb[i][h] = zero_bias_bf16x2(z);
        }

    float acc[G][NB][4];
#pragma unroll
    for (int i = 0; i < G; ++i)
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[i][b][c] = 0.0f;

    for (int64_t kwin = kbeg + (int64_t)warp * SK_WIN; kwin < kend; kwin += SK_WARPS * SK_WIN) {
        const int64_t kt = kwin + 32 * t;          // this lane's 32-code slice
        const bool active = kt < kend;

        // Weight codes: 16 bytes of rows g and g+8 of each 16-row group.
        uint4 wq[G][2];
#pragma unroll
        for (int i = 0; i < G; ++i)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (active)
                    wq[i][h] = ldg_stream_u4(a.packed + (n0 + 16 * i + g + 8 * h) * row_bytes + kt / 2);
                else
                    wq[i][h] = make_uint4(0u, 0u, 0u, 0u);
            }

        // Activations: for word w (8 codes k..k+7) the B operand pairs are (x_i, x_{i+4}).
        uint32_t xb[NB][4][4];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            const int64_t m = m0 + 8 * b + g;
            const bool ok = active && m < a.M;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (ok) v = ldg_u4(a.x + m * a.K + kt + 8 * w);
                // v.x = (x0,x1) v.y = (x2,x3) v.z = (x4,x5) v.w = (x6,x7)
                xb[b][w][0] = prmt(v.x, v.z, 0x5410u);   // (x0, x4)
                xb[b][w][1] = prmt(v.x, v.z, 0x7632u);   // (x1, x5)
                xb[b][w][2] = prmt(v.y, v.w, 0x5410u);   // (x2, x6)
                xb[b][w][3] = prmt(v.y, v.w, 0x7632u);   // (x3, x7)
            }
        }

#pragma unroll
        for (int i = 0; i < G; ++i) {
            const uint32_t wa[4] = {wq[i][0].x, wq[i][0].y, wq[i][0].z, wq[i][0].w};
            const uint32_t wb[4] = {wq[i][1].x, wq[i][1].y, wq[i][1].z, wq[i][1].w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                uint32_t ra[4], rb[4];
                cvt_w4_pairs_i_i4(wa[w], zb[i][0], ra);
                cvt_w4_pairs_i_i4(wb[w], zb[i][1], rb);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const uint32_t af[4] = {ra[2 * hh], rb[2 * hh], ra[2 * hh + 1], rb[2 * hh + 1]};
#pragma unroll
                    for (int b = 0; b < NB; ++b)
                        mma_bf16_16816(acc[i][b], af, xb[b][w][2 * hh], xb[b][w][2 * hh + 1]);
                }
            }
        }
    }

    // Cross-warp reduction (fixed order).
#pragma unroll
    for (int i = 0; i < G; ++i)
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            red[warp][16 * i + g][8 * b + 2 * t] = acc[i][b][0];
            red[warp][16 * i + g][8 * b + 2 * t + 1] = acc[i][b][1];
            red[warp][16 * i + g + 8][8 * b + 2 * t] = acc[i][b][2];
            red[warp][16 * i + g + 8][8 * b + 2 * t + 1] = acc[i][b][3];
        }
    __syncthreads();

    const int tm = (int)imin64(TM, a.M - m0);
    const int S = gridDim.y;
    if (S > 1) {
        // Publish this slice's partial sums [S][M][N] and take a ticket.
        for (int e = threadIdx.x; e < RT * TM; e += blockDim.x) {
            const int rr = e % RT, mm = e / RT;
            if (mm < tm) {
                float v = red[0][rr][mm];
#pragma unroll
                for (int w = 1; w < SK_WARPS; ++w) v += red[w][rr][mm];
                a.part[((int64_t)ks * a.M + m0 + mm) * a.N + n0 + rr] = v;
            }
        }
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) {
            unsigned* ticket = a.tickets + (int64_t)blockIdx.z * gridDim.x + blockIdx.x;
            const unsigned prev = atomicAdd(ticket, 1u);
            s_last = (prev == (unsigned)S - 1) ? 1u : 0u;
            if (s_last) *ticket = 0u;  // all slices arrived: re-arm for the next call
        }
        __syncthreads();
        if (!s_last) return;
        __threadfence();
    }

    // Epilogue (one CTA per tile): sum slices in order, scale, add the EC term, round once.
    if (a.u != nullptr) pdl_wait_primary();
    for (int e = threadIdx.x; e < RT * TM; e += blockDim.x) {
        const int rr = e % RT, mm = e / RT;
        if (mm >= tm) continue;
        const int64_t n = n0 + rr, m = m0 + mm;
        float v;
        if (S > 1) {
            v = 0.0f;
            for (int s = 0; s < S; ++s) v += __ldcg(a.part + ((int64_t)s * a.M + m) * a.N + n);
        } else {
            v = red[0][rr][mm];
#pragma unroll
            for (int w = 1; w < SK_WARPS; ++w) v += red[w][rr][mm];
        }
        float y = __half2float(a.scale[n]) * v;
        if (a.u != nullptr) {
            const float* um = a.u + m * a.rank;
            float ec = 0.0f;
            for (int j = 0; j < a.rank; ++j) ec = fmaf(__ldcg(um + j), bf16_bits_to_f32(a.B[(int64_t)j * a.N + n]), ec);
            y += ec;
        }
        if (a.y_fp32)
            reinterpret_cast<float*>(a.y)[m * a.N + n] = y;
        else
            reinterpret_cast<__nv_bfloat16*>(a.y)[m * a.N + n] = __float2bfloat16_rn(y);
    }
}

template <int NB, int G>
static cudaError_t launch_splitk_t(const SplitKArgs& a, int split, cudaStream_t stream, bool pdl) {
    const dim3 grid((unsigned)(a.N / (16 * G)), (unsigned)split, (unsigned)((a.M + 8 * NB - 1) / (8 * NB)));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(SK_WARPS * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, splitk_w4_kernel<NB, G>, a);
}

cudaError_t launch_splitk(const SplitKArgs& a, int nb, int g, int split, cudaStream_t stream, bool pdl) {
#define SPEAR_SK_CASE(NB_, G_) \
    if (nb == NB_ && g == G_) return launch_splitk_t<NB_, G_>(a, split, stream, pdl);
    SPEAR_SK_CASE(1, 1) SPEAR_SK_CASE(1, 2) SPEAR_SK_CASE(1, 4) SPEAR_SK_CASE(1, 8)
    SPEAR_SK_CASE(2, 1) SPEAR_SK_CASE(2, 2) SPEAR_SK_CASE(2, 4) SPEAR_SK_CASE(2, 8)
    SPEAR_SK_CASE(4, 1) SPEAR_SK_CASE(4, 2) SPEAR_SK_CASE(4, 4)
#undef SPEAR_SK_CASE
    return cudaErrorInvalidValue;
}

}  // namespace spear
