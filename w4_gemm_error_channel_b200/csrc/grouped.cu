// grouped.cu -- the W4 GEMM with group-wise scales and zero-points (GPTQ/AWQ-style groups).
//
// SPEAR technical summary, section 3.1: the method sits on top of several quantisation backends
// (RTN, GPTQ, AWQ, OmniQuant), which keep one scale and zero-point per group of G consecutive input
// channels of a row instead of one per row.  Then the scale no longer factors out of the K sum:
//
//     y[m, n] = sum_g s[n, g] sum_{k in g} (q[n, k] - z[n, g]) x[m, k]      (+ the EC term)
//
// w4g_gemm_kernel streams the packed weights like the fused decode kernel: each lane of a warp
// takes 32 codes of a 128-code window of 16 weight rows (a 16-byte load per row), turns them into
// exact bf16 (q - z) and feeds mma.sync m16n8k16 with the weights as the 16-row operand and 8 tokens
// as the other; the activation pairs are permuted to match the order the codes leave the
// converter.  One m16n8k16 step mixes codes from all four 32-code pieces of its window, so the
// group scale can be applied once per window: G is a multiple of 128, every window lies inside one
// group, and the window's products are scaled by s[n, g] as they are added to the accumulators.
// The four warps of a CTA take every fourth window and their sums are added in a fixed order in
// shared memory (no atomics: the result is deterministic).
//
// With a compensator, the kernel writes the fp32 main term and the EC runs beside it exactly as on
// the semi-fused prefill path (launch_ec_beside): the tcgen05 kernel's EC tiles compute u = g t on a
// side stream and ec_up_add adds u B after both.
#include "common.cuh"
#include "kernels.h"

namespace spear {

constexpr int GW_WARPS = 4;
constexpr int GW_THREADS = 32 * GW_WARPS;
constexpr int GW_WIN = 128;              // K codes per warp step (4 lanes x 32 codes)

// One CTA: 16 RG weight rows x 8 NB tokens, the whole K.
template <int NB, int RG>
__global__ void __launch_bounds__(GW_THREADS) w4g_gemm_kernel(GroupedArgs a) {
    constexpr int RT = 16 * RG;
    constexpr int TM = 8 * NB;
    constexpr int RS = RT + 4;           // padded rows: the fragment stores below are conflict-free
    __shared__ __align__(16) float red[GW_WARPS][TM][RS];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t n0 = (int64_t)blockIdx.x * RT;
    const int64_t m0 = (int64_t)blockIdx.y * TM;
    const int64_t ng = a.K / a.group;
    const int64_t row_bytes = a.K / 2;
    const int nwin = (int)(a.K / GW_WIN);

    float acc[RG][NB][4];
#pragma unroll
    for (int i = 0; i < RG; ++i)
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[i][b][c] = 0.0f;

    for (int win = warp; win < nwin; win += GW_WARPS) {
        const int64_t kw = (int64_t)win * GW_WIN;
        const int64_t kt = kw + 32 * t;
        const int64_t grp = kw / a.group;
        uint4 wq[RG][2];
        uint32_t zb[RG][2];
        float sc[RG][2];
#pragma unroll
        for (int i = 0; i < RG; ++i)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int64_t row = n0 + 16 * i + g + 8 * h;
                wq[i][h] = ldg_stream_u4(a.packed + row * row_bytes + kt / 2);
                zb[i][h] = zero_bias_bf16x2((uint32_t)__half2float(a.zero[row * ng + grp]));
                sc[i][h] = __half2float(a.scale[row * ng + grp]);
            }
        // Activations: for word w (codes k..k+7) the B operand pairs are (x_i, x_{i+4}).
        uint32_t xb[NB][4][4];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            const int64_t m = m0 + 8 * b + g;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (m < a.M) v = ldg_u4(a.x + m * a.K + kt + 8 * w);
                xb[b][w][0] = prmt(v.x, v.z, 0x5410u);
                xb[b][w][1] = prmt(v.x, v.z, 0x7632u);
                xb[b][w][2] = prmt(v.y, v.w, 0x5410u);
                xb[b][w][3] = prmt(v.y, v.w, 0x7632u);
            }
        }
#pragma unroll
        for (int i = 0; i < RG; ++i) {
            float part[NB][4];
#pragma unroll
            for (int b = 0; b < NB; ++b) part[b][0] = part[b][1] = part[b][2] = part[b][3] = 0.0f;
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
                        mma_bf16_16816(part[b], af, xb[b][w][2 * hh], xb[b][w][2 * hh + 1]);
                }
            }
            // part[b]: [0], [1] at row g (tokens 2t, 2t + 1); [2], [3] at row g + 8.
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                acc[i][b][0] = fmaf(sc[i][0], part[b][0], acc[i][b][0]);
                acc[i][b][1] = fmaf(sc[i][0], part[b][1], acc[i][b][1]);
                acc[i][b][2] = fmaf(sc[i][1], part[b][2], acc[i][b][2]);
                acc[i][b][3] = fmaf(sc[i][1], part[b][3], acc[i][b][3]);
            }
        }
    }

#pragma unroll
    for (int i = 0; i < RG; ++i)
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            red[warp][8 * b + 2 * t][16 * i + g] = acc[i][b][0];
            red[warp][8 * b + 2 * t + 1][16 * i + g] = acc[i][b][1];
            red[warp][8 * b + 2 * t][16 * i + g + 8] = acc[i][b][2];
            red[warp][8 * b + 2 * t + 1][16 * i + g + 8] = acc[i][b][3];
        }
    __syncthreads();
    for (int e = threadIdx.x; e < TM * RT; e += GW_THREADS) {
        const int mm = e / RT, rr = e - mm * RT;
        const int64_t m = m0 + mm;
        if (m >= a.M) continue;
        float v = red[0][mm][rr];
#pragma unroll
        for (int w = 1; w < GW_WARPS; ++w) v += red[w][mm][rr];
        const int64_t o = m * a.N + n0 + rr;
        if (a.ymain)
            a.ymain[o] = v;
        else if (a.y_fp32)
            reinterpret_cast<float*>(a.y)[o] = v;
        else
            reinterpret_cast<__nv_bfloat16*>(a.y)[o] = __float2bfloat16_rn(v);
    }
}

template <int NB, int RG>
static cudaError_t launch_w4g_t(const GroupedArgs& a, cudaStream_t stream) {
    const dim3 grid((unsigned)(a.N / (16 * RG)), (unsigned)((a.M + 8 * NB - 1) / (8 * NB)));
    cudaGetLastError();   // report this launch only, not an earlier call's error
    w4g_gemm_kernel<NB, RG><<<grid, GW_THREADS, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_w4g_gemm(const GroupedArgs& a, cudaStream_t stream) {
    if (a.M <= 0) return cudaSuccess;
    if (a.group <= 0 || a.group % GW_WIN != 0 || a.K % a.group != 0 || a.N % 32 != 0) return cudaErrorInvalidValue;
    // Tokens per CTA: the smallest of 8, 16, 32 that holds the batch (more token chunks re-read the
    // weights from L2); 32 weight rows per CTA once 16-row tiles would exceed four CTAs per SM.
    const bool wide = a.N >= 16 * 4 * 148;
    if (a.M <= 8) return wide ? launch_w4g_t<1, 2>(a, stream) : launch_w4g_t<1, 1>(a, stream);
    if (a.M <= 16) return wide ? launch_w4g_t<2, 2>(a, stream) : launch_w4g_t<2, 1>(a, stream);
    return wide ? launch_w4g_t<4, 2>(a, stream) : launch_w4g_t<4, 1>(a, stream);
}

}  // namespace spear
