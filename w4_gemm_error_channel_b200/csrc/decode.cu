// decode.cu -- the fused decode kernel: W4 weight streaming + per-token-gated EC in one launch.
//
// SPEAR (Post-Quantization Error-Adaptive Recovery), technical summary section 2.2A: in the
// memory-bound decode phase the compensator is fused into the low-bit GEMM so that the whole
// compensation path is one kernel.  The layer is
//
//   y[m,n] = s[n] * sum_k x[m,k] (q[n,k] - z[n])  +  sum_j u[m,j] B[j,n],
//   u[m,j] = g[m] t[m,j],  t = x A,  g = sigmoid(x w_g + b_g).
//
// One grid, two kinds of CTA (128 threads each):
//   * EC CTAs (the lowest block indices, so they are dispatched first) each take one 16-column
//     group of A (or the gate vector) over 512 rows and compute, on the tensor cores, the partial
//     sums of t (or of the gate pre-activation) for their token chunk.  They add them into the
//     chunk's int64 fixed-point accumulators (2^-32 resolution; integer addition is exact, so the
//     sum does not depend on arrival order).  The low 8 bits of every word count the K slices
//     added so far, so the word itself says when it is complete: no separate flag is published;
//   * GEMM CTAs own 16*G weight rows, a K slice of at most 512*WPW codes and 8*NB tokens.  Every
//     weight byte of the CTA is requested from HBM first (registers), then the kernel waits for
//     its predecessor in the stream (programmatic dependent launch) before reading x.  Lane
//     (g = lane/4, t = lane%4) of warp w holds 16 bytes (32 codes) of rows g and g+8 of each
//     16-row group for the 128-wide K windows w, w+4, ...; codes become exact bf16 (q - z) in
//     registers and feed mma.sync m16n8k16 with the weights as the M=16 operand and the tokens as
//     N=8.  Inside each MMA the K order is permuted to pairs (k, k+4), and x is loaded with the
//     same permutation, which leaves the dot product unchanged;
//   * the four warps meet in shared memory in a fixed order and each unit (4 rows of one token)
//     gets its main term s[n] * acc.  Each GEMM CTA then reads the accumulator words of its share
//     (r/S columns) of the EC term until they are complete (a bounded wait), forms
//     u = sigmoid(p + b_g) t and adds u B (the B slice was prefetched with cp.async at the
//     start).  The S K slices of a row tile form one thread-block cluster: every rank pushes each
//     unit to the rank that owns it in distributed shared memory, and after one cluster barrier
//     the owner sums the unit over ranks 0..S-1 in rank order and rounds once to bf16.
// No floating-point atomics: results are deterministic for a given plan.  The last GEMM CTA of a
// token chunk to read the accumulators clears them, so the zeroed part of the workspace is zero
// again after every call.
#include "common.cuh"
#include "kernels.h"

namespace spear {

constexpr int DK_WARPS = 4;
constexpr int DK_THREADS = DK_WARPS * 32;
constexpr int DK_WIN = 128;            // K codes per warp window
constexpr unsigned SPIN_LIMIT = 1u << 21;

// ---------------------------------------------------------------------------------------------
// Small helpers
// ---------------------------------------------------------------------------------------------
SPEAR_DEVI void cp_async_16(void* smem, const void* gmem) {
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}

SPEAR_DEVI unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// ---------------------------------------------------------------------------------------------
// EC role: one EC CTA computes, on the tensor cores, the partial sums over 512 rows of A (a "K
// slice") of one 16-column group of t = x A, or of the gate pre-activation p = x w_g.  Tokens
// are the M=16 operand of mma.sync m16n8k16 and columns of A are N.  The 16 columns of group P
// form two n8 tiles, "even" (columns 16P + 2i) and "odd" (16P + 2i + 1), so that one 32-bit load
// of A (two adjacent columns of one row) feeds both tiles; the gate group is one n8 tile whose
// column 0 is w_g.  Warp w takes rows 128 w .. 128 w + 127 of the slice, with its fragments of A
// in registers (requested before the wait on the previous kernel); the warps meet in shared
// memory and the CTA adds its sums into the int64 fixed-point accumulators, so each accumulator
// receives one addition per K slice.
// ---------------------------------------------------------------------------------------------
constexpr int EC_KR = 512;                   // rows of A per EC CTA
constexpr int EC_KK = EC_KR / DK_WARPS / 16; // k16 steps per warp
constexpr int EC_RS = 20;                    // padded row of the cross-warp buffer (16 columns)
constexpr float FIX_ONE = 4294967296.0f;     // 2^32: fixed-point resolution 2^-32
// Each accumulator word holds (sum << 8) + (number of K slices added so far): every addition adds
// its fixed-point value shifted left by 8 plus one, so a reader knows from the word alone when
// all slices are in.  That leaves 55 bits for the signed sum: |t| and |p| stay below 2^23.
constexpr int FIX_COUNT_BITS = 8;
constexpr unsigned long long FIX_COUNT_MASK = (1ull << FIX_COUNT_BITS) - 1;
constexpr float FIX_TOTAL = 8388608.0f;      // 2^23

// K slices of the compensator, each adding once into every accumulator word.
__host__ __device__ inline int ec_slices(int64_t K) { return (int)((K + EC_KR - 1) / EC_KR); }

// EC CTAs per token chunk: one per (K slice, column group), the gate group included.
int decode_ec_ctas_per_chunk(int64_t K, int rank) {
    return rank > 0 ? (int)((K + EC_KR - 1) / EC_KR) * (rank / 16 + 1) : 0;
}

// Signed fixed-point values added as two's-complement 64-bit integers (exact, order-free).
SPEAR_DEVI void red_add_s64(long long* p, long long v) {
    asm volatile("red.relaxed.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"((unsigned long long)v) : "memory");
}

SPEAR_DEVI long long ld_relaxed_s64(const long long* p) {
    long long v;
    asm volatile("ld.relaxed.gpu.global.s64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

SPEAR_DEVI uint32_t ldg_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

template <int TM>
SPEAR_DEVI void ec_role(const DecodeArgs& a, int s, int chunk, unsigned char* dyn) {
    constexpr int MT = (TM + 15) / 16;       // m16 token tiles
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
    const int r = a.rank, NG = r / 16;
    const int P = s % (NG + 1), slice = s / (NG + 1);
    const bool gate = P == NG;
    const int64_t kw = (int64_t)slice * EC_KR + 16 * EC_KK * warp;   // this warp's first row
    const int64_t m0 = (int64_t)chunk * TM;
    const int tm = (int)imin64(TM, a.M - m0);

    // Raw words of A (or w_g): rows kw + 16 kk + 2q + {0, 1, 8, 9}, two adjacent columns each.
    // Every load is issued here, unconditionally (a step past the end of A re-reads its first
    // rows and is zeroed below), so that all of them are in flight before the wait.
    uint32_t wv[EC_KK][4];
#pragma unroll
    for (int kk = 0; kk < EC_KK; ++kk) {
        const int64_t row = (kw + 16 * kk < a.K ? kw + 16 * kk : 0) + 2 * q;
        if (!gate) {
            const uint16_t* p = a.A + row * r + 16 * P + 2 * g;
            wv[kk][0] = ldg_u32(p);
            wv[kk][1] = ldg_u32(p + r);
            wv[kk][2] = ldg_u32(p + 8 * r);
            wv[kk][3] = ldg_u32(p + 9 * r);
        } else {
            wv[kk][0] = ldg_u32(a.wg + row);
            wv[kk][1] = ldg_u32(a.wg + row + 8);
            wv[kk][2] = wv[kk][3] = 0u;
        }
    }

    // x may be the previous kernel's output; the previous call may still use the workspace.
    pdl_wait_primary();
    // Keep every use of the words below the wait, so that the x loads are not held up behind them.
#pragma unroll
    for (int kk = 0; kk < EC_KK; ++kk)
        asm volatile("" : "+r"(wv[kk][0]), "+r"(wv[kk][1]), "+r"(wv[kk][2]), "+r"(wv[kk][3]));

    // x fragments of all token tiles: every load in flight before the first use.
    uint32_t xa[MT][EC_KK][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int t0 = 16 * mt + g, t1 = t0 + 8;
#pragma unroll
        for (int kk = 0; kk < EC_KK; ++kk) {
            const int64_t k = kw + 16 * kk + 2 * q;
            const bool in = kw + 16 * kk < a.K;
            xa[mt][kk][0] = (in && t0 < tm) ? ldg_u32(a.x + (m0 + t0) * a.K + k) : 0u;
            xa[mt][kk][1] = (in && t1 < tm) ? ldg_u32(a.x + (m0 + t1) * a.K + k) : 0u;
            xa[mt][kk][2] = (in && t0 < tm) ? ldg_u32(a.x + (m0 + t0) * a.K + k + 8) : 0u;
            xa[mt][kk][3] = (in && t1 < tm) ? ldg_u32(a.x + (m0 + t1) * a.K + k + 8) : 0u;
        }
    }

    // B fragments: [kk][0..1] the even tile, [kk][2..3] the odd tile; the gate tile has w_g in
    // column 0 (lanes g == 0).  K is a multiple of 64, so a k16 step lies wholly inside or outside.
    uint32_t b[EC_KK][4];
#pragma unroll
    for (int kk = 0; kk < EC_KK; ++kk) {
        const bool in = kw + 16 * kk < a.K;
        if (!gate) {
            b[kk][0] = in ? prmt(wv[kk][0], wv[kk][1], 0x5410u) : 0u;
            b[kk][1] = in ? prmt(wv[kk][2], wv[kk][3], 0x5410u) : 0u;
            b[kk][2] = in ? prmt(wv[kk][0], wv[kk][1], 0x7632u) : 0u;
            b[kk][3] = in ? prmt(wv[kk][2], wv[kk][3], 0x7632u) : 0u;
        } else {
            b[kk][0] = (in && g == 0) ? wv[kk][0] : 0u;
            b[kk][1] = (in && g == 0) ? wv[kk][1] : 0u;
            b[kk][2] = b[kk][3] = 0u;
        }
    }

    // Lane (g, q) ends with columns 4q + {0, 1, 2, 3} of the group for tokens 16 mt + g and + 8.
    float* red_ec = reinterpret_cast<float*>(dyn);      // [DK_WARPS][TM][EC_RS]
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int t0 = 16 * mt + g, t1 = t0 + 8;
        float de[4] = {0.f, 0.f, 0.f, 0.f}, dod[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < EC_KK; ++kk) {
            mma_bf16_16816(de, xa[mt][kk], b[kk][0], b[kk][1]);
            if (!gate) mma_bf16_16816(dod, xa[mt][kk], b[kk][2], b[kk][3]);
        }
        if (t0 < TM)
            *reinterpret_cast<float4*>(red_ec + (warp * TM + t0) * EC_RS + 4 * q) = make_float4(de[0], dod[0], de[1], dod[1]);
        if (t1 < TM)
            *reinterpret_cast<float4*>(red_ec + (warp * TM + t1) * EC_RS + 4 * q) = make_float4(de[2], dod[2], de[3], dod[3]);
    }
    __syncthreads();

    // Cross-warp sums (fixed order), then exact integer accumulation across K slices.  Each slice
    // is held to its share of the 2^23 bound on |t| and |p|.
    const float lim = FIX_TOTAL / (float)ec_slices(a.K);
    long long* tc = a.tacc + (int64_t)chunk * TM * (r + 1);
    const int ncol = gate ? 1 : 16;
    for (int o = threadIdx.x; o < tm * ncol; o += DK_THREADS) {
        const int m = o / ncol, c = o % ncol;
        float v = red_ec[m * EC_RS + c];
#pragma unroll
        for (int w = 1; w < DK_WARPS; ++w) v += red_ec[(w * TM + m) * EC_RS + c];
        if (!(fabsf(v) < lim)) {
            atomicOr(a.err, 2u);
            v = 0.0f;
        }
        const unsigned long long fx = (unsigned long long)__float2ll_rn(v * FIX_ONE);
        red_add_s64(tc + (int64_t)m * (r + 1) + (gate ? r : 16 * P + c), (long long)((fx << FIX_COUNT_BITS) | 1ull));
    }
    pdl_launch_dependents();
}

// ---------------------------------------------------------------------------------------------
// GEMM role.
// ---------------------------------------------------------------------------------------------
// GROUPED: scale and zero-point per (row, group of a.group codes), a.group a multiple of 128 and
// every K slice a multiple of 128, so that each 128-code window lies inside one group: the window's
// products are scaled by s[n, group] as they are added to the accumulators, and the epilogue's
// per-row scale is 1.
template <int NB, int G, int WPW, bool GROUPED>
SPEAR_DEVI void gemm_role(const DecodeArgs& a, int tile, int ks, int chunk, unsigned char* dyn) {
    constexpr int RT = 16 * G;        // weight rows per CTA
    constexpr int TM = 8 * NB;        // tokens per CTA
    constexpr int RT4 = RT / 4;
    constexpr int RS = RT + 4;        // padded row: the fragment stores below are conflict-free
    __shared__ __align__(16) float red[DK_WARPS][TM][RS];
    // K slices pushed here by the cluster's ranks: [rank][this CTA's share of the tile].
    __shared__ __align__(16) float4 recv[TM * RT4];
    __shared__ float s_scale[RT];
    __shared__ unsigned s_flag;
    uint16_t* Bs = reinterpret_cast<uint16_t*>(dyn);                           // [ec_jr][RT] bf16
    float* us = reinterpret_cast<float*>(dyn + (size_t)a.ec_jr * RT * 2);      // [TM][ec_jr + 1]
    float* mlp_t = us + TM * (a.ec_jr + 1);                                    // MLP gate: [TM][r + 1] t
    float* mlp_h = mlp_t + TM * (a.rank + 1);                                  //           [TM][H + 1] hidden

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t n0 = (int64_t)tile * RT;
    const int S = a.split;
    const int64_t m0 = (int64_t)chunk * TM;
    const int64_t kbeg = (int64_t)ks * a.k_slice;
    const int64_t kend = imin64(kbeg + a.k_slice, a.K);
    const int64_t row_bytes = a.K / 2;
    // With a separate EC pass the CTA writes its fp32 main term to the workspace and leaves the
    // compensator to the apply kernel.
    const bool has_ec = a.rank > 0 && a.ymain == nullptr;
    const int j0 = ks * a.ec_jr;
    const int nj = has_ec ? max(0, min(a.rank, j0 + a.ec_jr) - j0) : 0;

    if (S > 1) cluster_arrive_relaxed();

    // ---- Prologue: only inputs that no earlier kernel in the stream can be writing. ----
    if (nj > 0) {
        constexpr int CH = RT / 8;     // 16-byte pieces per B row slice
        for (int c = threadIdx.x; c < nj * CH; c += DK_THREADS) {
            const int jj = c / CH, cc = c % CH;
            cp_async_16(Bs + jj * RT + cc * 8, a.B + (int64_t)(j0 + jj) * a.N + n0 + cc * 8);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    for (int i = threadIdx.x; i < RT; i += DK_THREADS) s_scale[i] = GROUPED ? 1.0f : __half2float(a.scale[n0 + i]);
    uint32_t zb[G][2];
    if (!GROUPED) {
#pragma unroll
        for (int i = 0; i < G; ++i)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                zb[i][h] = zero_bias_bf16x2((uint32_t)__half2float(a.zero[n0 + 16 * i + g + 8 * h]));
    }
    const int64_t ngroups = GROUPED ? a.K / a.group : 1;
    // Unconditional loads (a lane past the slice end re-reads the slice start) keep every request
    // in flight before the wait below; such lanes feed zero activations instead.
    uint4 wq[WPW][G][2];
#pragma unroll
    for (int w8 = 0; w8 < WPW; ++w8) {
        int64_t kt = kbeg + (int64_t)(warp + DK_WARPS * w8) * DK_WIN + 32 * t;
        kt = kt < kend ? kt : kbeg;
#pragma unroll
        for (int i = 0; i < G; ++i)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                wq[w8][i][h] = ldg_stream_u4(a.packed + (n0 + 16 * i + g + 8 * h) * row_bytes + kt / 2);
    }

    pdl_wait_primary();

    float acc[G][NB][4];
#pragma unroll
    for (int i = 0; i < G; ++i)
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[i][b][c] = 0.0f;

#pragma unroll
    for (int w8 = 0; w8 < WPW; ++w8) {
        const int64_t kt = kbeg + (int64_t)(warp + DK_WARPS * w8) * DK_WIN + 32 * t;
        const bool active = kt < kend;
        float sc[G][2];
        if (GROUPED) {
            // The window's group (clamped for lanes past the slice end, whose x is zero).
            const int64_t kw = kbeg + (int64_t)(warp + DK_WARPS * w8) * DK_WIN;
            const int64_t grp = imin64(kw / a.group, ngroups - 1);
#pragma unroll
            for (int i = 0; i < G; ++i)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int64_t o = (n0 + 16 * i + g + 8 * h) * ngroups + grp;
                    zb[i][h] = zero_bias_bf16x2((uint32_t)__half2float(a.zero[o]));
                    sc[i][h] = __half2float(a.scale[o]);
                }
        }
        // Activations: for word w (codes k..k+7) the B operand pairs are (x_i, x_{i+4}).
        uint32_t xb[NB][4][4];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            const int64_t m = m0 + 8 * b + g;
            const bool ok = active && m < a.M;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (ok) v = ldg_u4(a.x + m * a.K + kt + 8 * w);
                xb[b][w][0] = prmt(v.x, v.z, 0x5410u);   // (x0, x4)
                xb[b][w][1] = prmt(v.x, v.z, 0x7632u);   // (x1, x5)
                xb[b][w][2] = prmt(v.y, v.w, 0x5410u);   // (x2, x6)
                xb[b][w][3] = prmt(v.y, v.w, 0x7632u);   // (x3, x7)
            }
        }
#pragma unroll
        for (int i = 0; i < G; ++i) {
            const uint32_t wa[4] = {wq[w8][i][0].x, wq[w8][i][0].y, wq[w8][i][0].z, wq[w8][i][0].w};
            const uint32_t wb[4] = {wq[w8][i][1].x, wq[w8][i][1].y, wq[w8][i][1].z, wq[w8][i][1].w};
            float part[NB][4];                 // GROUPED: this window's products, scaled below
            if (GROUPED) {
#pragma unroll
                for (int b = 0; b < NB; ++b) part[b][0] = part[b][1] = part[b][2] = part[b][3] = 0.0f;
            }
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
                        mma_bf16_16816(GROUPED ? part[b] : acc[i][b], af, xb[b][w][2 * hh], xb[b][w][2 * hh + 1]);
                }
            }
            if (GROUPED) {
                // [0], [1]: row g (tokens 2t, 2t + 1); [2], [3]: row g + 8.
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    acc[i][b][0] = fmaf(sc[i][0], part[b][0], acc[i][b][0]);
                    acc[i][b][1] = fmaf(sc[i][0], part[b][1], acc[i][b][1]);
                    acc[i][b][2] = fmaf(sc[i][1], part[b][2], acc[i][b][2]);
                    acc[i][b][3] = fmaf(sc[i][1], part[b][3], acc[i][b][3]);
                }
            }
        }
    }

    // Cross-warp partial sums (summed below in a fixed order).
#pragma unroll
    for (int i = 0; i < G; ++i)
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            red[warp][8 * b + 2 * t][16 * i + g] = acc[i][b][0];
            red[warp][8 * b + 2 * t + 1][16 * i + g] = acc[i][b][1];
            red[warp][8 * b + 2 * t][16 * i + g + 8] = acc[i][b][2];
            red[warp][8 * b + 2 * t + 1][16 * i + g + 8] = acc[i][b][3];
        }
    pdl_launch_dependents();
    const int tm = (int)imin64(TM, a.M - m0);
    __syncthreads();

    // Output units: 4 rows of one token, e4 = token * RT4 + row / 4.  The main term of each unit,
    // s[n] * (sum over warps), is formed here, before the wait for the compensator.
    auto main_part = [&](int e4) {
        const int r4 = e4 % RT4, mm = min(e4 / RT4, TM - 1);
        float4 acc = *reinterpret_cast<const float4*>(&red[0][mm][4 * r4]);
#pragma unroll
        for (int w = 1; w < DK_WARPS; ++w) {
            const float4 p = *reinterpret_cast<const float4*>(&red[w][mm][4 * r4]);
            acc.x += p.x; acc.y += p.y; acc.z += p.z; acc.w += p.w;
        }
        acc.x *= s_scale[4 * r4]; acc.y *= s_scale[4 * r4 + 1];
        acc.z *= s_scale[4 * r4 + 2]; acc.w *= s_scale[4 * r4 + 3];
        return acc;
    };
    const int units = tm * RT4;
    // With few units and an EC term, TPU lanes (a power of two, at most a warp) share one unit's
    // EC columns and meet by shuffles in a fixed order; otherwise thread i takes units i, i + 128, ...
    const bool spread = nj > 0 && 2 * units <= DK_THREADS;
    int tpu = 1;
    if (spread)
        while (2 * tpu * units <= DK_THREADS && tpu < 32) tpu *= 2;
    const int se4 = threadIdx.x / tpu, sub = threadIdx.x % tpu;
    constexpr int UPT = (TM * RT4 + DK_THREADS - 1) / DK_THREADS;
    float4 v[UPT];
    if (spread) {
        v[0] = (se4 < units && sub == 0) ? main_part(se4) : make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
#pragma unroll
        for (int q = 0; q < UPT; ++q) v[q] = main_part(threadIdx.x + q * DK_THREADS);
    }

    // This CTA's reader counter (level 1 of the two-level consumer counters; see
    // retire_accumulators) and thread 0's ticket from it.
    unsigned reader_ticket = 0u;
    auto reader_counter = [&]() {
        const int grp = (tile * S + ks) / CONSUMER_GROUP;
        return a.consumed1 + (int64_t)chunk * GROUPS_MAX + grp;
    };
    if (has_ec) {
        // u = sigmoid(p + b_g) t for this CTA's EC columns.  Element c = mm * nj + jj; thread i
        // takes c = i, i + 128, ... (stepping without dividing) and reads the words of t[mm, j0 + jj]
        // and p[mm] until both hold every K slice (a bounded wait); each element recomputes its
        // token's gate, so one pass and one barrier suffice.
        const long long* tc = a.tacc + (int64_t)chunk * TM * (a.rank + 1);
        const int ujr = a.ec_jr + 1, total = tm * nj;
        const unsigned long long want = (unsigned long long)ec_slices(a.K) & FIX_COUNT_MASK;
        if (nj > 0 && a.mlp.w1 != nullptr) {
            // The bottleneck-MLP gate reads every column of t: all tm x r words (bounded wait on
            // their slice counts), then h = relu(W1 t + b1), then gamma and u for this CTA's columns.
            const int r = a.rank, H = a.mlp.hidden, tot = tm * r;
            constexpr int UB = 8;
            // First wait on this CTA's own columns only (CTAs of a chunk watch different words, as
            // with the scalar gate), then read every column, by then almost surely complete.
            {
                const int own = tm * nj;
                unsigned it = 0;
                for (;;) {
                    bool done = true;
                    for (int c = threadIdx.x; c < own; c += DK_THREADS) {
                        const long long v = ld_relaxed_s64(tc + (int64_t)(c / nj) * (r + 1) + j0 + c % nj);
                        done = done && ((unsigned long long)v & FIX_COUNT_MASK) == want;
                    }
                    if (__syncthreads_and(done)) break;
                    if (++it > SPIN_LIMIT) break;     // the reads below give up and flag it
                    if (it > 16) __nanosleep(64);
                }
            }
            for (int base = 0; base < tot; base += UB * DK_THREADS) {   // uniform trip count
                const long long* ptr[UB];
                bool valid[UB];
#pragma unroll
                for (int u = 0; u < UB; ++u) {
                    const int c = base + (int)threadIdx.x + u * DK_THREADS;
                    valid[u] = c < tot;
                    ptr[u] = tc + (valid[u] ? (int64_t)(c / r) * (r + 1) + c % r : 0);
                }
                long long tv[UB];
                unsigned it = 0;
                for (;;) {
                    bool done = true;
#pragma unroll
                    for (int u = 0; u < UB; ++u) tv[u] = valid[u] ? ld_relaxed_s64(ptr[u]) : 0ll;
#pragma unroll
                    for (int u = 0; u < UB; ++u)
                        done = done && (!valid[u] || ((unsigned long long)tv[u] & FIX_COUNT_MASK) == want);
                    if (__syncthreads_and(done)) break;
                    if (++it > SPIN_LIMIT) {
                        if (threadIdx.x == 0) atomicOr(a.err, 1u);
#pragma unroll
                        for (int u = 0; u < UB; ++u) tv[u] = 0ll;
                        break;
                    }
                    if (it > 16) __nanosleep(64);
                }
#pragma unroll
                for (int u = 0; u < UB; ++u) {
                    const int c = base + (int)threadIdx.x + u * DK_THREADS;
                    if (valid[u]) mlp_t[(c / r) * (r + 1) + c % r] = __ll2float_rn(tv[u] >> FIX_COUNT_BITS) * (1.0f / FIX_ONE);
                }
            }
            __syncthreads();
            // One thread per output, token index fastest: the threads of a warp read one or two rows
            // of W1 (W2) at a time (broadcast loads), and the padded rows of t (h) keep the
            // shared-memory reads free of bank conflicts.
            for (int o = threadIdx.x; o < tm * H; o += DK_THREADS) {
                const int mm = o % tm, i = o / tm;
                const float* w1 = a.mlp.w1 + (int64_t)i * r;
                const float* tr = mlp_t + mm * (r + 1);
                float pre = __ldg(a.mlp.b1 + i);
#pragma unroll 8
                for (int j = 0; j < r; ++j) pre = fmaf(__ldg(w1 + j), tr[j], pre);
                mlp_h[mm * (H + 1) + i] = fmaxf(pre, 0.0f);
            }
            __syncthreads();
            for (int c = threadIdx.x; c < tm * nj; c += DK_THREADS) {
                const int mm = c % tm, jj = c / tm, j = j0 + jj;
                const float* w2 = a.mlp.w2 + (int64_t)j * H;
                const float* hr = mlp_h + mm * (H + 1);
                float pre = __ldg(a.mlp.b2 + j);
#pragma unroll 8
                for (int i = 0; i < H; ++i) pre = fmaf(__ldg(w2 + i), hr[i], pre);
                us[mm * ujr + jj] = a.mlp.alpha * mlp_t[mm * (r + 1) + j] / (1.0f + expf(-pre));
            }
            asm volatile("cp.async.wait_all;" ::: "memory");
        } else if (nj > 0) {
            const int dmm = DK_THREADS / nj, djj = DK_THREADS % nj;
            int mm = threadIdx.x / nj, jj = threadIdx.x % nj;
            constexpr int UB = 8;         // elements per thread per pass, loads issued together
            for (int base = 0; base < total; base += UB * DK_THREADS) {   // uniform trip count
                const long long* tp[UB];
                const long long* pp[UB];
                int um[UB], uj[UB];
                bool valid[UB];
#pragma unroll
                for (int u = 0; u < UB; ++u) {
                    valid[u] = base + (int)threadIdx.x + u * DK_THREADS < total;
                    um[u] = mm;
                    uj[u] = jj;
                    tp[u] = tc + (int64_t)(valid[u] ? mm : 0) * (a.rank + 1) + j0 + (valid[u] ? jj : 0);
                    pp[u] = tc + (int64_t)(valid[u] ? mm : 0) * (a.rank + 1) + a.rank;
                    mm += dmm;
                    jj += djj;
                    if (jj >= nj) { jj -= nj; ++mm; }
                }
                long long tv[UB], pv[UB];
                unsigned it = 0;
                for (;;) {
                    bool done = true;
#pragma unroll
                    for (int u = 0; u < UB; ++u) {
                        tv[u] = valid[u] ? ld_relaxed_s64(tp[u]) : 0ll;
                        pv[u] = valid[u] ? ld_relaxed_s64(pp[u]) : 0ll;
                    }
#pragma unroll
                    for (int u = 0; u < UB; ++u)
                        done = done && (!valid[u] || (((unsigned long long)tv[u] & FIX_COUNT_MASK) == want &&
                                                      ((unsigned long long)pv[u] & FIX_COUNT_MASK) == want));
                    if (__syncthreads_and(done)) break;
                    if (++it > SPIN_LIMIT) {          // give up: flag it and add nothing
                        if (threadIdx.x == 0) atomicOr(a.err, 1u);
#pragma unroll
                        for (int u = 0; u < UB; ++u) tv[u] = pv[u] = 0ll;
                        break;
                    }
                    if (it > 16) __nanosleep(64);
                }
#pragma unroll
                for (int u = 0; u < UB; ++u) {
                    if (valid[u]) {
                        const float t_ = __ll2float_rn(tv[u] >> FIX_COUNT_BITS) * (1.0f / FIX_ONE);
                        const float p_ = __ll2float_rn(pv[u] >> FIX_COUNT_BITS) * (1.0f / FIX_ONE);
                        us[um[u] * ujr + uj[u]] = __fdividef(t_, 1.0f + __expf(-(p_ + a.b_g)));
                    }
                }
            }
            asm volatile("cp.async.wait_all;" ::: "memory");
        }
        __syncthreads();
        // Every thread has read its accumulator words: count this CTA as a reader now, so that the
        // atomic's round trip overlaps the epilogue instead of delaying the CTA's exit.
        if (threadIdx.x == 0) reader_ticket = atomicAdd(reader_counter(), 1u);

        // This slice's EC columns: sum_j u[m, j] B[j, n] added to each unit.
        if (spread) {
            if (se4 < units) {
                const int r4 = se4 % RT4, mu = se4 / RT4;
                const float* ur = us + mu * ujr;
                const uint16_t* br = Bs + 4 * r4;
#pragma unroll 8
                for (int jj = sub; jj < nj; jj += tpu) {
                    const float uq = ur[jj];
                    const uint2 bb = *reinterpret_cast<const uint2*>(br + jj * RT);
                    v[0].x = fmaf(uq, __uint_as_float(bb.x << 16), v[0].x);
                    v[0].y = fmaf(uq, __uint_as_float(bb.x & 0xFFFF0000u), v[0].y);
                    v[0].z = fmaf(uq, __uint_as_float(bb.y << 16), v[0].z);
                    v[0].w = fmaf(uq, __uint_as_float(bb.y & 0xFFFF0000u), v[0].w);
                }
            }
            for (int o = 1; o < tpu; o *= 2) {
                v[0].x += __shfl_down_sync(0xFFFFFFFFu, v[0].x, o);
                v[0].y += __shfl_down_sync(0xFFFFFFFFu, v[0].y, o);
                v[0].z += __shfl_down_sync(0xFFFFFFFFu, v[0].z, o);
                v[0].w += __shfl_down_sync(0xFFFFFFFFu, v[0].w, o);
            }
        } else {
#pragma unroll 4
            for (int jj = 0; jj < nj; ++jj) {
#pragma unroll
                for (int q = 0; q < UPT; ++q) {
                    const int e4 = threadIdx.x + q * DK_THREADS;
                    const int r4 = e4 % RT4, mu = min(e4 / RT4, TM - 1);
                    const float uq = us[mu * ujr + jj];
                    const uint2 bb = *reinterpret_cast<const uint2*>(Bs + jj * RT + 4 * r4);
                    v[q].x = fmaf(uq, __uint_as_float(bb.x << 16), v[q].x);
                    v[q].y = fmaf(uq, __uint_as_float(bb.x & 0xFFFF0000u), v[q].y);
                    v[q].z = fmaf(uq, __uint_as_float(bb.y << 16), v[q].z);
                    v[q].w = fmaf(uq, __uint_as_float(bb.y & 0xFFFF0000u), v[q].w);
                }
            }
        }
    }

    auto store4 = [&](int64_t m, int r4, float4 o) {
        if (a.ymain != nullptr) {
            reinterpret_cast<float4*>(a.ymain + m * a.N + n0)[r4] = o;
        } else if (a.y_fp32) {
            reinterpret_cast<float4*>(reinterpret_cast<float*>(a.y) + m * a.N + n0)[r4] = o;
        } else {
            const __nv_bfloat162 lo = __floats2bfloat162_rn(o.x, o.y), hi = __floats2bfloat162_rn(o.z, o.w);
            uint2 pk;
            pk.x = *reinterpret_cast<const uint32_t*>(&lo);
            pk.y = *reinterpret_cast<const uint32_t*>(&hi);
            reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(a.y) + m * a.N + n0)[r4] = pk;
        }
    };
    // The S K slices of a row tile (one cluster) meet in distributed shared memory: unit e4 of the
    // tile belongs to rank e4 / per, and every rank pushes its value of the unit to that owner.
    const int per = TM * RT4 / S;
    auto emit = [&](int e4, float4 o) {
        if (S == 1) {
            store4(m0 + e4 / RT4, e4 % RT4, o);
        } else {
            const int owner = e4 / per;
            st_dsmem_f4(&recv[ks * per + (e4 - owner * per)], (unsigned)owner, o);
        }
    };
    if (S > 1) cluster_wait();
    if (spread) {
        if (se4 < units && sub == 0) emit(se4, v[0]);
    } else {
#pragma unroll
        for (int q = 0; q < UPT; ++q) {
            const int e4 = threadIdx.x + q * DK_THREADS;
            if (e4 < units) emit(e4, v[q]);
        }
    }

    // Every GEMM CTA of the chunk has read the accumulators and counted itself (its ticket, taken
    // right after its reads): the last one clears them and the arrival counter for the next call.
    // Two counter levels (groups of CONSUMER_GROUP CTAs, then groups) keep same-address atomics few.
    auto retire_accumulators = [&]() {
        if (!has_ec) return;
        if (threadIdx.x == 0) {
            const int per_chunk = a.row_tiles * S;
            const int idx = tile * S + ks;                 // this CTA's index within the chunk
            const int grp = idx / CONSUMER_GROUP;
            const int in_grp = min(CONSUMER_GROUP, per_chunk - grp * CONSUMER_GROUP);
            const int groups = (per_chunk + CONSUMER_GROUP - 1) / CONSUMER_GROUP;
            unsigned* c1 = a.consumed1 + (int64_t)chunk * GROUPS_MAX + grp;
            unsigned last = 0u;
            if (reader_ticket == (unsigned)in_grp - 1) {
                *c1 = 0u;                                  // group complete: re-arm
                last = (atomicAdd(&a.consumed[chunk], 1u) == (unsigned)groups - 1) ? 1u : 0u;
            }
            s_flag = last;
        }
        __syncthreads();
        if (s_flag) {
            long long* tc = a.tacc + (int64_t)chunk * TM * (a.rank + 1);
            for (int c = threadIdx.x; c < tm * (a.rank + 1); c += DK_THREADS) tc[c] = 0ll;
            if (threadIdx.x == 0) {
                a.consumed[chunk] = 0u;
                a.arrivals[chunk] = 0u;
            }
        }
    };
    if (S == 1) {
        retire_accumulators();
        return;
    }

    // After the barrier every push has landed; the owner sums its units over ranks 0..S-1 in rank
    // order and rounds once.  No rank touches another's shared memory after the barrier.
    cluster_sync_all();
    for (int l = threadIdx.x; l < per; l += DK_THREADS) {
        const int e4 = ks * per + l;
        const int r4 = e4 % RT4, mm = e4 / RT4;
        if (mm >= tm) continue;
        float4 o = recv[l];
        for (int q = 1; q < S; ++q) {
            const float4 p = recv[q * per + l];
            o.x += p.x; o.y += p.y; o.z += p.z; o.w += p.w;
        }
        store4(m0 + mm, r4, o);
    }
    retire_accumulators();
}

template <int NB, int G, int WPW, bool GROUPED>
__global__ void __launch_bounds__(DK_THREADS, 4) w4ec_decode_kernel(DecodeArgs a) {
    extern __shared__ __align__(16) unsigned char dyn_smem[];
    int bid = blockIdx.x;
    if (bid < a.ec_ctas) {                 // EC CTAs, padded to whole clusters
        const int E = a.rank > 0 ? a.ec_splits * a.mchunks : 0;
        if (bid < E) ec_role<8 * NB>(a, bid % a.ec_splits, bid / a.ec_splits, dyn_smem);
        return;
    }
    bid -= a.ec_ctas;
    const int ks = bid % a.split;          // = the rank within the cluster
    const int rest = bid / a.split;
    gemm_role<NB, G, WPW, GROUPED>(a, rest % a.row_tiles, ks, rest / a.row_tiles, dyn_smem);
}

// ---------------------------------------------------------------------------------------------
// Separate EC pass (apply kernel).  Launched right after the decode kernel with programmatic
// dependent launch, so its wait returns once every EC and GEMM CTA of that launch is complete:
// the accumulators and the fp32 main term are final and need no polling.  CTA b takes 128 output
// rows (thread i <-> row 128 b + i) and every token of the launch:
//   u[m, j] = sigmoid(p[m] + b_g) t[m, j]          (from the accumulator words, in shared memory)
//   y[m, n] = main[m, n] + sum_j u[m, j] B[j, n]   (B tile prefetched before the wait)
// The last CTA to finish clears the accumulators for the next call.
// ---------------------------------------------------------------------------------------------
constexpr int AP_ROWS = 128;
constexpr int AP_TOK = 16;              // tokens per pass over u

__global__ void __launch_bounds__(AP_ROWS) w4ec_apply_kernel(DecodeArgs a) {
    extern __shared__ __align__(16) unsigned char dyn_smem[];
    const int r = a.rank;
    uint16_t* Bs = reinterpret_cast<uint16_t*>(dyn_smem);                          // [r][AP_ROWS]
    float* us = reinterpret_cast<float*>(dyn_smem + (size_t)r * AP_ROWS * 2);      // [AP_TOK][r]
    float* hs = us + AP_TOK * r;                                                   // MLP gate: [AP_TOK][H]
    const bool mlp = a.mlp.w1 != nullptr;
    __shared__ unsigned s_last;
    const int64_t n0 = (int64_t)blockIdx.x * AP_ROWS;
    const int64_t n = n0 + threadIdx.x;
    constexpr int CH = AP_ROWS / 8;
    for (int c = threadIdx.x; c < r * CH; c += AP_ROWS) {
        const int jj = c / CH, cc = c % CH;
        cp_async_16(Bs + jj * AP_ROWS + cc * 8, a.B + (int64_t)jj * a.N + n0 + cc * 8);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");

    pdl_wait_primary();
    asm volatile("cp.async.wait_all;" ::: "memory");

    for (int64_t mb = 0; mb < a.M; mb += AP_TOK) {
        const int tk = (int)imin64(AP_TOK, a.M - mb);
        __syncthreads();                          // the previous pass is done with us
        // u of these tokens: all loads of a thread's elements in flight together.
        constexpr int UB = (AP_TOK * 256 + AP_ROWS - 1) / AP_ROWS;   // ranks up to 256
        long long tv[UB], pv[UB];
#pragma unroll
        for (int u = 0; u < UB; ++u) {
            const int c = threadIdx.x + u * AP_ROWS;
            const int mm = c / r, j = c % r;
            const bool ok = c < tk * r;
            const long long* row = a.tacc + (mb + (ok ? mm : 0)) * (int64_t)(r + 1);
            tv[u] = ok ? __ldcg(row + j) : 0ll;
            pv[u] = ok ? __ldcg(row + r) : 0ll;
        }
#pragma unroll
        for (int u = 0; u < UB; ++u) {
            const int c = threadIdx.x + u * AP_ROWS;
            if (c < tk * r) {
                const float t_ = __ll2float_rn(tv[u] >> FIX_COUNT_BITS) * (1.0f / FIX_ONE);
                const float p_ = __ll2float_rn(pv[u] >> FIX_COUNT_BITS) * (1.0f / FIX_ONE);
                us[c] = mlp ? t_ : t_ / (1.0f + expf(-(p_ + a.b_g)));
            }
        }
        if (mlp) {
            // Bottleneck-MLP gate: h = relu(W1 t + b1), then u = alpha sigmoid(W2 h + b2) t in place.
            const int H = a.mlp.hidden;
            __syncthreads();
            for (int o = threadIdx.x; o < tk * H; o += AP_ROWS) {
                const int mm = o % tk, i = o / tk;
                const float* w1 = a.mlp.w1 + (int64_t)i * r;
                float pre = __ldg(a.mlp.b1 + i);
#pragma unroll 8
                for (int j = 0; j < r; ++j) pre = fmaf(__ldg(w1 + j), us[mm * r + j], pre);
                hs[mm * (H + 1) + i] = fmaxf(pre, 0.0f);
            }
            __syncthreads();
            for (int c = threadIdx.x; c < tk * r; c += AP_ROWS) {
                const int mm = c / r, j = c % r;
                const float* w2 = a.mlp.w2 + (int64_t)j * H;
                float pre = __ldg(a.mlp.b2 + j);
#pragma unroll 8
                for (int i = 0; i < H; ++i) pre = fmaf(__ldg(w2 + i), hs[mm * (H + 1) + i], pre);
                us[c] = a.mlp.alpha * us[c] / (1.0f + expf(-pre));
            }
        }
        float mv[AP_TOK];
#pragma unroll
        for (int mm = 0; mm < AP_TOK; ++mm) mv[mm] = mm < tk ? __ldcg(a.ymain + (mb + mm) * a.N + n) : 0.0f;
        __syncthreads();
#pragma unroll
        for (int mm = 0; mm < AP_TOK; ++mm) {
            if (mm >= tk) break;
            const int64_t m = mb + mm;
            float v = mv[mm];
            const float* ur = us + mm * r;
#pragma unroll 8
            for (int j = 0; j < r; ++j) v = fmaf(ur[j], bf16_bits_to_f32(Bs[j * AP_ROWS + threadIdx.x]), v);
            if (a.y_fp32)
                reinterpret_cast<float*>(a.y)[m * a.N + n] = v;
            else
                reinterpret_cast<__nv_bfloat16*>(a.y)[m * a.N + n] = __float2bfloat16_rn(v);
        }
    }
    pdl_launch_dependents();

    // Every CTA has read the accumulators before its acq_rel count; the last one clears them.
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned prev;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(a.consumed) : "memory");
        s_last = (prev == gridDim.x - 1) ? 1u : 0u;
    }
    __syncthreads();
    if (s_last) {
        for (int64_t c = threadIdx.x; c < a.M * (int64_t)(r + 1); c += AP_ROWS) a.tacc[c] = 0ll;
        if (threadIdx.x == 0) *a.consumed = 0u;
    }
}

size_t apply_dyn_smem_bytes(int rank, int gate_hidden) {
    return (size_t)rank * AP_ROWS * 2 + (size_t)AP_TOK * rank * 4 + (size_t)AP_TOK * (gate_hidden + 1) * 4;
}

cudaError_t launch_apply(const DecodeArgs& a, cudaStream_t stream) {
    const size_t dyn = apply_dyn_smem_bytes(a.rank, a.mlp.w1 ? a.mlp.hidden : 0);
    // The limit is raised to this launch's size when it is below (thread-safe, per device).
    static std::mutex mu;
    static size_t opted[kMaxDevices] = {0};
    cudaError_t oe = opt_in_smem_at_least((const void*)w4ec_apply_kernel, dyn, mu, opted);
    if (oe != cudaSuccess) return oe;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.N / AP_ROWS));
    cfg.blockDim = dim3(AP_ROWS);
    cfg.dynamicSmemBytes = dyn;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, w4ec_apply_kernel, a);
}

// ---------------------------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------------------------
size_t decode_dyn_smem_bytes(int nb, int g, int ec_jr, int rank, int gate_hidden) {
    if (rank <= 0) return 0;
    size_t gemm = (size_t)ec_jr * 16 * g * 2 + (size_t)8 * nb * (ec_jr + 1) * 4;
    if (gate_hidden > 0) gemm += (size_t)8 * nb * (rank + 1 + gate_hidden + 1) * 4;   // MLP gate: t, hidden rows
    const size_t ec = (size_t)DK_WARPS * 8 * nb * EC_RS * 4;
    return gemm > ec ? gemm : ec;
}

bool decode_config_supported(int nb, int g, int wpw) {
    if (!(nb == 1 || nb == 2 || nb == 4)) return false;
    if (nb == 4 && g * wpw > 4) return false;      // would spill registers
    if (g == 8) return wpw == 1 && nb <= 2;
    if (g == 4) return wpw == 1 || wpw == 2;
    if (g == 2) return wpw == 1 || wpw == 2 || wpw == 4;
    if (g == 1) return wpw == 1 || wpw == 2 || wpw == 4 || wpw == 8;
    return false;
}

template <int NB, int G, int WPW, bool GROUPED>
static cudaError_t launch_t(const DecodeArgs& a, cudaStream_t stream) {
    static_assert(WPW * G <= 8, "weight registers");
    const unsigned grid = (unsigned)(a.ec_ctas + a.row_tiles * a.split * a.mchunks);
    const size_t dyn = decode_dyn_smem_bytes(NB, G, a.ec_jr, a.rank, a.mlp.w1 ? a.mlp.hidden : 0);
    // Static plus dynamic shared memory above 48 KB needs the opt-in attribute (once per device).
    static std::mutex mu;
    static size_t opted[kMaxDevices] = {0};
    cudaError_t oe = opt_in_smem_at_least((const void*)w4ec_decode_kernel<NB, G, WPW, GROUPED>, dyn, mu, opted);
    if (oe != cudaSuccess) return oe;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(DK_THREADS);
    cfg.dynamicSmemBytes = dyn;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)a.split;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.split > 1 ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, w4ec_decode_kernel<NB, G, WPW, GROUPED>, a);
}

cudaError_t launch_decode(const DecodeArgs& a, int nb, int g, int wpw, cudaStream_t stream) {
#define SPEAR_DK_CASE(NB_, G_, W_) \
    if (nb == NB_ && g == G_ && wpw == W_)                                                          \
        return a.group > 0 ? launch_t<NB_, G_, W_, true>(a, stream) : launch_t<NB_, G_, W_, false>(a, stream);
#define SPEAR_DK_NB(NB_)                                                                              \
    SPEAR_DK_CASE(NB_, 1, 1) SPEAR_DK_CASE(NB_, 1, 2) SPEAR_DK_CASE(NB_, 1, 4) SPEAR_DK_CASE(NB_, 1, 8) \
    SPEAR_DK_CASE(NB_, 2, 1) SPEAR_DK_CASE(NB_, 2, 2) SPEAR_DK_CASE(NB_, 2, 4)                          \
    SPEAR_DK_CASE(NB_, 4, 1) SPEAR_DK_CASE(NB_, 4, 2)
    SPEAR_DK_NB(1) SPEAR_DK_NB(2) SPEAR_DK_NB(4)
    SPEAR_DK_CASE(1, 8, 1) SPEAR_DK_CASE(2, 8, 1)
#undef SPEAR_DK_NB
#undef SPEAR_DK_CASE
    return cudaErrorInvalidValue;
}

}  // namespace spear
