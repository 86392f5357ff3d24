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
//   * EC CTAs (the lowest block indices, so they are dispatched first) each take 128 rows of A
//     (warp w: 32 rows; lane l: column pairs l, l+32, ...; the gate column by a warp reduction),
//     compute partial sums of t and of the gate pre-activation, add them into the token chunk's
//     int64 fixed-point accumulators (2^-32 resolution; integer addition is exact, so the sum
//     does not depend on arrival order) and count themselves in the chunk's arrival counter;
//   * GEMM CTAs own 16*G weight rows, a K slice of at most 512*WPW codes and 8*NB tokens.  Every
//     weight byte of the CTA is requested from HBM first (registers), then the kernel waits for
//     its predecessor in the stream (programmatic dependent launch) before reading x.  Lane
//     (g = lane/4, t = lane%4) of warp w holds 16 bytes (32 codes) of rows g and g+8 of each
//     16-row group for the 128-wide K windows w, w+4, ...; codes become exact bf16 (q - z) in
//     registers and feed mma.sync m16n8k16 with the weights as the M=16 operand and the tokens as
//     N=8.  Inside each MMA the K order is permuted to pairs (k, k+4), and x is loaded with the
//     same permutation, which leaves the dot product unchanged;
//   * the four warps meet in shared memory in a fixed order.  Each GEMM CTA then waits, with a
//     bounded spin, until all EC CTAs of its token chunk have arrived, forms g = sigmoid(p + b_g)
//     and u = g t for its share (r/S columns) of the EC term from the accumulators, scales by
//     s[n] and adds u B (the B slice was prefetched with cp.async at the start).  The S K slices
//     of a row tile form one thread-block cluster and meet in distributed shared memory: after a
//     cluster barrier, rank q sums its share of the tile over ranks 0..S-1 in rank order and
//     rounds once to bf16.
// No floating-point atomics: results are deterministic for a given plan.  Counters and
// accumulators re-arm themselves, so the zeroed part of the workspace is zero again after every
// call.
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

SPEAR_DEVI void bf16x8_to_f32(const uint4 v, float f[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// ---------------------------------------------------------------------------------------------
// EC role: partial t = x A and p = x w_g over 128 rows of A for one token chunk.
// Warp w takes rows kbeg + 16 w .. + 15.  Lane l accumulates column pairs (2p, 2p + 1),
// p = l, l + 32, ..., so a warp reads whole rows of A; the gate column is a per-lane product
// (lane l < 16 <-> row l of the warp) reduced across the warp.  The warps meet in
// shared memory, and the CTA's sums go into the int64 fixed-point accumulators.
// ---------------------------------------------------------------------------------------------
constexpr int EC_ROWS = 64;                  // rows of A per EC CTA (16 per warp)
constexpr int EC_WROWS = EC_ROWS / DK_WARPS;
constexpr double FIX_SCALE = 4294967296.0;   // 2^32
constexpr float FIX_LIMIT = 67108864.0f;     // 2^26: |CTA partial| bound, so 32 slices fit in int64

// Signed fixed-point values added as two's-complement 64-bit integers (exact, order-free).
SPEAR_DEVI void red_add_s64(long long* p, long long v) {
    asm volatile("red.relaxed.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"((unsigned long long)v) : "memory");
}

SPEAR_DEVI uint32_t ldg_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

template <int TM>
SPEAR_DEVI void ec_role(const DecodeArgs& a, int s, int chunk, unsigned char* dyn) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = a.rank, NP = r / 2, NC = (NP + 31) / 32, RS = r + 4;
    uint16_t* xs = reinterpret_cast<uint16_t*>(dyn);                            // [TM][EC_ROWS]
    float* red_ec = reinterpret_cast<float*>(dyn + (size_t)TM * EC_ROWS * 2);    // [DK_WARPS][8][RS]
    const int64_t kc0 = (int64_t)s * EC_ROWS;
    const int64_t kw = kc0 + EC_WROWS * warp;            // this warp's first row
    const int64_t m0 = (int64_t)chunk * TM;
    const int tm = (int)imin64(TM, a.M - m0);

    // Prefetch (before the wait) the first 64 columns of this warp's rows and its gate weight.
    uint32_t a0[EC_WROWS];
#pragma unroll
    for (int i = 0; i < EC_WROWS; ++i)
        a0[i] = (kw + i < a.K && lane < NP) ? ldg_u32(a.A + (kw + i) * r + 2 * lane) : 0u;
    const float wgv = (lane < EC_WROWS && kw + lane < a.K) ? bf16_bits_to_f32(a.wg[kw + lane]) : 0.0f;

    // x may be the previous kernel's output; the previous call may still use the workspace.
    pdl_wait_primary();

    for (int i = threadIdx.x; i < TM * (EC_ROWS / 8); i += DK_THREADS) {
        const int m = i / (EC_ROWS / 8), k8 = i % (EC_ROWS / 8);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (m < tm && kc0 + 8 * k8 < a.K) v = ldg_u4(a.x + (m0 + m) * a.K + kc0 + 8 * k8);
        *reinterpret_cast<uint4*>(xs + m * EC_ROWS + 8 * k8) = v;
    }
    __syncthreads();

    // Column pairs p of this lane against the warp's 32 rows, for tokens ms .. ms+7.
    auto columns = [&](const uint32_t (&av)[EC_WROWS], int p, int ms) {
        float acc[8][2];
#pragma unroll
        for (int m = 0; m < 8; ++m) acc[m][0] = acc[m][1] = 0.0f;
#pragma unroll
        for (int i = 0; i < EC_WROWS; ++i) {
            const float lo = __uint_as_float(av[i] << 16), hi = __uint_as_float(av[i] & 0xFFFF0000u);
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const float xv = bf16_bits_to_f32(xs[(ms + m) * EC_ROWS + EC_WROWS * warp + i]);
                acc[m][0] = fmaf(xv, lo, acc[m][0]);
                acc[m][1] = fmaf(xv, hi, acc[m][1]);
            }
        }
        if (p < NP) {
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                red_ec[(warp * 8 + m) * RS + 2 * p] = acc[m][0];
                red_ec[(warp * 8 + m) * RS + 2 * p + 1] = acc[m][1];
            }
        }
    };

    for (int ms = 0; ms < tm; ms += 8) {
        columns(a0, lane, ms);
        for (int c = 1; c < NC; ++c) {
            const int p = lane + 32 * c;
            uint32_t av[EC_WROWS];
#pragma unroll
            for (int i = 0; i < EC_WROWS; ++i) av[i] = (kw + i < a.K && p < NP) ? ldg_u32(a.A + (kw + i) * r + 2 * p) : 0u;
            columns(av, p, ms);
        }
        // Gate pre-activation: lane l < 16 holds row kw + l (wgv = 0 on the other lanes).
        float gp[8];
        const int gl = lane < EC_WROWS ? lane : 0;
#pragma unroll
        for (int m = 0; m < 8; ++m) gp[m] = bf16_bits_to_f32(xs[(ms + m) * EC_ROWS + EC_WROWS * warp + gl]) * wgv;
#pragma unroll
        for (int m = 0; m < 8; ++m)
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) gp[m] += __shfl_xor_sync(0xFFFFFFFFu, gp[m], o);
        if (lane == 0) {
#pragma unroll
            for (int m = 0; m < 8; ++m) red_ec[(warp * 8 + m) * RS + r] = gp[m];
        }
        __syncthreads();
        // Cross-warp sums (fixed order), then exact integer accumulation across CTAs.
        for (int o = threadIdx.x; o < 8 * (r + 1); o += DK_THREADS) {
            const int m = o / (r + 1), j = o % (r + 1);
            if (ms + m >= tm) continue;
            float v = red_ec[m * RS + j];
#pragma unroll
            for (int w = 1; w < DK_WARPS; ++w) v += red_ec[(w * 8 + m) * RS + j];
            if (!(fabsf(v) < FIX_LIMIT)) {
                atomicOr(a.err, 2u);
                v = 0.0f;
            }
            red_add_s64(a.tacc + (chunk * TM + ms + m) * (int64_t)(r + 1) + j, __double2ll_rn((double)v * FIX_SCALE));
        }
        __syncthreads();
    }
    __syncthreads();
    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        // The barrier above orders every thread's accumulator additions before this fence; the
        // release add then publishes the arrival.
        __threadfence();
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&a.arrivals[chunk]) : "memory");
    }
}

// ---------------------------------------------------------------------------------------------
// Cluster helpers (distributed shared memory).
// ---------------------------------------------------------------------------------------------
SPEAR_DEVI void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
SPEAR_DEVI float4 ld_dsmem_f4(const float* local, unsigned rank) {
    uint32_t la = (uint32_t)__cvta_generic_to_shared(local), ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(la), "r"(rank));
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(ra) : "memory");
    return v;
}

// ---------------------------------------------------------------------------------------------
// GEMM role.
// ---------------------------------------------------------------------------------------------
template <int NB, int G, int WPW>
SPEAR_DEVI void gemm_role(const DecodeArgs& a, int tile, int ks, int chunk, unsigned char* dyn) {
    constexpr int RT = 16 * G;        // weight rows per CTA
    constexpr int TM = 8 * NB;        // tokens per CTA
    __shared__ float red[DK_WARPS][RT][TM + 1];
    __shared__ __align__(16) float ps[TM * RT];      // this K slice's finished partial, [token][row]
    __shared__ float s_scale[RT];
    __shared__ unsigned s_flag;
    uint16_t* Bs = reinterpret_cast<uint16_t*>(dyn);                           // [ec_jr][RT] bf16
    float* us = reinterpret_cast<float*>(dyn + (size_t)a.ec_jr * RT * 2);      // [TM][ec_jr + 1]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t n0 = (int64_t)tile * RT;
    const int S = a.split;
    const int64_t m0 = (int64_t)chunk * TM;
    const int64_t kbeg = (int64_t)ks * a.k_slice;
    const int64_t kend = imin64(kbeg + a.k_slice, a.K);
    const int64_t row_bytes = a.K / 2;
    const bool has_ec = a.rank > 0;
    const int j0 = ks * a.ec_jr;
    const int nj = has_ec ? max(0, min(a.rank, j0 + a.ec_jr) - j0) : 0;

    // ---- Prologue: only inputs that no earlier kernel in the stream can be writing. ----
    if (nj > 0) {
        constexpr int CH = RT / 8;     // 16-byte pieces per B row slice
        for (int c = threadIdx.x; c < nj * CH; c += DK_THREADS) {
            const int jj = c / CH, cc = c % CH;
            cp_async_16(Bs + jj * RT + cc * 8, a.B + (int64_t)(j0 + jj) * a.N + n0 + cc * 8);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    for (int i = threadIdx.x; i < RT; i += DK_THREADS) s_scale[i] = __half2float(a.scale[n0 + i]);
    uint32_t zb[G][2];
#pragma unroll
    for (int i = 0; i < G; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h)
            zb[i][h] = zero_bias_bf16x2((uint32_t)__half2float(a.zero[n0 + 16 * i + g + 8 * h]));
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

    // Cross-warp partial sums (summed below in a fixed order).
#pragma unroll
    for (int i = 0; i < G; ++i)
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            red[warp][16 * i + g][8 * b + 2 * t] = acc[i][b][0];
            red[warp][16 * i + g][8 * b + 2 * t + 1] = acc[i][b][1];
            red[warp][16 * i + g + 8][8 * b + 2 * t] = acc[i][b][2];
            red[warp][16 * i + g + 8][8 * b + 2 * t + 1] = acc[i][b][3];
        }
    pdl_launch_dependents();
    const int tm = (int)imin64(TM, a.M - m0);

    if (has_ec) {
        // Every EC CTA of this token chunk has added its partial sums (bounded wait).
        if (threadIdx.x == 0) {
            unsigned it = 0, ok = 1;
            while (ld_acquire_u32(&a.arrivals[chunk]) < (unsigned)a.ec_splits) {
                if (++it > SPIN_LIMIT) { atomicOr(a.err, 1u); ok = 0; break; }
                if (it > 256) __nanosleep(64);
            }
            s_flag = ok;
        }
        __syncthreads();
        // g = sigmoid(p + b_g) and u = g t for this CTA's EC columns, from the exact accumulators.
        const long long* tc = a.tacc + (int64_t)chunk * TM * (a.rank + 1);
        for (int c = threadIdx.x; c < tm * (nj + 1); c += DK_THREADS) {
            const int mm = c / (nj + 1), jj = c % (nj + 1);
            const int col = jj < nj ? j0 + jj : a.rank;
            const long long v = s_flag ? __ldcg(tc + (int64_t)mm * (a.rank + 1) + col) : 0ll;
            us[mm * (a.ec_jr + 1) + jj] = (float)((double)v * (1.0 / FIX_SCALE));
        }
        __syncthreads();
        for (int mm = threadIdx.x; mm < tm; mm += DK_THREADS) {
            const float p = us[mm * (a.ec_jr + 1) + nj] + a.b_g;
            us[mm * (a.ec_jr + 1) + nj] = 1.0f / (1.0f + expf(-p));
        }
        __syncthreads();
        for (int c = threadIdx.x; c < tm * nj; c += DK_THREADS) {
            const int mm = c / nj, jj = c % nj;
            us[mm * (a.ec_jr + 1) + jj] *= us[mm * (a.ec_jr + 1) + nj];
        }
        if (nj > 0) asm volatile("cp.async.wait_all;" ::: "memory");
    }
    __syncthreads();
    if (has_ec) {
        // Every GEMM CTA of the chunk has read the accumulators: the last one clears them and the
        // arrival counter for the next call.  Two counter levels (groups of CONSUMER_GROUP CTAs,
        // then groups) keep same-address atomics few.
        if (threadIdx.x == 0) {
            const int per_chunk = a.row_tiles * S;
            const int idx = tile * S + ks;                 // this CTA's index within the chunk
            const int grp = idx / CONSUMER_GROUP;
            const int in_grp = min(CONSUMER_GROUP, per_chunk - grp * CONSUMER_GROUP);
            const int groups = (per_chunk + CONSUMER_GROUP - 1) / CONSUMER_GROUP;
            unsigned* c1 = a.consumed1 + (int64_t)chunk * GROUPS_MAX + grp;
            unsigned last = 0u;
            if (atomicAdd(c1, 1u) == (unsigned)in_grp - 1) {
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
    }

    // Per element: s[n] * (sum over warps) + this slice's EC columns.
    for (int e = threadIdx.x; e < RT * TM; e += DK_THREADS) {
        const int rr = e % RT, mm = e / RT;
        float v = 0.0f;
        if (mm < tm) {
            v = red[0][rr][mm];
#pragma unroll
            for (int w = 1; w < DK_WARPS; ++w) v += red[w][rr][mm];
            v *= s_scale[rr];
            for (int jj = 0; jj < nj; ++jj)
                v = fmaf(us[mm * (a.ec_jr + 1) + jj], bf16_bits_to_f32(Bs[jj * RT + rr]), v);
        }
        if (S == 1) {
            if (mm < tm) {
                const int64_t n = n0 + rr, m = m0 + mm;
                if (a.y_fp32)
                    reinterpret_cast<float*>(a.y)[m * a.N + n] = v;
                else
                    reinterpret_cast<__nv_bfloat16*>(a.y)[m * a.N + n] = __float2bfloat16_rn(v);
            }
        } else {
            ps[mm * RT + rr] = v;
        }
    }
    if (S == 1) return;

    // The S K slices of this row tile (one cluster) meet in distributed shared memory: rank ks sums
    // its share of the tile over ranks 0..S-1 in rank order, then rounds once.
    cluster_sync_all();
    constexpr int RT4 = RT / 4;
    const int total4 = tm * RT4;
    const int per = (total4 + S - 1) / S;
    const int e_beg = ks * per, e_end = min(total4, e_beg + per);
    for (int e = e_beg + threadIdx.x; e < e_end; e += DK_THREADS) {
        const int r4 = e % RT4, mm = e / RT4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int q = 0; q < S; ++q) {
            const float4 p = ld_dsmem_f4(ps + mm * RT + 4 * r4, (unsigned)q);
            v.x += p.x; v.y += p.y; v.z += p.z; v.w += p.w;
        }
        const int64_t m = m0 + mm;
        if (a.y_fp32) {
            reinterpret_cast<float4*>(reinterpret_cast<float*>(a.y) + m * a.N + n0)[r4] = v;
        } else {
            const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
            uint2 pk;
            pk.x = *reinterpret_cast<const uint32_t*>(&lo);
            pk.y = *reinterpret_cast<const uint32_t*>(&hi);
            reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(a.y) + m * a.N + n0)[r4] = pk;
        }
    }
    // Keep this CTA's shared memory alive until every rank has read it.
    cluster_sync_all();
}

template <int NB, int G, int WPW>
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
    gemm_role<NB, G, WPW>(a, rest % a.row_tiles, ks, rest / a.row_tiles, dyn_smem);
}

// ---------------------------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------------------------
size_t decode_dyn_smem_bytes(int nb, int g, int ec_jr, int rank) {
    if (rank <= 0) return 0;
    const size_t gemm = (size_t)ec_jr * 16 * g * 2 + (size_t)8 * nb * (ec_jr + 1) * 4;
    const size_t ec = (size_t)8 * nb * EC_ROWS * 2 + (size_t)DK_WARPS * 8 * (rank + 4) * 4;
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

template <int NB, int G, int WPW>
static cudaError_t launch_t(const DecodeArgs& a, cudaStream_t stream) {
    static_assert(WPW * G <= 8, "weight registers");
    const unsigned grid = (unsigned)(a.ec_ctas + a.row_tiles * a.split * a.mchunks);
    const size_t dyn = decode_dyn_smem_bytes(NB, G, a.ec_jr, a.rank);
    // Static plus dynamic shared memory above 48 KB needs the opt-in attribute (per device).
    static size_t opted[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dyn > 0 && dev >= 0 && dev < 64 && dyn > opted[dev]) {
        cudaError_t e = cudaFuncSetAttribute(w4ec_decode_kernel<NB, G, WPW>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
        if (e != cudaSuccess) return e;
        opted[dev] = dyn;
    }
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
    return cudaLaunchKernelEx(&cfg, w4ec_decode_kernel<NB, G, WPW>, a);
}

cudaError_t launch_decode(const DecodeArgs& a, int nb, int g, int wpw, cudaStream_t stream) {
#define SPEAR_DK_CASE(NB_, G_, W_) \
    if (nb == NB_ && g == G_ && wpw == W_) return launch_t<NB_, G_, W_>(a, stream);
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
