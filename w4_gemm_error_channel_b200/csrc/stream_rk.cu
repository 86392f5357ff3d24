// stream_rk.cu -- the register-path stream-K kernel for decode batches (up to 64 tokens).
//
// SPEAR (Post-Quantization Error-Adaptive Recovery), technical summary section 2.2A: decode is
// bound by the weight stream and the compensator is fused into the low-bit GEMM.  The layer is
//
//   y[m,n] = s[n] * sum_k x[m,k] (q[n,k] - z[n])  +  sum_j u[m,j] B[j,n],
//   u[m,j] = g[m] t[m,j],  t = x A,  g = sigmoid(x w_g + b_g).
//
// Same work split as the tcgen05 stream kernel (stream.cu): 128-row weight tiles cut into K chunks
// of KC codes, the chunks spread evenly over a persistent grid (stream-K), segments processed
// last-first, partial tiles handed to the finalising CTA through the workspace in CTA order, and
// the compensator's x A sliced over the CTAs into exact fixed-point accumulators.  The int4 -> bf16
// conversion goes into registers, straight into mma.sync m16n8k16: at decode sizes a tcgen05 MMA
// over 128 rows x 16 codes costs about the same whatever the token count, so staging converted
// weights for it caps the stream, while the register path leaves the issue slots to the
// conversion.
//
// The weights come in the tile order written by spear_tile_w4 (pack.cu): 8 KiB blocks of 128
// rows x 128 codes, a row's 64 bytes at row * 64, and inside each 32-bit word the nibbles ordered
// so that the mask 0x000F000F after a shift by 4i picks two consecutive codes (2i, 2i + 1).  A unit
// (KC codes of a tile) is then one contiguous bulk copy, every lane's weight load is a
// conflict-free 16-byte read, and x pairs need no permutes.  Per CTA, 10 warps:
//   warp 0      producer: per unit one bulk copy of the weights, then the bf16 x tile (64-code
//               boxes, 128-byte swizzle), both on the stage's one barrier.  The first stages'
//               weights go before the wait on the previous kernel, x after it.  For each finalised
//               tile with a compensator, B[:, tile] into a buffer of its own.
//   warps 1-8   compute: warp w takes 16 * KC/128 weight rows and one 128-code block of each unit
//               (KC = 256: four row quarters x two blocks, exchanged once per segment in a fixed
//               order).  Lane (g, t) holds 32 codes of rows g and g + 8 per row group.  Then the
//               segment's epilogue: partial sum out, or finalisation with the lower CTAs' partial
//               sums, the compensator term E[n, m] = sum_j B[j, n] u[m, j] on mma.sync (B from
//               shared memory by ldmatrix.trans, u split into bf16 hi + lo), y = s[n] D + E.
//   warp 9      the compensator's work item: one 16-column group of x A (or x w_g) over one K
//               slice, A fragments loaded straight into registers; then, in a CTA that finalises
//               a tile, u for every token (off the compute warps' path).
// Every wait is bounded in time; on timeout a bit of the error word is set and the site recorded.
#include "kernels.h"
#include "stream_common.cuh"

namespace spear {

constexpr int RK_THREADS = 320;
constexpr int RK_COMPUTE_WARPS = 8;
constexpr int RK_BLOCK_BYTES = 128 * 64;       // one 128 x 128-code block of the tile order
constexpr int RK_EC_KR_MAX = 1024;             // rows of A per compensator item, at most

// Tagged words (a value and its ready tag in one aligned 64-bit word) and the compensator's
// accumulators are written and read as single 64-bit accesses at the L2 (.cg: never from a
// stale L1 line), so a reader sees a word's tag and value from the same write.  These are plain
// loads and stores: strong (.relaxed.gpu) ones were measured to issue one after another, which
// made a finaliser's reads take one L2 round trip per word.
SPEAR_DEVI void st_cg_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.global.cg.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
SPEAR_DEVI unsigned long long ld_cg_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.global.cg.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
SPEAR_DEVI unsigned long long rk_tagged(float v) { return (1ull << 32) | (unsigned long long)__float_as_uint(v); }
SPEAR_DEVI void named_bar_compute() { asm volatile("bar.sync 1, 256;" ::: "memory"); }   // warps 1-8
SPEAR_DEVI uint4 lds128(uint32_t saddr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(saddr));
    return v;
}
// Full-barrier wait with a cheap first test.
SPEAR_DEVI bool rk_wait(uint64_t* bar, uint32_t parity) {
    return mbar_try(bar, parity) || mbar_wait_ns(bar, parity, SK_WAIT_NS);
}

// u for every token of the tile, by one warp: groups of RK_UT tokens (RK_UT g .. RK_UT g + RK_UT - 1
// for g = first, first + step, ...); lane l reads the accumulator words l, l + 32, ... of every token
// of the group (t, then the gate pre-activation in word r), all at once, until each holds all
// slices (bounded); then u[m][j] = sigmoid(p[m] + b_g) t[m][j] (fp32, zero past M) goes to ubuf
// [rows][ustride].  One round of loads per RK_UT tokens.
constexpr int RK_UT = 4;
SPEAR_DEVI void rk_compute_u(const StreamArgs& a, const unsigned long long* tacc, float* ubuf, int ustride, int rows,
                             int first, int step, int lane) {
    constexpr int WMAX = 5;                              // words per lane and token: r + 1 <= 160
    const int r = a.rank;
    const int nw = (r + 1 + 31) / 32;
    const int gi = r / 32, gl = r % 32;                  // the gate word: chunk gi of lane gl
    const unsigned long long want = (unsigned long long)a.ec_slices;
    for (int m0 = RK_UT * first; m0 < rows; m0 += RK_UT * step) {
        unsigned long long v[RK_UT][WMAX];
        const uint64_t t0 = globaltimer_ns();
        for (;;) {
            bool done = true;
#pragma unroll
            for (int q = 0; q < RK_UT; ++q)
#pragma unroll
                for (int i = 0; i < WMAX; ++i) {
                    const int j = lane + 32 * i;
                    const bool in = i < nw && j <= r && m0 + q < a.M;
                    v[q][i] = in ? ld_cg_u64(tacc_word(tacc, a, m0 + q, j)) : want;
                    done = done && ((v[q][i] & 0xFFull) == want);
                }
            if (__all_sync(0xFFFFFFFFu, done)) break;
            if (__any_sync(0xFFFFFFFFu, globaltimer_ns() - t0 > SK_WAIT_NS)) {
                if (lane == 0) sk_fail(a.err, SK_ERR_FLAG, SITE_EC_TACC, m0);
                break;
            }
            __nanosleep(64);
        }
#pragma unroll
        for (int q = 0; q < RK_UT; ++q) {
            unsigned long long gw = 0;
#pragma unroll
            for (int i = 0; i < WMAX; ++i) gw = i == gi ? v[q][i] : gw;
            gw = __shfl_sync(0xFFFFFFFFu, gw, gl);
            const int m = m0 + q;
            const float gate = m < a.M ? 1.0f / (1.0f + expf(-(__ll2float_rn((long long)gw >> SK_FIX_COUNT_BITS) * (1.0f / SK_FIX_ONE) + a.b_g))) : 0.0f;
#pragma unroll
            for (int i = 0; i < WMAX; ++i) {
                const int j = lane + 32 * i;
                if (i < nw && j < r && m < rows)
                    ubuf[m * ustride + j] = __ll2float_rn((long long)v[q][i] >> SK_FIX_COUNT_BITS) * (1.0f / SK_FIX_ONE) * gate;
            }
        }
    }
}

// The compensator's work item of one CTA (one warp): 16 columns of t = x A (column group grp < r/16)
// or the gate pre-activation p = x w_g (grp == r/16) over rows [k0, k0 + rows) of A, every token.
// Tokens are the M = 16 operand of mma.sync m16n8k16 and the 16 columns two n8 tiles (even and
// odd columns) so that one 32-bit word of a row feeds both; the gate is one n8 tile with w_g in
// column 0.  The fragments of A come straight from global memory in chunks of KS k-steps, the
// first chunk before the wait on the previous kernel (A does not depend on it), x after it.
// Each accumulator word gets one addition per K slice.
SPEAR_DEVI void rk_ec_item(const StreamArgs& a, int64_t k0, int rows, int grp, unsigned long long* tacc) {
    constexpr int KS = 4;                   // k16 steps per chunk
    constexpr int MB = 4;                   // 16-token blocks (M <= 64)
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int r = a.rank;
    const bool gate = grp == r / 16;
    const float lim = SK_FIX_TOTAL / (float)a.ec_slices;
    const int ksteps = rows / 16;
    const int mblocks = (int)((a.M + 15) / 16);
    float de[MB][4], dod[MB][4];
#pragma unroll
    for (int mb = 0; mb < MB; ++mb)
#pragma unroll
        for (int v = 0; v < 4; ++v) de[mb][v] = dod[mb][v] = 0.0f;
    uint32_t w[KS][4];
    auto load_a = [&](int kb) {
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            const int kr = 16 * (kb + kk) + 2 * t;
            const bool in = kb + kk < ksteps;
            if (!gate) {
                const uint16_t* p = a.A + (k0 + kr) * r + 16 * grp + 2 * g;
                w[kk][0] = in ? ldg_u32_nc(p) : 0u;
                w[kk][1] = in ? ldg_u32_nc(p + r) : 0u;
                w[kk][2] = in ? ldg_u32_nc(p + 8 * r) : 0u;
                w[kk][3] = in ? ldg_u32_nc(p + 9 * r) : 0u;
            } else {
                const uint16_t* p = a.wg + k0 + kr;
                w[kk][0] = in && g == 0 ? ldg_u32_nc(p) : 0u;
                w[kk][1] = in && g == 0 ? ldg_u32_nc(p + 8) : 0u;
                w[kk][2] = w[kk][3] = 0u;
            }
        }
    };
    load_a(0);
    pdl_wait_primary();
    for (int kb = 0; kb < ksteps; kb += KS) {
        if (kb > 0) load_a(kb);
#pragma unroll
        for (int mb = 0; mb < MB; ++mb) {
            if (mb >= mblocks) break;
            const int64_t ma = 16 * mb + g, mb8 = ma + 8;
            uint32_t xa[KS][4];
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                const int64_t k = k0 + 16 * (kb + kk) + 2 * t;
                const bool in = kb + kk < ksteps;
                xa[kk][0] = in && ma < a.M ? __ldcg(reinterpret_cast<const unsigned*>(a.x + ma * a.K + k)) : 0u;
                xa[kk][1] = in && mb8 < a.M ? __ldcg(reinterpret_cast<const unsigned*>(a.x + mb8 * a.K + k)) : 0u;
                xa[kk][2] = in && ma < a.M ? __ldcg(reinterpret_cast<const unsigned*>(a.x + ma * a.K + k + 8)) : 0u;
                xa[kk][3] = in && mb8 < a.M ? __ldcg(reinterpret_cast<const unsigned*>(a.x + mb8 * a.K + k + 8)) : 0u;
            }
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                if (kb + kk >= ksteps) break;
                if (!gate) {
                    mma_bf16_16816(de[mb], xa[kk], prmt(w[kk][0], w[kk][1], 0x5410u), prmt(w[kk][2], w[kk][3], 0x5410u));
                    mma_bf16_16816(dod[mb], xa[kk], prmt(w[kk][0], w[kk][1], 0x7632u), prmt(w[kk][2], w[kk][3], 0x7632u));
                } else {
                    mma_bf16_16816(de[mb], xa[kk], w[kk][0], w[kk][1]);
                }
            }
        }
    }
    // Lane (g, t) holds columns 16 grp + 4t + {0, 1, 2, 3} (even tile: +0, +2; odd: +1, +3) of
    // tokens 16 mb + g (entries 0, 1) and 16 mb + g + 8 (entries 2, 3); the gate tile's column 0
    // is in t == 0.
    auto add = [&](int64_t m, int col, float v) {
        if (m >= a.M) return;
        if (!(fabsf(v) < lim)) {
            atomicOr(a.err, SK_ERR_RANGE);
            v = 0.0f;
        }
        const unsigned long long fx = (unsigned long long)__float2ll_rn(v * SK_FIX_ONE);
        red_add_u64(tacc_word(tacc, a, m, col), (fx << SK_FIX_COUNT_BITS) | 1ull);
    };
#pragma unroll
    for (int mb = 0; mb < MB; ++mb) {
        if (mb >= mblocks) break;
        const int64_t ma = 16 * mb + g, mb8 = ma + 8;
        if (!gate) {
            const int c0 = 16 * grp + 4 * t;
            add(ma, c0, de[mb][0]); add(ma, c0 + 1, dod[mb][0]); add(ma, c0 + 2, de[mb][1]); add(ma, c0 + 3, dod[mb][1]);
            add(mb8, c0, de[mb][2]); add(mb8, c0 + 1, dod[mb][2]); add(mb8, c0 + 2, de[mb][3]); add(mb8, c0 + 3, dod[mb][3]);
        } else if (t == 0) {
            add(ma, r, de[mb][0]);
            add(mb8, r, de[mb][2]);
        }
    }
}

template <int NB, int KC>
__global__ void __launch_bounds__(RK_THREADS, (NB <= 4 ? 2 : 1))
w4_stream_rk_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_b,
                    const StreamArgs a) {
    constexpr int BN = 8 * NB;                // token tile
    constexpr int NBLK = KC / 128;            // 128-code blocks per unit
    constexpr int RG = KC / 128;              // 16-row groups per compute warp
    constexpr int WBYTES = NBLK * RK_BLOCK_BYTES;
    constexpr int XBOX = BN * 128;            // one 64-code x box
    constexpr int XBYTES = (KC / 64) * XBOX;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int NST = a.nst;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + a.off_bar);      // weights and x landed
    uint64_t* empty = full + NST;                                         // stage consumed (8 warps)
    uint64_t* bfull = empty + NST;                                        // B slice landed
    uint64_t* bempty = bfull + 1;                                         // B slice consumed (8 warps)
    uint64_t* u_ready = bempty + 1;                                       // u in shared memory

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    const int u0 = sk_u0(a, c), u1 = sk_u0(a, c + 1);
    const int nseg = u0 < u1 ? (u1 - 1) / a.nch - u0 / a.nch + 1 : 0;
    const bool has_ec = a.rank > 0;
    unsigned char* stages = smem;
    unsigned char* bbuf = smem + a.off_b;                 // B[:, tile]: two [r][64] boxes, 128-byte swizzle
    float* ubuf = reinterpret_cast<float*>(smem + a.off_u);   // u fp32 [BN][r + 4]
    const int ustride = a.rank + 4;
    float* red = reinterpret_cast<float*>(smem + a.off_red);  // block exchange [4][2][32][4 NB]
    // Compensator work item of this CTA: K slice c / ec_groups, column group c % ec_groups.
    const bool has_slice = has_ec && c < a.ec_slices * a.ec_groups;
    const int ec_grp = has_slice ? c % a.ec_groups : 0;
    const int64_t ec_k0 = has_slice ? (int64_t)(c / a.ec_groups) * a.ec_kr : 0;
    const int ec_rows = has_slice ? (int)imin64(a.ec_kr, a.K - ec_k0) : 0;

    if (threadIdx.x == 0) {
        prefetch_tmap(&tmap_x);
        if (has_ec) prefetch_tmap(&tmap_b);
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], RK_COMPUTE_WARPS);
        }
        mbar_init(bfull, 1);
        mbar_init(bempty, RK_COMPUTE_WARPS);
        mbar_init(u_ready, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    // The next kernel in the stream may be scheduled now; its own wait still covers this grid.
    pdl_launch_dependents();

    if (warp == 0) {
        // ---------------- producer ----------------
        if (lane == 0) {
            bool ok = true;
            int issued = 0, bnext = 0;
            const int64_t nblk_row = a.K / 128;                   // blocks per tile
            auto stage_of = [&](int sq) { return stages + (size_t)(sq % NST) * a.stage_bytes; };
            // Weights of unit sq (its barrier expects the x bytes as well).
            auto issue_w = [&](int sq, int tile, int kci) {
                const int s = sq % NST;
                mbar_arrive_expect_tx(&full[s], (uint32_t)(WBYTES + XBYTES));
                bulk_load(stage_of(sq), a.packed + ((int64_t)tile * nblk_row + (int64_t)kci * NBLK) * RK_BLOCK_BYTES,
                          (uint32_t)WBYTES, &full[s]);
                issued = sq + 1;
            };
            auto issue_x = [&](int sq, int kci) {
                const int s = sq % NST;
                unsigned char* xs = stage_of(sq) + WBYTES;
#pragma unroll
                for (int b = 0; b < KC / 64; ++b) tma_load_2d(xs + b * XBOX, &tmap_x, kci * KC + 64 * b, 0, &full[s]);
            };
            // B slice of the fe-th finalised tile (processing order).
            auto fin_tile = [&](int fe) {
                int k = 0;
                for (int i = 0; i < nseg; ++i) {
                    const SkSeg sg = sk_seg(a, u0, u1, i);
                    if (sg.fin && k++ == fe) return sg.tile;
                }
                return 0;
            };
            auto issue_b = [&](int fe) {
                const int tile = fin_tile(fe);
                mbar_arrive_expect_tx(bfull, (uint32_t)(2 * a.rank * 128));
                tma_load_2d(bbuf, &tmap_b, tile * 128, 0, bfull);
                tma_load_2d(bbuf + a.rank * 128, &tmap_b, tile * 128 + 64, 0, bfull);
            };
            int nfin = 0;                     // finalised tiles of this CTA (each needs its B slice)
            if (has_ec)
                for (int i = 0; i < nseg; ++i) nfin += sk_seg(a, u0, u1, i).fin ? 1 : 0;
            // Weights of the first stages and the first B slice before the wait; x after it.
            int seq = 0;
            for (int i = 0; i < nseg && seq < NST; ++i) {
                const SkSeg sg = sk_seg(a, u0, u1, i);
                for (int kci = sg.kb; kci < sg.ke && seq < NST; ++kci, ++seq) issue_w(seq, sg.tile, kci);
            }
            if (nfin > 0) issue_b(bnext++);
            pdl_wait_primary();
            seq = 0;
            for (int i = 0; i < nseg && ok; ++i) {
                const SkSeg sg = sk_seg(a, u0, u1, i);
                for (int kci = sg.kb; kci < sg.ke && ok; ++kci, ++seq) {
                    if (seq < NST) {
                        issue_x(seq, kci);
                        continue;
                    }
                    // Wait for the stage to be consumed; meanwhile load the next B slice as soon as
                    // the previous one is released (an epilogue may be waiting for it).
                    const int s = seq % NST;
                    const uint32_t ph = ((seq / NST) - 1) & 1;
                    const uint64_t t0 = globaltimer_ns();
                    for (uint32_t it = 0;; ++it) {
                        if (mbar_try(&empty[s], ph)) break;
                        if (bnext < nfin && mbar_try(bempty, (bnext - 1) & 1)) issue_b(bnext++);
                        if ((it & 63) == 63 && globaltimer_ns() - t0 > SK_WAIT_NS) {
                            sk_fail(a.err, SK_ERR_MBAR, SITE_PROD_SEMPTY, seq);
                            ok = false;
                            break;
                        }
                    }
                    if (!ok) break;
                    issue_w(seq, sg.tile, kci);
                    issue_x(seq, kci);
                }
            }
            while (ok && bnext < nfin) {
                if (!mbar_wait_ns(bempty, (bnext - 1) & 1, SK_WAIT_NS)) {
                    sk_fail(a.err, SK_ERR_MBAR, SITE_PROD_SEMPTY, -1);
                    break;
                }
                issue_b(bnext++);
            }
            // Never leave with copies in flight: wait (bounded) for the last copies of every stage.
            // Weights and x of a unit go out together once the first NST units' x are out, and
            // a wait that gives up stops the loop before a unit's weights, so every issued stage
            // also got its x.
            for (int s = 0; s < NST && s < issued; ++s) {
                const int last = s + (issued - 1 - s) / NST * NST;
                if (!mbar_wait_ns(&full[s], (last / NST) & 1, SK_WAIT_NS)) sk_fail(a.err, SK_ERR_MBAR, SITE_EXIT, last);
            }
            if (bnext > 0 && !mbar_wait_ns(bfull, (bnext - 1) & 1, SK_WAIT_NS)) sk_fail(a.err, SK_ERR_MBAR, SITE_EXIT, -2);
        }
    } else if (warp <= RK_COMPUTE_WARPS) {
        // ---------------- compute warps ----------------
        const int cw = warp - 1;
        const int g = lane >> 2, t = lane & 3;
        const int blk = KC == 256 ? cw >> 2 : 0;              // 128-code block of each unit
        const int rgb = KC == 256 ? 2 * (cw & 3) : cw;         // first 16-row group of this warp
        // Lane-constant shared-memory offsets in a stage: weights of row 16 rgb + g (row group j:
        // + 1024 j; rows + 8: + 512), and for word w of the lane's 16 bytes (codes 16 t + 8 w, or
        // 64 + 16 t + 8 (w - 2) for w >= 2, in the tile order) the x chunk (box 2 blk + w/2, chunk
        // 2 t + w % 2) of token g (token 8 b + g: + 1024 b), 128-byte swizzle on the token row.  The
        // four lanes t of a quarter-warp read four different chunks of one box: no bank conflict.
        const uint32_t wl = (uint32_t)(blk * RK_BLOCK_BYTES + (16 * rgb + g) * 64 + 16 * t);
        uint32_t xl[4];
#pragma unroll
        for (int w = 0; w < 4; ++w)
            xl[w] = (uint32_t)(WBYTES + (2 * blk + (w >> 1)) * XBOX + g * 128 + (((2 * t + (w & 1)) ^ g) << 4));
        const uint32_t sm_stages = smem_u32(stages);
        const int rbase0 = 16 * rgb + g;                       // tile row of (j = 0, h = 0)
        // Zero-points of the first segment, requested before the wait on the previous kernel.
        unsigned short zn[RG][2];
        if (nseg > 0) {
            const int64_t tr = (int64_t)sk_seg(a, u0, u1, 0).tile * 128 + rbase0;
#pragma unroll
            for (int j = 0; j < RG; ++j)
#pragma unroll
                for (int h = 0; h < 2; ++h) zn[j][h] = __half_as_ushort(a.zero[tr + 16 * j + 8 * h]);
        }
        // Every wait below depends on x, which follows the previous kernel: wait for it first.
        pdl_wait_primary();
        bool ok = true;
        int s = 0;
        uint32_t ph = 0;
        int fe = 0;
        bool u_seen = false;
        for (int i = 0; i < nseg; ++i) {
            const SkSeg sg = sk_seg(a, u0, u1, i);
            uint32_t zb[RG][2];
#pragma unroll
            for (int j = 0; j < RG; ++j)
#pragma unroll
                for (int h = 0; h < 2; ++h) zb[j][h] = zero_bias_bf16x2((uint32_t)__half2float(__ushort_as_half(zn[j][h])));
            // The next segment's zero-points, in flight during this one.
            if (i + 1 < nseg) {
                const int64_t tr = (int64_t)sk_seg(a, u0, u1, i + 1).tile * 128 + rbase0;
#pragma unroll
                for (int j = 0; j < RG; ++j)
#pragma unroll
                    for (int h = 0; h < 2; ++h) zn[j][h] = __half_as_ushort(a.zero[tr + 16 * j + 8 * h]);
            }
            // Scales of the rows this warp finalises (KC = 256: row group rgb + blk), in flight
            // during the main loop.
            uint32_t s_pair = 0;                                 // fp16 scales of rows n_lo, n_lo + 8
            if (sg.fin) {
                const int64_t n = (int64_t)sg.tile * 128 + 16 * (KC == 256 ? rgb + blk : rgb) + g;
                s_pair = (uint32_t)__half_as_ushort(a.scale[n]) | ((uint32_t)__half_as_ushort(a.scale[n + 8]) << 16);
            }
            // One 8-token tile: each word pair's second MMA goes to a second set of accumulators, so
            // consecutive MMAs do not wait on one another (added together at the segment end).
            constexpr bool SPLIT = NB == 1;
            float acc[RG][NB][4], acc2[RG][NB][4];
#pragma unroll
            for (int j = 0; j < RG; ++j)
#pragma unroll
                for (int b = 0; b < NB; ++b)
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[j][b][q] = acc2[j][b][q] = 0.0f;

            for (int kci = sg.kb; kci < sg.ke; ++kci) {
                if (ok && !rk_wait(&full[s], ph)) {
                    sk_fail(a.err, SK_ERR_MBAR, SITE_CVT_WFULL, kci);
                    ok = false;
                }
                const uint32_t st = sm_stages + (uint32_t)(s * a.stage_bytes);
                uint4 wa[RG], wb[RG];
#pragma unroll
                for (int j = 0; j < RG; ++j) {
                    wa[j] = lds128(st + wl + 1024 * j);
                    wb[j] = lds128(st + wl + 1024 * j + 512);
                }
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    // x codes of word w, every token: natural bf16 pairs.
                    uint4 xv[NB];
#pragma unroll
                    for (int b = 0; b < NB; ++b) xv[b] = lds128(st + xl[w] + 1024 * b);
#pragma unroll
                    for (int j = 0; j < RG; ++j) {
                        const uint32_t qa = w == 0 ? wa[j].x : w == 1 ? wa[j].y : w == 2 ? wa[j].z : wa[j].w;
                        const uint32_t qb = w == 0 ? wb[j].x : w == 1 ? wb[j].y : w == 2 ? wb[j].z : wb[j].w;
                        uint32_t ra[4], rb[4];
                        cvt_w4_pairs_i_i4(qa, zb[j][0], ra);
                        cvt_w4_pairs_i_i4(qb, zb[j][1], rb);
                        const uint32_t af0[4] = {ra[0], rb[0], ra[1], rb[1]};
                        const uint32_t af1[4] = {ra[2], rb[2], ra[3], rb[3]};
#pragma unroll
                        for (int b = 0; b < NB; ++b) {
                            mma_bf16_16816(acc[j][b], af0, xv[b].x, xv[b].y);
                            mma_bf16_16816(SPLIT ? acc2[j][b] : acc[j][b], af1, xv[b].z, xv[b].w);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
                if (++s == NST) {
                    s = 0;
                    ph ^= 1u;
                }
            }

            if constexpr (SPLIT) {
#pragma unroll
                for (int j = 0; j < RG; ++j)
#pragma unroll
                    for (int b = 0; b < NB; ++b)
#pragma unroll
                        for (int q = 0; q < 4; ++q) acc[j][b][q] += acc2[j][b][q];
            }
            // ---- this warp's final sums for one 16-row group (KC = 256: blocks exchanged) ----
            float fin[NB][4];
            if constexpr (KC == 256) {
                const int qd = cw & 3, h = cw >> 2;
                float* give = red + ((qd * 2 + (1 - h)) * 32 + lane) * (4 * NB);   // the row group handed over
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    // acc[1 - h][b], selected without indexing the array by a run-time value
                    const float v0 = h ? acc[0][b][0] : acc[1][b][0], v1 = h ? acc[0][b][1] : acc[1][b][1];
                    const float v2 = h ? acc[0][b][2] : acc[1][b][2], v3 = h ? acc[0][b][3] : acc[1][b][3];
                    *reinterpret_cast<float4*>(give + 4 * b) = make_float4(v0, v1, v2, v3);
                }
                named_bar_compute();
                const float* take = red + ((qd * 2 + h) * 32 + lane) * (4 * NB);
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    const float4 o = *reinterpret_cast<const float4*>(take + 4 * b);
                    // Fixed order: block 0's sum, then block 1's.
                    if (h == 0) {
                        fin[b][0] = acc[0][b][0] + o.x; fin[b][1] = acc[0][b][1] + o.y;
                        fin[b][2] = acc[0][b][2] + o.z; fin[b][3] = acc[0][b][3] + o.w;
                    } else {
                        fin[b][0] = o.x + acc[1][b][0]; fin[b][1] = o.y + acc[1][b][1];
                        fin[b][2] = o.z + acc[1][b][2]; fin[b][3] = o.w + acc[1][b][3];
                    }
                }
                named_bar_compute();              // the exchange buffer is free again
            } else {
#pragma unroll
                for (int b = 0; b < NB; ++b)
#pragma unroll
                    for (int q = 0; q < 4; ++q) fin[b][q] = acc[0][b][q];
            }

            // ---- epilogue: rows 16 rgf + g (+ 8) of the tile; tokens 8 b + 2 t (+ 1) ----
            const int rgf = KC == 256 ? rgb + blk : rgb;
            const int row0 = 16 * rgf + g;
            const int64_t n_lo = (int64_t)sg.tile * 128 + row0;
            unsigned long long* parts = reinterpret_cast<unsigned long long*>(a.partial);
            if (!sg.fin) {
                // Partial sum of a tile that a higher CTA finalises: [BN][128] 64-bit words, the fp32
                // value in the low half and the ready tag 1 in the high half, each one store.  The
                // reader polls the words themselves and zeroes them after use: no flag, no fence.
                unsigned long long* own = parts + (size_t)c * BN * 128;
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    const int m = 8 * b + 2 * t;
                    st_cg_u64(own + m * 128 + row0, rk_tagged(fin[b][0]));
                    st_cg_u64(own + (m + 1) * 128 + row0, rk_tagged(fin[b][1]));
                    st_cg_u64(own + m * 128 + row0 + 8, rk_tagged(fin[b][2]));
                    st_cg_u64(own + (m + 1) * 128 + row0 + 8, rk_tagged(fin[b][3]));
                }
                continue;
            }
            const float s_lo = __half2float(__ushort_as_half((unsigned short)(s_pair & 0xFFFFu)));
            const float s_hi = __half2float(__ushort_as_half((unsigned short)(s_pair >> 16)));
            const int c_lo = sg.kb > 0 ? sk_cta_of(a, sg.tile * a.nch) : c;
            if (c_lo < c) {
                // Lower CTAs computed the tile's first chunks: add their partial sums in CTA order,
                // then this CTA's own.  PB CTAs' words are polled at a time, all loads in flight
                // together, until their tags say ready (bounded); each lane zeroes what it read.
                constexpr int PB = NB <= 1 ? 4 : (NB <= 2 ? 2 : 1);
                float p[NB][4];
                for (int base = c_lo; base < c; base += PB) {
                    unsigned long long q[PB][NB][4];
                    const uint64_t t0 = globaltimer_ns();
                    for (;;) {
                        bool ready = true;
#pragma unroll
                        for (int k = 0; k < PB; ++k) {
                            const bool in = base + k < c;
                            const unsigned long long* pp = parts + (size_t)(in ? base + k : base) * BN * 128;
                            constexpr unsigned long long kReady = 1ull << 32;
#pragma unroll
                            for (int b = 0; b < NB; ++b) {
                                const int m = 8 * b + 2 * t;
                                q[k][b][0] = in ? ld_cg_u64(pp + m * 128 + row0) : kReady;
                                q[k][b][1] = in ? ld_cg_u64(pp + (m + 1) * 128 + row0) : kReady;
                                q[k][b][2] = in ? ld_cg_u64(pp + m * 128 + row0 + 8) : kReady;
                                q[k][b][3] = in ? ld_cg_u64(pp + (m + 1) * 128 + row0 + 8) : kReady;
#pragma unroll
                                for (int v = 0; v < 4; ++v) ready = ready && (q[k][b][v] >> 32) == 1ull;
                            }
                        }
                        if (ready) break;
                        if (globaltimer_ns() - t0 > SK_WAIT_NS) {
                            sk_fail(a.err, SK_ERR_FLAG, SITE_EPI_FLAG, base);
                            break;
                        }
                        __nanosleep(32);
                    }
#pragma unroll
                    for (int k = 0; k < PB; ++k) {
                        if (base + k >= c) break;
                        unsigned long long* pp = parts + (size_t)(base + k) * BN * 128;
#pragma unroll
                        for (int b = 0; b < NB; ++b) {
                            const int m = 8 * b + 2 * t;
#pragma unroll
                            for (int v = 0; v < 4; ++v) {
                                const float x = __uint_as_float((uint32_t)q[k][b][v]);
                                p[b][v] = (base + k == c_lo) ? x : p[b][v] + x;
                            }
                            st_cg_u64(pp + m * 128 + row0, 0ull);
                            st_cg_u64(pp + (m + 1) * 128 + row0, 0ull);
                            st_cg_u64(pp + m * 128 + row0 + 8, 0ull);
                            st_cg_u64(pp + (m + 1) * 128 + row0 + 8, 0ull);
                        }
                    }
                }
#pragma unroll
                for (int b = 0; b < NB; ++b)
#pragma unroll
                    for (int v = 0; v < 4; ++v) fin[b][v] = p[b][v] + fin[b][v];
            }
            float e[NB][4];
#pragma unroll
            for (int b = 0; b < NB; ++b) e[b][0] = e[b][1] = e[b][2] = e[b][3] = 0.0f;
            if (has_ec) {
                if (!u_seen) {
                    // u for every token, formed by the compensator's warp once its item is done.
                    if (!mbar_wait_ns(u_ready, 0, SK_WAIT_NS)) {
                        if (lane == 0) sk_fail(a.err, SK_ERR_MBAR, SITE_MMA_UREADY, fe);
                        ok = false;
                    }
                    u_seen = true;
                }
                // E[n, m] = sum_j B[j, n] u[m, j]: B^T fragments by ldmatrix.trans from the B buffer
                // ([j][64] boxes, 128-byte swizzle), u as bf16 hi + lo parts.
                if (ok && !mbar_wait_ns(bfull, fe & 1, SK_WAIT_NS)) {
                    sk_fail(a.err, SK_ERR_MBAR, SITE_MMA_BUNIT, fe);
                    ok = false;
                }
                const int mat = lane >> 3, rr = lane & 7;
                const int nb = 16 * rgf + (mat & 1) * 8;                 // first row of this lane's 8x8 matrix
                const unsigned char* bbox = bbuf + (nb >> 6) * (a.rank * 128);
                for (int j0 = 0; j0 < a.rank; j0 += 16) {
                    const int jr = j0 + (mat >> 1) * 8 + rr;
                    uint32_t af[4];
                    ldsm_x4_trans(af, bbox + jr * 128 + (((((nb & 63) >> 3) ^ (jr & 7)) & 7) << 4));
#pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        const float* ur = ubuf + (8 * b + g) * ustride + j0 + 2 * t;
                        const float2 u01 = *reinterpret_cast<const float2*>(ur);
                        const float2 u89 = *reinterpret_cast<const float2*>(ur + 8);
                        const __nv_bfloat162 h0 = __floats2bfloat162_rn(u01.x, u01.y);
                        const __nv_bfloat162 h1 = __floats2bfloat162_rn(u89.x, u89.y);
                        const __nv_bfloat162 l0 = __floats2bfloat162_rn(u01.x - __low2float(h0), u01.y - __high2float(h0));
                        const __nv_bfloat162 l1 = __floats2bfloat162_rn(u89.x - __low2float(h1), u89.y - __high2float(h1));
                        mma_bf16_16816(e[b], af, *reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1));
                        mma_bf16_16816(e[b], af, *reinterpret_cast<const uint32_t*>(&l0), *reinterpret_cast<const uint32_t*>(&l1));
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bempty);
                ++fe;
            }
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                const int64_t m = 8 * b + 2 * t;
                const float y00 = fmaf(s_lo, fin[b][0], e[b][0]), y01 = fmaf(s_lo, fin[b][1], e[b][1]);
                const float y10 = fmaf(s_hi, fin[b][2], e[b][2]), y11 = fmaf(s_hi, fin[b][3], e[b][3]);
                if (a.y_fp32) {
                    float* y = reinterpret_cast<float*>(a.y);
                    if (m < a.M) { y[m * a.N + n_lo] = y00; y[m * a.N + n_lo + 8] = y10; }
                    if (m + 1 < a.M) { y[(m + 1) * a.N + n_lo] = y01; y[(m + 1) * a.N + n_lo + 8] = y11; }
                } else {
                    __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(a.y);
                    if (m < a.M) { y[m * a.N + n_lo] = __float2bfloat16_rn(y00); y[m * a.N + n_lo + 8] = __float2bfloat16_rn(y10); }
                    if (m + 1 < a.M) {
                        y[(m + 1) * a.N + n_lo] = __float2bfloat16_rn(y01);
                        y[(m + 1) * a.N + n_lo + 8] = __float2bfloat16_rn(y11);
                    }
                }
            }
        }
    } else {
        // ---------------- compensator (warp 9) ----------------
        unsigned long long* tacc = reinterpret_cast<unsigned long long*>(a.tacc);
        if (has_slice) rk_ec_item(a, ec_k0, ec_rows, ec_grp, tacc);
        else pdl_wait_primary();
        // In a CTA that finalises a tile: u for every token while the compute warps still stream
        // weights, off their path; then this CTA's read of the accumulators is retired.
        bool fin_any = false;
        for (int i = 0; i < nseg; ++i) fin_any = fin_any || sk_seg(a, u0, u1, i).fin;
        if (has_ec && fin_any) {
            rk_compute_u(a, tacc, ubuf, ustride, BN, 0, 1, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(u_ready);
            ec_retire(a, tacc);
        }
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------------------------
static int rk_align(int v, int a) { return (v + a - 1) / a * a; }

bool stream_rk_configure(StreamArgs& a, int bn, int kc, bool deep) {
    if (!(bn == 8 || bn == 16 || bn == 32 || bn == 64) || !(kc == 128 || kc == 256)) return false;
    if (a.K % kc != 0 || a.N % 128 != 0 || a.M < 1 || a.M > bn || a.rank > 128) return false;
    if (bn == 64 && !deep) return false;             // 64 tokens need the registers of one CTA per SM
    a.kc = kc;
    a.nch = (int)(a.K / kc);
    a.ntiles = (int)(a.N / 128);
    a.units = a.ntiles * a.nch;
    if (a.grid < 1 || a.grid > a.units || a.grid > (int)STREAM_GRID_MAX) return false;
    a.stage_bytes = rk_align((kc / 128) * RK_BLOCK_BYTES + (kc / 64) * bn * 128, 1024);
    a.jb = a.nbu = 0;
    a.ec_kr = a.ec_slices = 0;
    a.ec_groups = 1;
    int b_bytes = 0, u_bytes = 0, a_bytes = 0, wg_bytes = 0, g_bytes = 0;
    if (a.rank > 0) {
        // (K slice, column group) items, one per CTA: as many K slices as the grid allows
        // (at most 255 for the 8-bit count), rows a multiple of 16, at most RK_EC_KR_MAX.
        a.ec_groups = a.rank / 16 + 1;
        int64_t slices = a.grid / a.ec_groups;
        if (slices > 255) slices = 255;
        if (slices < 1) return false;
        int64_t kr = (a.K + slices - 1) / slices;
        kr = (kr + 15) / 16 * 16;
        if (kr > RK_EC_KR_MAX) return false;
        a.ec_kr = (int)kr;
        a.ec_slices = (int)((a.K + kr - 1) / kr);
        if ((int64_t)a.ec_slices * a.ec_groups > a.grid) return false;
        b_bytes = 2 * a.rank * 128;
        u_bytes = rk_align(bn * (a.rank + 4) * 4, 128);
        a_bytes = wg_bytes = 0;               // the compensator's warp reads A and w_g into registers
    }
    const int red_bytes = kc == 256 ? 4 * 2 * 32 * 4 * (bn / 8) * 4 : 0;
    const int bar_bytes = 8 * (2 * 16 + 6) + 16;
    const int fixed = b_bytes + u_bytes + a_bytes + wg_bytes + g_bytes + red_bytes + bar_bytes + 1024;
    const int budget = deep ? (int)SMEM_OPTIN_MAX : 110 * 1024;
    int nst = (budget - fixed) / a.stage_bytes;
    if (nst > 16) nst = 16;
    if (nst < 2) return false;
    a.nst = nst;
    a.na = 0;
    a.tmem_cols = 0;
    a.off_b = nst * a.stage_bytes;                    // 1024-aligned (stages are)
    a.off_u = a.off_b + rk_align(b_bytes, 1024);
    a.off_a = a.off_u + u_bytes;
    a.off_wg = a.off_a + a_bytes;
    a.off_g = a.off_wg + wg_bytes;
    a.off_red = a.off_g + g_bytes;
    a.off_bar = a.off_red + red_bytes;
    a.smem_bytes = a.off_bar + bar_bytes + 1024;
    if (a.smem_bytes > (int)SMEM_OPTIN_MAX) return false;
    // The deep ring keeps one CTA per SM: reserve more than half of the SM's shared memory.
    if (deep && a.smem_bytes < 116 * 1024) a.smem_bytes = 116 * 1024;
    a.finalizers = 0;
    for (int cc = 0; cc < a.grid; ++cc) {
        const int v0 = (int)((int64_t)a.units * cc / a.grid), v1 = (int)((int64_t)a.units * (cc + 1) / a.grid);
        if (v0 < v1 && (v1 % a.nch == 0 || (v1 - 1) / a.nch > v0 / a.nch)) ++a.finalizers;
    }
    a.nfin = 0;        // counted per CTA on the device
    return true;
}

template <int NB, int KC>
static cudaError_t launch_rk_t(const StreamArgs& a, cudaStream_t stream) {
    CUtensorMap mx, mb;
    if (!make_map_2d(&mx, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.K, (uint64_t)a.M, 64, 8 * NB,
                     CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (a.rank > 0) {
        if (!make_map_2d(&mb, a.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.N, (uint64_t)a.rank, 64,
                         (uint32_t)a.rank, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    } else {
        mb = mx;   // unused
    }
    static std::once_flag once[kMaxDevices];
    static cudaError_t opt_status[kMaxDevices];
    cudaError_t oe = opt_in_smem((const void*)w4_stream_rk_kernel<NB, KC>, SMEM_OPTIN_MAX, once, opt_status);
    if (oe != cudaSuccess) return oe;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.grid);
    cfg.blockDim = dim3(RK_THREADS);
    cfg.dynamicSmemBytes = (size_t)a.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, w4_stream_rk_kernel<NB, KC>, mx, mb, a);
}

cudaError_t launch_stream_rk(const StreamArgs& a, int bn, cudaStream_t stream) {
    // Bulk copies of the tile-ordered weights need a 16-byte aligned base.
    if ((reinterpret_cast<uintptr_t>(a.packed) & 15u) != 0) return cudaErrorInvalidValue;
#define SPEAR_RK(NB_)                                                                   \
    if (bn == 8 * NB_) return a.kc == 256 ? launch_rk_t<NB_, 256>(a, stream) : launch_rk_t<NB_, 128>(a, stream);
    SPEAR_RK(1) SPEAR_RK(2) SPEAR_RK(4) SPEAR_RK(8)
#undef SPEAR_RK
    return cudaErrorInvalidValue;
}

}  // namespace spear
