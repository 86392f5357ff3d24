// stream.cu -- the small-batch kernel: a persistent, stream-K, TMA + tcgen05 W4 GEMM with the gated
// compensator fused in, for batches of up to 64 tokens (decode and small chunks).
//
// SPEAR (Post-Quantization Error-Adaptive Recovery), technical summary section 2.2A: decode is
// bound by the weight stream, and the compensator is fused into the low-bit GEMM so that the layer
// is one kernel.  The layer is
//
//   y[m,n] = s[n] * sum_k x[m,k] (q[n,k] - z[n])  +  sum_j u[m,j] B[j,n],
//   u[m,j] = g[m] t[m,j],  t = x A,  g = sigmoid(x w_g + b_g).
//
// Work.  The weights are cut into tiles of 128 rows (the MMA's M and the 128 TMEM lanes) and each
// tile into K chunks of KC codes; the chunks, tile-major, form one list of units, and CTA c of the
// P in the grid takes units [U c / P, U (c + 1) / P).  Every SM therefore streams the same number
// of weight bytes whatever N is (stream-K), and a CTA's range covers a few "segments": runs of
// chunks of one tile.  A CTA processes its segments last-first (each one forward in K):
//   * its last segment, if it stops inside a tile, leaves a partial sum: it is written to the
//     workspace (fp32) with a release flag, early in the kernel;
//   * every other segment ends at a tile's last chunk, so this CTA finalises that tile: a whole
//     tile needs nothing else; a tile that started in lower CTAs adds their partial sums (already
//     written: they were those CTAs' first work), in CTA order, then its own.  Sums are in a
//     fixed order, so the output does not depend on timing.
// Per CTA, 11 warps:
//   warp 0      TMA producer: per unit, the packed tile (128 rows x KC/2 bytes, swizzled) and the
//               bf16 x tile (tokens x KC codes, 64-code boxes, 128-byte swizzle) into a ring of
//               stages; the weights of the first stages are requested before the wait on the
//               previous kernel (programmatic dependent launch), x after it.  For a finalised
//               tile with a compensator it then brings B[:, tile] (MN-major) through the ring.
//   warp 1      allocates TMEM and issues tcgen05.mma (one thread): D[n, m] += (q - z)[n, k] x[m, k]
//               with the converted weights in TMEM (A operand) and x in shared memory; for a
//               finalised tile E[n, m] = sum_j B[j, n] u[m, j] (u split into bf16 hi + lo parts).
//   warps 2-9   convert 64-code sub-chunks of the packed tile into exact bf16 (q - z) and store
//               them to TMEM (tcgen05.st, one weight row per thread; the two groups of four warps
//               take alternate sub-chunks), then run the epilogue of each segment:
//               y = s[n] (sum of partials) + E, rounded once.
//   warp 10     the compensator's x A: CTA c takes rows [c ec_kr, (c + 1) ec_kr) of A and w_g
//               (bulk-copied before the wait), computes its partial t and gate pre-activation on
//               mma.sync and adds them, exactly, into the int64 fixed-point accumulators of the
//               workspace (the low 8 bits of every word count the slices added).  A CTA that
//               finalises a tile then reads all the words once they are complete (bounded wait),
//               forms u = sigmoid(p + b_g) t and stores it, split in two bf16 parts, as the MMA
//               operand of the E term.  The last reader clears the accumulators.
// Every mbarrier and flag wait is bounded; on timeout the kernel sets a bit of the error word and
// stops waiting (its output is then undefined).
#include "kernels.h"
#include "stream_common.cuh"

namespace spear {

constexpr int SK_THREADS = 352;
SPEAR_DEVI void named_bar_conv() { asm volatile("bar.sync 1, 256;" ::: "memory"); }   // warps 2-9

// 32 x 32-bit TMEM columns of the converted weights: 64 codes of one row, natural order
// (column c holds codes 2c and 2c + 1).
SPEAR_DEVI void convert_row64(const unsigned char* stage, uint32_t row, uint32_t sub, uint32_t pitch, uint32_t zb,
                              uint32_t out[32]) {
    const uint4 w0 = *reinterpret_cast<const uint4*>(stage + swz_off(row, 2 * sub, pitch));
    const uint4 w1 = *reinterpret_cast<const uint4*>(stage + swz_off(row, 2 * sub + 1, pitch));
    cvt_w4_pairs_natural(w0.x, zb, out);
    cvt_w4_pairs_natural(w0.y, zb, out + 4);
    cvt_w4_pairs_natural(w0.z, zb, out + 8);
    cvt_w4_pairs_natural(w0.w, zb, out + 12);
    cvt_w4_pairs_natural(w1.x, zb, out + 16);
    cvt_w4_pairs_natural(w1.y, zb, out + 20);
    cvt_w4_pairs_natural(w1.z, zb, out + 24);
    cvt_w4_pairs_natural(w1.w, zb, out + 28);
}

// ---------------------------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------------------------
template <int BN>
__global__ void __launch_bounds__(SK_THREADS, 2)
w4_stream_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                 const __grid_constant__ CUtensorMap tmap_b, const StreamArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int NST = a.nst, NA = a.na;
    uint64_t* wfull = reinterpret_cast<uint64_t*>(smem + a.off_bar);   // weights (or B slice) landed
    uint64_t* xfull = wfull + NST;                                       // x landed (a plain arrive for B units)
    uint64_t* sempty = xfull + NST;                                      // stage consumed by the MMAs
    uint64_t* afull = sempty + NST;                                      // converted sub-chunk in TMEM
    uint64_t* aempty = afull + NA;                                       // TMEM sub-chunk slot free again
    uint64_t* dfull = aempty + NA;                                       // [2] accumulator complete
    uint64_t* dempty = dfull + 2;                                        // [2] accumulator read out
    uint64_t* efull = dempty + 2;                                        // EC accumulator complete
    uint64_t* eempty = efull + 1;                                        // EC accumulator read out
    uint64_t* u_ready = eempty + 1;                                      // u stored in shared memory
    uint64_t* ec_bar = u_ready + 1;                                      // A and w_g slices landed
    uint64_t* mma_done = ec_bar + 1;                                     // every MMA retired (exit path)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    const int u0 = sk_u0(a, c), u1 = sk_u0(a, c + 1);
    const int nseg = u0 < u1 ? (u1 - 1) / a.nch - u0 / a.nch + 1 : 0;
    const bool has_ec = a.rank > 0;
    // This CTA finalises a tile iff its range holds some tile's last chunk.
    const bool finalizes = u0 < u1 && (u1 % a.nch == 0 || (u1 - 1) / a.nch > u0 / a.nch);
    const int pitch = a.kc / 2;                    // bytes per weight row in a stage
    const int subs = a.kc / 64;                    // 64-code sub-chunks per unit
    unsigned char* stages = smem;
    unsigned char* ubuf = smem + a.off_u;          // u hi then lo: [2][r / 64 blocks][BN][128 B]
    const int ublk = (a.rank + 63) / 64;
    uint16_t* As = reinterpret_cast<uint16_t*>(smem + a.off_a);
    uint16_t* wgs = reinterpret_cast<uint16_t*>(smem + a.off_wg);
    const bool has_slice = has_ec && c < a.ec_slices;
    const int64_t ec_k0 = (int64_t)c * a.ec_kr;
    const int ec_rows = has_slice ? (int)imin64(a.ec_kr, a.K - ec_k0) : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&wfull[s], 1);
            mbar_init(&xfull[s], 1);
            mbar_init(&sempty[s], 1);
        }
        for (int s = 0; s < NA; ++s) {
            mbar_init(&afull[s], 128);     // the four warps of one converter group
            mbar_init(&aempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&dfull[b], 1);
            mbar_init(&dempty[b], 256);    // both converter groups
        }
        mbar_init(efull, 1);
        mbar_init(eempty, 256);
        mbar_init(u_ready, 1);
        mbar_init(ec_bar, 1);
        mbar_init(mma_done, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(a.tmem_cols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // The next kernel in the stream may be scheduled now; its own wait still covers this grid.
    pdl_launch_dependents();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t tmem_a = tmem_base;                         // NA x 32 columns: converted sub-chunks
    const uint32_t tmem_d = tmem_base + 32 * NA;               // [2] x BN: main accumulators
    const uint32_t tmem_e = tmem_d + 2 * BN;                   // BN: compensator accumulator

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            bool ok = true;
            int seq = 0;
            int issued_w = 0, issued_x = 0;   // loads are issued in sequence order
            auto issue_w = [&](int sq, int tile, int kci, int bu) {
                const int s = sq % NST;
                unsigned char* st = stages + (size_t)s * a.stage_bytes;
                if (bu < 0) {
                    mbar_arrive_expect_tx(&wfull[s], (uint32_t)(SK_ROWS * pitch));
                    tma_load_2d(st, &tmap_w, kci * pitch, tile * SK_ROWS, &wfull[s]);
                } else {
                    mbar_arrive_expect_tx(&wfull[s], (uint32_t)(2 * a.jb * 128));
                    tma_load_2d(st, &tmap_b, tile * SK_ROWS, bu * a.jb, &wfull[s]);
                    tma_load_2d(st + a.jb * 128, &tmap_b, tile * SK_ROWS + 64, bu * a.jb, &wfull[s]);
                }
                issued_w = sq + 1;
            };
            auto issue_x = [&](int sq, int kci, int bu) {
                const int s = sq % NST;
                if (bu < 0) {
                    unsigned char* xs = stages + (size_t)s * a.stage_bytes + SK_ROWS * pitch;
                    mbar_arrive_expect_tx(&xfull[s], (uint32_t)(subs * BN * 128));
                    for (int b = 0; b < subs; ++b)
                        tma_load_2d(xs + b * BN * 128, &tmap_x, kci * a.kc + 64 * b, 0, &xfull[s]);
                } else {
                    mbar_arrive(&xfull[s]);    // B units carry no x: keep the phases in step
                }
                issued_x = sq + 1;
            };
            // Units in processing order; the first NST get their weights before the wait.
            for (int pass = 0; pass < 2 && ok; ++pass) {
                seq = 0;
                for (int i = 0; i < nseg && ok; ++i) {
                    const SkSeg sg = sk_seg(a, u0, u1, i);
                    const int nb = (sg.fin && has_ec) ? a.nbu : 0;
                    for (int v = sg.kb; v < sg.ke + nb && ok; ++v, ++seq) {
                        const int kci = v < sg.ke ? v : 0;
                        const int bu = v < sg.ke ? -1 : v - sg.ke;
                        if (pass == 0) {
                            if (seq >= NST) break;
                            issue_w(seq, sg.tile, kci, bu);
                        } else if (seq < NST) {
                            issue_x(seq, kci, bu);
                        } else {
                            const int s = seq % NST;
                            if (!mbar_wait_ns(&sempty[s], ((seq / NST) - 1) & 1, SK_WAIT_NS)) {
                                sk_fail(a.err, SK_ERR_MBAR, SITE_PROD_SEMPTY, seq);
                                ok = false;
                                break;
                            }
                            issue_w(seq, sg.tile, kci, bu);
                            issue_x(seq, kci, bu);
                        }
                    }
                }
                if (pass == 0) pdl_wait_primary();    // x may be written by the previous kernel
            }
            // Never leave with copies in flight: wait (bounded) for the last load of every stage.
            for (int s = 0; s < NST; ++s) {
                if (s < issued_w) {
                    const int last = s + (issued_w - 1 - s) / NST * NST;
                    if (!mbar_wait_ns(&wfull[s], (last / NST) & 1, SK_WAIT_NS)) sk_fail(a.err, SK_ERR_MBAR, SITE_EXIT, last);
                }
                if (s < issued_x) {
                    const int last = s + (issued_x - 1 - s) / NST * NST;
                    if (!mbar_wait_ns(&xfull[s], (last / NST) & 1, SK_WAIT_NS)) sk_fail(a.err, SK_ERR_MBAR, SITE_EXIT, last);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            bool ok = true;
            int seq = 0, asq = 0, ecount = 0;
            int dcount[2] = {0, 0};
            bool u_seen = false;
            unsigned site = 0;
            // The x loads follow the previous kernel; wait for it here too, so that the waits
            // below span this kernel's work only.
            pdl_wait_primary();
            constexpr uint32_t idesc = idesc_bf16_f32(SK_ROWS, BN);
            constexpr uint32_t idesc_e = idesc_bf16_f32(SK_ROWS, BN) | IDESC_A_MN;
            for (int i = 0; i < nseg && ok; ++i) {
                const SkSeg sg = sk_seg(a, u0, u1, i);
                const int buf = i & 1;
                bool first = true;
                for (int kci = sg.kb; kci < sg.ke && ok; ++kci, ++seq) {
                    const int s = seq % NST;
                    const uint32_t ph = (seq / NST) & 1;
                    if (!mbar_wait_ns(&xfull[s], ph, SK_WAIT_NS)) { site = SITE_MMA_XFULL; ok = false; break; }
                    const unsigned char* xs = stages + (size_t)s * a.stage_bytes + SK_ROWS * pitch;
                    for (int sc = 0; sc < subs; ++sc, ++asq) {
                        const int slot = asq % NA;
                        if (!mbar_wait_ns(&afull[slot], (asq / NA) & 1, SK_WAIT_NS)) { site = SITE_MMA_AFULL; ok = false; break; }
                        tc_fence_after();
                        if (first) {
                            if (dcount[buf] > 0 && !mbar_wait_ns(&dempty[buf], (dcount[buf] - 1) & 1, SK_WAIT_NS)) {
                                site = SITE_MMA_DEMPTY;
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                        }
                        const uint64_t bd = smem_desc_k_sw128(xs + sc * BN * 128);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)   // 16 codes = 8 TMEM columns = 32 bytes of x
                            mma_bf16_ts(tmem_d + buf * BN, tmem_a + slot * 32 + 8 * kk, bd + 2 * kk, idesc,
                                        (first && kk == 0) ? 0u : 1u);
                        first = false;
                        mma_commit(&aempty[slot]);
                    }
                    if (ok) mma_commit(&sempty[s]);
                }
                if (!ok) break;
                mma_commit(&dfull[buf]);
                ++dcount[buf];
                if (sg.fin && has_ec) {
                    // E[n, m] = sum_j B[j, n] (u_hi + u_lo)[m, j], B slices through the ring.
                    if (!u_seen) {
                        if (!mbar_wait_ns(u_ready, 0, SK_WAIT_NS)) { site = SITE_MMA_UREADY; ok = false; break; }
                        u_seen = true;
                    }
                    if (ecount > 0 && !mbar_wait_ns(eempty, (ecount - 1) & 1, SK_WAIT_NS)) { site = SITE_MMA_EEMPTY; ok = false; break; }
                    tc_fence_after();
                    bool efirst = true;
                    for (int bu = 0; bu < a.nbu && ok; ++bu, ++seq) {
                        const int s = seq % NST;
                        const uint32_t ph = (seq / NST) & 1;
                        if (!mbar_wait_ns(&wfull[s], ph, SK_WAIT_NS) || !mbar_wait_ns(&xfull[s], ph, SK_WAIT_NS)) { site = SITE_MMA_BUNIT; ok = false; break; }
                        tc_fence_after();
                        const unsigned char* bs = stages + (size_t)s * a.stage_bytes;
                        const uint64_t ad = smem_desc_mn_sw128(bs, (uint32_t)(a.jb * 128));
                        const int j0 = bu * a.jb;
                        const int nj = min(a.jb, a.rank - j0);
                        for (int part = 0; part < 2; ++part) {
                            for (int kk = 0; kk < nj / 16; ++kk) {
                                const int j = j0 + 16 * kk;
                                const unsigned char* ub = ubuf + ((size_t)part * ublk + j / 64) * BN * 128;
                                const uint64_t ud = smem_desc_k_sw128(ub) + (uint64_t)((j % 64) / 8);
                                mma_bf16_ss(tmem_e, ad + 128 * kk, ud, idesc_e, efirst ? 0u : 1u);
                                efirst = false;
                            }
                        }
                        mma_commit(&sempty[s]);
                    }
                    if (!ok) break;
                    mma_commit(efull);
                    ++ecount;
                }
            }
            if (!ok) sk_fail(a.err, SK_ERR_MBAR, site, seq);
            // Every MMA issued so far has retired before TMEM is released.
            mma_commit(mma_done);
            if (!mbar_wait_ns(mma_done, 0, SK_WAIT_NS)) sk_fail(a.err, SK_ERR_MBAR, SITE_EXIT, seq);
        }
    } else if (warp < 10) {
        // ---------------- converters, then each segment's epilogue ----------------
        const int q = warp & 3;                        // TMEM lane quadrant of this warp
        const int grp = (warp - 2) >> 2;               // sub-chunk parity this warp converts
        const int rowt = q * 32 + lane;                // weight row within the tile = TMEM lane
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        constexpr int HC = BN / 2;                     // accumulator columns (tokens) per thread
        const int m0 = grp * HC;
        bool ok = true;
        int seq = 0, asq = 0, ecount = 0;
        int dcount[2] = {0, 0};
        // Conversion touches only this grid's inputs; the first global write (an epilogue) waits
        // for the previous kernel, which may still read y or this workspace.
        bool waited = false;
        for (int i = 0; i < nseg; ++i) {
            const SkSeg sg = sk_seg(a, u0, u1, i);
            const int64_t n = (int64_t)sg.tile * SK_ROWS + rowt;
            const uint32_t zb = zero_bias_bf16x2((uint32_t)__half2float(a.zero[n]));
            const float sc = __half2float(a.scale[n]);
            for (int kci = sg.kb; kci < sg.ke; ++kci, ++seq) {
                const int s = seq % NST;
                if (ok && !mbar_wait_ns(&wfull[s], (seq / NST) & 1, SK_WAIT_NS)) {
                    sk_fail(a.err, SK_ERR_MBAR, SITE_CVT_WFULL, seq);
                    ok = false;
                }
                ok = __all_sync(0xFFFFFFFFu, ok);      // the TMEM stores below need the whole warp
                const unsigned char* st = stages + (size_t)s * a.stage_bytes;
                for (int sub = 0; sub < subs; ++sub, ++asq) {
                    if ((asq & 1) != grp) continue;
                    const int slot = asq % NA;
                    const int use = asq / NA;
                    if (use > 0 && !waited) {
                        // Slots are freed by MMAs that need x, which follows the previous kernel.
                        pdl_wait_primary();
                        waited = true;
                    }
                    if (ok && use > 0 && !mbar_wait_ns(&aempty[slot], (use - 1) & 1, SK_WAIT_NS)) {
                        sk_fail(a.err, SK_ERR_MBAR, SITE_CVT_AEMPTY, asq);
                        ok = false;
                    }
                    ok = __all_sync(0xFFFFFFFFu, ok);
                    if (ok) {
                        uint32_t o[32];
                        convert_row64(st, (uint32_t)rowt, (uint32_t)sub, (uint32_t)pitch, zb, o);
                        tmem_st32(tmem_a + lane_base + slot * 32, o);
                        tmem_wait_st();
                    }
                    tc_fence_before();
                    mbar_arrive(&afull[slot]);
                }
            }
            // The B units that follow a finalised segment are not waited for here: the epilogue's wait
            // for the E accumulator implies them, and a wait here could fall two phases behind a stage
            // that the MMA has already handed back to the producer.
            if (sg.fin && has_ec) seq += a.nbu;

            // ---- epilogue of segment i, in chunks of 8 tokens per thread ----
            if (!waited) {
                pdl_wait_primary();
                waited = true;
            }
            const int buf = i & 1;
            if (ok && !mbar_wait_ns(&dfull[buf], dcount[buf] & 1, SK_WAIT_NS)) {
                sk_fail(a.err, SK_ERR_MBAR, SITE_EPI_DFULL, i);
                ok = false;
            }
            ++dcount[buf];
            const bool fin_ec = sg.fin && has_ec;
            if (fin_ec) {
                if (ok && !mbar_wait_ns(efull, ecount & 1, SK_WAIT_NS)) {
                    sk_fail(a.err, SK_ERR_MBAR, SITE_EPI_EFULL, i);
                    ok = false;
                }
                ++ecount;
            }
            tc_fence_after();
            // Lower CTAs computed the first chunks of a tile that started before this range: wait
            // for their partial sums (written as their first work, so normally long ready).
            const int c_lo = (sg.fin && sg.kb > 0) ? sk_cta_of(a, sg.tile * a.nch) : c;
            if (c_lo < c) {
                if (threadIdx.x == 64) {
                    for (int cc = c_lo; cc < c; ++cc) {
                        unsigned v;
                        if (!poll_until<unsigned>(ld_acquire_gpu, a.flags + cc, [](unsigned w) { return w != 0u; }, v))
                            sk_fail(a.err, SK_ERR_FLAG, SITE_EPI_FLAG, cc);
                    }
                }
                named_bar_conv();
            }
            float* own = a.partial + (size_t)c * BN * SK_ROWS;
#pragma unroll 1
            for (int cb = 0; cb < HC; cb += 8) {
                float v[8];
                tmem_ld8(tmem_d + buf * BN + m0 + cb + lane_base, v);
                if (!sg.fin) {
                    // Partial sum of a tile that a higher CTA finalises: [BN][128] fp32.
#pragma unroll
                    for (int j = 0; j < 8; ++j) __stcg(own + (m0 + cb + j) * SK_ROWS + rowt, v[j]);
                    continue;
                }
                if (c_lo < c) {
                    // The lower CTAs' partial sums in CTA order, then this CTA's own.
                    float t8[8];
                    for (int cc = c_lo; cc < c; ++cc) {
                        const float* pp = a.partial + (size_t)cc * BN * SK_ROWS + (m0 + cb) * SK_ROWS + rowt;
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const float w = __ldcg(pp + j * SK_ROWS);
                            t8[j] = cc == c_lo ? w : t8[j] + w;
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 8; ++j) v[j] = t8[j] + v[j];
                }
                float e8[8];
                if (fin_ec) tmem_ld8(tmem_e + m0 + cb + lane_base, e8);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int64_t m = m0 + cb + j;
                    if (m >= a.M) break;
                    const float yv = fin_ec ? fmaf(sc, v[j], e8[j]) : sc * v[j];
                    if (a.y_fp32)
                        reinterpret_cast<float*>(a.y)[m * a.N + n] = yv;
                    else
                        reinterpret_cast<__nv_bfloat16*>(a.y)[m * a.N + n] = __float2bfloat16_rn(yv);
                }
            }
            tc_fence_before();
            mbar_arrive(&dempty[buf]);
            if (fin_ec) mbar_arrive(eempty);
            if (!sg.fin) {
                __threadfence();
                named_bar_conv();
                if (threadIdx.x == 64) st_release_gpu(a.flags + c, 1u);
            } else if (c_lo < c) {
                named_bar_conv();                 // every thread has read the partial sums
                if (threadIdx.x == 64)
                    for (int cc = c_lo; cc < c; ++cc) a.flags[cc] = 0u;   // re-armed for the next call
            }
        }
    } else {
        // ---------------- compensator (warp 10) ----------------
        if (has_slice && lane == 0) {
            const uint32_t abytes = (uint32_t)(ec_rows * a.rank * 2), gbytes = (uint32_t)(ec_rows * 2);
            mbar_arrive_expect_tx(ec_bar, abytes + gbytes);
            bulk_load(As, a.A + ec_k0 * a.rank, abytes, ec_bar);
            bulk_load(wgs, a.wg + ec_k0, gbytes, ec_bar);
        }
        pdl_wait_primary();
        unsigned long long* tacc = reinterpret_cast<unsigned long long*>(a.tacc);
        if (has_slice) {
            if (mbar_wait_ns(ec_bar, 0, SK_WAIT_NS))
                ec_slice(a, As, wgs, ec_k0, ec_rows, tacc);
            else if (lane == 0)
                sk_fail(a.err, SK_ERR_MBAR, SITE_EC_BAR, 0);
        }
        if (has_ec && finalizes) {
            // u = sigmoid(p + b_g) t as bf16 hi + lo in the K-major, 128-byte-swizzled layout of the
            // E MMA's B operand (rows = tokens; rows past M are zero).
            float* gs = reinterpret_cast<float*>(smem + a.off_g);
            ec_compute_u(a, tacc, gs, BN, ublk * 64, [&](int m, int j, float uv) {
                const __nv_bfloat16 hi = __float2bfloat16_rn(uv);
                const __nv_bfloat16 lo = __float2bfloat16_rn(uv - __bfloat162float(hi));
                // Block j / 64, row m, byte 2 (j % 64) of a 128-byte row, 128-byte swizzle.
                const uint32_t off = (uint32_t)((j / 64) * BN * 128) + swz_off((uint32_t)m, (uint32_t)((j % 64) / 8), 128u) +
                                     (uint32_t)((j % 8) * 2);
                *reinterpret_cast<__nv_bfloat16*>(ubuf + off) = hi;
                *reinterpret_cast<__nv_bfloat16*>(ubuf + (size_t)ublk * BN * 128 + off) = lo;
            });
            fence_proxy_async_smem();      // generic stores -> visible to the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(u_ready);
            ec_retire(a, tacc);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(a.tmem_cols) : "memory");
    }
}

// ---------------------------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------------------------
static int align_up(int v, int a) { return (v + a - 1) / a * a; }

int stream_grid(int64_t N, int64_t K, int kc, int sms, bool deep) {
    // Two CTAs per SM with the shallow ring (each takes at most half of the SM's shared memory and
    // TMEM), one with the deep ring.
    const int64_t units = (N / SK_ROWS) * (K / kc);
    const int64_t cap = (int64_t)sms * (deep ? 1 : 2);
    return (int)(units < cap ? units : cap);
}

// Shared memory, TMEM and EC slicing for one launch; false if the configuration does not fit.
bool stream_configure(StreamArgs& a, int bn, int kc, bool deep) {
    // At least two 64-code sub-chunks per stage, so that both converter groups convert part of every
    // stage: a group that skipped a stage could otherwise fall two barrier phases behind it.
    if (!(bn == 16 || bn == 32 || bn == 64) || !(kc == 128 || kc == 256)) return false;
    if (a.K % kc != 0 || a.N % SK_ROWS != 0 || a.M < 1 || a.M > bn) return false;
    a.kc = kc;
    a.nch = (int)(a.K / kc);
    a.ntiles = (int)(a.N / SK_ROWS);
    a.units = a.ntiles * a.nch;
    if (a.grid < 1 || a.grid > a.units || a.grid > (int)STREAM_GRID_MAX) return false;
    const int w_bytes = SK_ROWS * kc / 2;
    const int x_bytes = bn * kc * 2;
    a.stage_bytes = align_up(w_bytes + x_bytes, 1024);
    // B units: jb rows of B[:, tile] (two 64-column boxes of jb x 128 bytes) per stage.
    a.jb = 0;
    a.nbu = 0;
    if (a.rank > 0) {
        int jb = (a.stage_bytes / 256) / 16 * 16;
        const int r16 = align_up(a.rank, 16);
        if (jb > r16) jb = r16;
        if (jb < 16 || jb > 256) return false;
        a.jb = jb;
        a.nbu = (a.rank + jb - 1) / jb;
    }
    // Compensator slices: one per CTA at most (the slice count fits the accumulators' 8-bit count).
    a.ec_kr = 0;
    a.ec_slices = 0;
    int a_bytes = 0, wg_bytes = 0, u_bytes = 0, g_bytes = 0;
    if (a.rank > 0) {
        a.ec_kr = sk_ec_rows(a.K, a.rank, a.grid);
        if (a.ec_kr == 0) return false;
        a.ec_slices = (int)((a.K + a.ec_kr - 1) / a.ec_kr);
        if (a.ec_slices > a.grid || a.ec_slices > 255) return false;
        a_bytes = align_up(a.ec_kr * a.rank * 2, 1024);
        wg_bytes = align_up(a.ec_kr * 2, 128);
        u_bytes = 2 * ((a.rank + 63) / 64) * bn * 128;
        g_bytes = align_up(bn * 4, 128);
    }
    const int bar_bytes = 8 * (3 * 16 + 2 * 8 + 10) + 16;
    const int fixed = u_bytes + a_bytes + wg_bytes + g_bytes + bar_bytes + 1024;   // + alignment slack
    const int budget = deep ? (int)SMEM_OPTIN_MAX : 110 * 1024;
    int nst = (budget - fixed) / a.stage_bytes;
    if (nst > 16) nst = 16;
    if (nst < 2) return false;
    a.nst = nst;
    a.off_u = nst * a.stage_bytes;
    a.off_a = a.off_u + u_bytes;
    a.off_wg = a.off_a + a_bytes;
    a.off_g = a.off_wg + wg_bytes;
    a.off_bar = a.off_g + g_bytes;
    a.smem_bytes = a.off_bar + bar_bytes + 1024;
    // The deep ring takes all of an SM's TMEM (512 columns), so no second CTA may share the SM:
    // reserve more than half of its shared memory.
    if (deep && a.smem_bytes < 116 * 1024) a.smem_bytes = 116 * 1024;
    // TMEM: NA converted sub-chunks (32 columns each), two main accumulators and the EC one.
    const int tmem_max = deep ? 512 : 256;
    int na = deep ? 8 : 4;
    while (na > 2 && 32 * na + 3 * bn > tmem_max) na -= 2;
    if (32 * na + 3 * bn > tmem_max) return false;
    a.na = na;
    const int need = 32 * na + 3 * bn;
    a.tmem_cols = need <= 32 ? 32 : need <= 64 ? 64 : need <= 128 ? 128 : need <= 256 ? 256 : 512;
    // CTAs that read the compensator's accumulators (those that finalise a tile).
    a.finalizers = 0;
    for (int cc = 0; cc < a.grid; ++cc) {
        const int v0 = (int)((int64_t)a.units * cc / a.grid), v1 = (int)((int64_t)a.units * (cc + 1) / a.grid);
        if (v0 < v1 && (v1 % a.nch == 0 || (v1 - 1) / a.nch > v0 / a.nch)) ++a.finalizers;
    }
    return true;
}

template <int BN>
static cudaError_t launch_stream_t(const StreamArgs& a, cudaStream_t stream) {
    CUtensorMap mw, mx, mb;
    const uint32_t pitch = (uint32_t)(a.kc / 2);
    const CUtensorMapSwizzle wswz = pitch == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                    : pitch == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
    if (!make_map_2d(&mw, a.packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)(a.K / 2), (uint64_t)a.N, pitch,
                     SK_ROWS, wswz))
        return cudaErrorInvalidValue;
    if (!make_map_2d(&mx, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.K, (uint64_t)a.M, 64, BN,
                     CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (a.rank > 0) {
        if (!make_map_2d(&mb, a.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.N, (uint64_t)a.rank, 64,
                         (uint32_t)a.jb, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    } else {
        mb = mx;   // unused
    }
    static std::once_flag once[kMaxDevices];
    static cudaError_t opt_status[kMaxDevices];
    cudaError_t oe = opt_in_smem((const void*)w4_stream_kernel<BN>, SMEM_OPTIN_MAX, once, opt_status);
    if (oe != cudaSuccess) return oe;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.grid);
    cfg.blockDim = dim3(SK_THREADS);
    cfg.dynamicSmemBytes = (size_t)a.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, w4_stream_kernel<BN>, mw, mx, mb, a);
}

cudaError_t launch_stream(const StreamArgs& a, int bn, cudaStream_t stream) {
    if (bn == 16) return launch_stream_t<16>(a, stream);
    if (bn == 32) return launch_stream_t<32>(a, stream);
    if (bn == 64) return launch_stream_t<64>(a, stream);
    return cudaErrorInvalidValue;
}

}  // namespace spear
