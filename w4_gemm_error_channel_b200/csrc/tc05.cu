// tc05.cu -- the prefill kernel: TMA + tcgen05 (TMEM accumulators) W4 GEMM for sm_100a.
//
// SPEAR (Post-Quantization Error-Adaptive Recovery), technical summary section 2.2A: prefill is
// compute-bound, so the low-bit GEMM must run on the tensor cores.  There is no tcgen05 kind that
// multiplies int4 by bf16 without changing x, so the int4 codes are turned into the exact bf16
// integers (q - z) in shared memory and the MMA is kind::f16 (bf16 x bf16 -> fp32 in TMEM).  The
// per-channel scale s[n] factors out of the K sum and is applied in the epilogue:
//
//   D[n, m] = sum_k (q[n,k] - z[n]) x[m,k]        (tcgen05.mma, fp32 accumulator in TMEM)
//   y[m, n] = s[n] D[n, m] (+ the EC term)         (epilogue: tcgen05.ld -> registers -> y)
//
// One CTA computes a 128 (weight rows) x BN (tokens) tile with 6 warps:
//   warp 0      TMA producer: per 64-wide K stage, the bf16 x tile (128-byte swizzle) and the
//               packed int4 tile (128 rows x 32 bytes) into a STAGES-deep shared-memory ring;
//   warp 1      allocates TMEM and issues tcgen05.mma (one thread), A operand from TMEM, B (x)
//               from shared memory, committing each stage back to the producer;
//   warps 2-5   convert each packed tile to bf16 (q - z) and store it to TMEM with tcgen05.st
//               (one weight row = one TMEM lane per thread), then run the epilogue.
// Keeping the converted weights out of shared memory leaves its bandwidth to the TMA stream and
// the x operand.
//
// The compensator: the first ceil(M / 128) blocks are EC tiles.  Each computes, for 128 tokens,
// t[j, m] = sum_k A[k, j] x[m, k] with tcgen05 (A read MN-major straight from its [K, r] layout by
// TMA) and the gate pre-activation on its converter warps, then stores u = g t (bf16) and raises
// its ready flag.  A main tile, after its K loop, waits (bounded) for the flags of its tokens, loads
// the u tile and the B slice (MN-major, from [r, N]) by TMA and accumulates E[n, m] = sum_j
// B[j, n] u[m, j] into TMEM; the epilogue writes y = s[n] D + E.
// K split (small grids with long K): a tile's K range is split over a cluster of 2, 4 or 8 CTAs;
// after their K loops the partial tiles meet in the owners' idle stage buffers through distributed
// shared memory and are summed in rank order.  EC tiles split the same way and sum t and the gate
// pre-activation before forming u.
// Every mbarrier and flag wait is bounded: on timeout the kernel records an error bit and stops.
#include <mutex>

#include "kernels.h"
#include "tcgen05.cuh"

namespace spear {

constexpr int TC_THREADS = 192;
constexpr int TC_BM = 128;               // weight rows per tile (MMA M)
constexpr int TC_BK = 64;                // K codes per stage
constexpr uint32_t WAIT_LIMIT = 1u << 24;

SPEAR_DEVI void named_bar_epi() { asm volatile("bar.sync 1, 128;" ::: "memory"); }   // warps 2-5

// ---------------------------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------------------------
template <int BN, int STAGES, int SUB>
struct TcSmem {
    static constexpr int X_BYTES = BN * TC_BK * 2;        // bf16 x tile (or u chunk), 128-byte swizzle
    static constexpr int A_BYTES = TC_BM * TC_BK * 2;     // bf16 MN-major tile (A or B slice)
    static constexpr int P_SUB = TC_BM * TC_BK / 2;       // packed int4 tile of 128 weight rows
    static constexpr int P_BYTES = SUB * P_SUB;           // SUB of them per stage
    static constexpr int X_OFF = 0;
    static constexpr int A_OFF = X_OFF + STAGES * X_BYTES;
    static constexpr int P_OFF = A_OFF + STAGES * A_BYTES;
    static constexpr int WG_OFF = P_OFF + STAGES * P_BYTES;              // w_g slice per stage (EC tiles)
    static constexpr int G_OFF = WG_OFF + STAGES * TC_BK * 2;            // gate values, 128 floats
    static constexpr int BAR_OFF = G_OFF + 128 * 4;
    static constexpr int TOTAL = BAR_OFF + 3 * STAGES * 8 + 16 + 16 + 1024;   // + alignment slack
    // TMEM columns: D of sub-tile b at [b BN, (b + 1) BN); converted weight stages from SUB BN,
    // 32 columns per (stage, sub-tile); E of sub-tile b at SUB BN + b BN reuses the stage columns
    // once the main K loop has retired.
    static constexpr int NEED = SUB * BN + (SUB * STAGES * 32 > SUB * BN ? SUB * STAGES * 32 : SUB * BN);
    static constexpr uint32_t TMEM_COLS = NEED <= 32 ? 32 : NEED <= 64 ? 64 : NEED <= 128 ? 128 : NEED <= 256 ? 256 : 512;
    // Two CTAs share an SM when both fit (shared memory and TMEM): one tile's prologue and
    // epilogue then overlap the other's MMAs.
    // The EC tile with the MLP gate stages t [128][r + 1 <= 129] and h [128][H + 1 <= 65] in fp32
    // from X_OFF.
    static_assert(WG_OFF - X_OFF >= 128 * 129 * 4 + 128 * 65 * 4, "MLP-gate staging fits in the stages");
    static constexpr int MIN_BLOCKS = (TOTAL <= 112 * 1024 && TMEM_COLS <= 256) ? 2 : 1;
};
constexpr int TC_EB = 128;               // tokens per EC tile

// Tiles: the first blocks are EC tiles (one per 128 tokens; compute u), the rest are main tiles
// (128 SUB weight rows, token block mb of BN tokens), token-block major.  With SUB = 2 the two
// 128-row sub-tiles share every x stage, which halves the x traffic from L2.  With a K split of
// S > 1 every tile is a cluster of S consecutive CTAs, one per K range (EC tiles too, unless the
// MLP gate is on), and the EC CTAs are padded to whole clusters.
template <int BN, int STAGES, int SUB>
__global__ void __launch_bounds__(TC_THREADS, (TcSmem<BN, STAGES, SUB>::MIN_BLOCKS))
w4_tc05_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
               const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
               const __grid_constant__ CUtensorMap tmap_u, const __grid_constant__ CUtensorMap tmap_g,
               const __grid_constant__ CUtensorMap tmap_x128, const __grid_constant__ CUtensorMap tmap_y,
               TcArgs a) {
    using L = TcSmem<BN, STAGES, SUB>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);       // TMA landed
    uint64_t* cvt = full + STAGES;                                         // stage ready for the MMA
    uint64_t* empty = cvt + STAGES;                                        // MMA done with the stage
    uint64_t* acc_full = empty + STAGES;                                   // accumulators complete
    uint64_t* main_done = acc_full + 1;                                    // main K loop retired
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(main_done + 1);
    float* s_gate = reinterpret_cast<float*>(smem + L::G_OFF);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool has_ec = a.rank > 0;
    const int S = a.split;                                                 // K splits per weight tile
    const int eblocks = (int)((a.M + TC_EB - 1) / TC_EB);
    // EC tiles split their K range the same way (one cluster per 128-token block), except with the
    // bottleneck-MLP gate, whose epilogue needs the whole of t in one CTA.
    const int SE = a.mlp.w1 != nullptr ? 1 : S;
    const int ec_ctas = has_ec ? eblocks * SE : 0;
    const int ec_pad = (ec_ctas + S - 1) / S * S;                          // EC CTAs, padded to whole clusters
    if ((int)blockIdx.x >= ec_ctas && (int)blockIdx.x < ec_pad) return;    // idle CTA of the last EC cluster
    const bool is_ec = (int)blockIdx.x < ec_ctas;
    const int KS = is_ec ? SE : S;                                         // K splits of this CTA's tile
    const int bi = is_ec ? (int)blockIdx.x : (int)blockIdx.x - ec_pad;
    const int ks = bi % KS;                                                // this CTA's K split = cluster rank
    const int t = bi / KS;
    const int ntiles = (int)(a.N / (TC_BM * SUB));
    const int mb = is_ec ? t : t / ntiles;                                 // EC: 128-token block; main: BN block
    const int64_t n0 = is_ec ? 0 : (int64_t)(t % ntiles) * TC_BM * SUB;
    const int64_t m0 = (int64_t)mb * (is_ec ? TC_EB : BN);
    const int ksteps = (int)(a.K / TC_BK) / KS;                            // K stages of this CTA
    const int kbase = ks * ksteps;                                         // its first K stage
    // EC MMA steps: 64 columns of u per chunk, one step per (chunk, sub-tile); with a K split the
    // first split of the tile adds the EC term.
    const int ec_chunks = (!is_ec && has_ec && ks == 0) ? ((a.rank + 63) / 64) * SUB : 0;
    const int rboxes = (a.rank + 63) / 64;                                 // 64-wide boxes of A per stage
    const int e_lo = (int)(m0 / TC_EB);                                    // EC blocks this main tile needs
    const int e_hi = min(eblocks, (int)((m0 + BN + TC_EB - 1) / TC_EB));

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&cvt[s], 128);        // every converter thread arrives
            mbar_init(&empty[s], 1);        // tcgen05.commit
        }
        mbar_init(acc_full, 1);
        mbar_init(main_done, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(L::TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = *tmem_slot;
    const uint32_t tmem_a = tmem_d + SUB * BN;   // converted weight stages (main K loop)
    const uint32_t tmem_e = tmem_d + SUB * BN;   // EC accumulators (after the main K loop)
    bool epi_ok = true;                          // converter warps: the accumulators completed
    float pg_part = 0.0f;                        // EC converter warps: gate pre-activation over this K split

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            // Weight-side operands (packed W, or A and w_g) of a stage; x only after the wait.
            auto load_weights = [&](int kt, int s) {
                if (is_ec) {
                    unsigned char* as = smem + L::A_OFF + s * L::A_BYTES;
                    mbar_arrive_expect_tx(&full[s], TC_EB * TC_BK * 2 + rboxes * (TC_BK * 64 * 2) + TC_BK * 2);
                    for (int bx = 0; bx < rboxes; ++bx)
                        tma_load_2d(as + bx * (TC_BK * 64 * 2), &tmap_a, bx * 64, (kbase + kt) * TC_BK, &full[s]);
                    tma_load_2d(smem + L::WG_OFF + s * TC_BK * 2, &tmap_g, (kbase + kt) * TC_BK, 0, &full[s]);
                } else {
                    mbar_arrive_expect_tx(&full[s], L::X_BYTES + L::P_BYTES);
                    for (int sb = 0; sb < SUB; ++sb)
                        tma_load_2d(smem + L::P_OFF + s * L::P_BYTES + sb * L::P_SUB, &tmap_w, (kbase + kt) * (TC_BK / 2),
                                    (int32_t)(n0 + sb * TC_BM), &full[s]);
                }
            };
            const int pre = ksteps < STAGES ? ksteps : STAGES;
            for (int kt = 0; kt < pre; ++kt) load_weights(kt, kt);
            pdl_wait_primary();            // x may be written by the previous kernel in the stream
            bool ok = true;
            for (int kt = 0; kt < ksteps && ok; ++kt) {
                const int s = kt % STAGES;
                if (kt >= STAGES) {
                    if (!mbar_wait(&empty[s], ((kt / STAGES) - 1) & 1)) { atomicOr(a.err, 4u); ok = false; break; }
                    load_weights(kt, s);
                }
                unsigned char* xs = smem + L::X_OFF + s * L::X_BYTES;
                tma_load_2d(xs, is_ec ? &tmap_x128 : &tmap_x, (kbase + kt) * TC_BK, (int32_t)m0, &full[s]);
            }
            if (ok && ec_chunks > 0) {
                // u of these tokens is written by their EC tiles: wait (bounded) until each flag
                // counts all SE EC CTAs of its block.
                for (int e = e_lo; e < e_hi && ok; ++e) {
                    unsigned it = 0;
                    while (ld_acquire_gpu(&a.ec_ready[e]) < (unsigned)SE) {
                        if (++it > WAIT_LIMIT) { atomicOr(a.err, 8u); ok = false; break; }
                        if (it > 64) __nanosleep(128);
                    }
                }
                asm volatile("fence.proxy.async.global;" ::: "memory");
                for (int c = 0; c < ec_chunks && ok; ++c) {
                    const int v = ksteps + c, s = v % STAGES;
                    if (v >= STAGES && !mbar_wait(&empty[s], ((v / STAGES) - 1) & 1)) { atomicOr(a.err, 4u); ok = false; break; }
                    unsigned char* xs = smem + L::X_OFF + s * L::X_BYTES;
                    unsigned char* as = smem + L::A_OFF + s * L::A_BYTES;
                    const int ch = c / SUB, nb0 = (int)n0 + (c % SUB) * TC_BM;
                    mbar_arrive_expect_tx(&full[s], L::X_BYTES + 2 * (64 * 64 * 2));
                    tma_load_2d(xs, &tmap_u, ch * 64, (int32_t)m0, &full[s]);                // u[m, 64ch ..]
                    tma_load_2d(as, &tmap_b, nb0, ch * 64, &full[s]);                        // B[64ch .., nb0 .. +64]
                    tma_load_2d(as + 64 * 64 * 2, &tmap_b, nb0 + 64, ch * 64, &full[s]);
                }
                // Every main tile of these tokens has seen the flags: the last one re-arms each.
                // EC block e is read by every weight tile of each token block that overlaps it.
                if (ok) {
                    for (int e = e_lo; e < e_hi; ++e) {
                        const int64_t t_lo = (int64_t)e * TC_EB;
                        const int64_t t_hi = ((int64_t)(e + 1) * TC_EB < a.M ? (int64_t)(e + 1) * TC_EB : a.M) - 1;
                        const unsigned readers = (unsigned)ntiles * (unsigned)(t_hi / BN - t_lo / BN + 1);
                        if (atomicAdd(&a.ec_consumed[e], 1u) == readers - 1) {
                            a.ec_consumed[e] = 0u;
                            a.ec_ready[e] = 0u;
                        }
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            bool ok = true;
            for (int kt = 0; kt < ksteps; ++kt) {
                const int s = kt % STAGES;
                if (!mbar_wait(&cvt[s], (kt / STAGES) & 1)) { atomicOr(a.err, 4u); ok = false; break; }
                tc_fence_after();
                const uint64_t bd = smem_desc_k_sw128(smem + L::X_OFF + s * L::X_BYTES);
                if (is_ec) {
                    constexpr uint32_t idesc = idesc_bf16_f32(TC_BM, TC_EB) | IDESC_A_MN;
                    const uint64_t ad = smem_desc_mn_sw128(smem + L::A_OFF + s * L::A_BYTES, TC_BK * 64 * 2);
#pragma unroll
                    for (int kk = 0; kk < TC_BK / 16; ++kk)   // 16 K rows = 2 groups of 1024 bytes
                        mma_bf16_ss(tmem_d, ad + 128 * kk, bd + 2 * kk, idesc, (kt > 0 || kk > 0) ? 1u : 0u);
                } else {
                    constexpr uint32_t idesc = idesc_bf16_f32(TC_BM, BN);
#pragma unroll
                    for (int sb = 0; sb < SUB; ++sb)
#pragma unroll
                        for (int kk = 0; kk < TC_BK / 16; ++kk)   // 16 bf16 = 8 TMEM columns = 2 descriptor units
                            mma_bf16_ts(tmem_d + sb * BN, tmem_a + (s * SUB + sb) * 32 + 8 * kk, bd + 2 * kk, idesc,
                                        (kt > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&empty[s]);
            }
            if (ok && ec_chunks > 0) {
                // The EC accumulator reuses the weight-stage columns: let the main loop retire first.
                mma_commit(main_done);
                if (!mbar_wait(main_done, 0)) { atomicOr(a.err, 4u); ok = false; }
                tc_fence_after();
            }
            constexpr uint32_t idesc_ec = idesc_bf16_f32(TC_BM, BN) | IDESC_A_MN;
            for (int c = 0; c < ec_chunks && ok; ++c) {
                // E[n, m] += sum_j B[j, n] u[m, j], 64 columns j per step (B slice MN-major).
                const int v = ksteps + c, s = v % STAGES;
                if (!mbar_wait(&cvt[s], (v / STAGES) & 1)) { atomicOr(a.err, 4u); ok = false; break; }
                tc_fence_after();
                const uint64_t ad = smem_desc_mn_sw128(smem + L::A_OFF + s * L::A_BYTES, 64 * 64 * 2);
                const uint64_t bd = smem_desc_k_sw128(smem + L::X_OFF + s * L::X_BYTES);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ss(tmem_e + (c % SUB) * BN, ad + 128 * kk, bd + 2 * kk, idesc_ec,
                                (c / SUB > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&empty[s]);
            }
            mma_commit(acc_full);
        }
    } else {
        // ---------------- converters / gate, then epilogue ----------------
        // Weight row of this thread: warp w may only access TMEM lanes 32*(w % 4) .. +31, and the
        // accumulator and weight-operand row n live in lane n, so warps 2, 3, 4, 5 take rows
        // 64, 96, 0, 32 (+lane).
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        uint32_t zb[SUB];
#pragma unroll
        for (int sb = 0; sb < SUB; ++sb)
            zb[sb] = is_ec ? 0u : zero_bias_bf16x2((uint32_t)__half2float(a.zero[n0 + sb * TC_BM + row]));
        float pg = 0.0f;                                   // EC tiles: gate pre-activation of token `row`
        bool ok = true;
        for (int kt = 0; kt < ksteps + ec_chunks; ++kt) {
            const int s = kt % STAGES;
            if (!mbar_wait(&full[s], (kt / STAGES) & 1)) { atomicOr(a.err, 4u); ok = false; break; }
            if (is_ec) {
                // Gate pre-activation: x[m, k] w_g[k] over this stage for token m = row.
                const unsigned char* xr = smem + L::X_OFF + s * L::X_BYTES + (row >> 3) * 1024 + (row & 7) * 128;
                const uint4* wgs = reinterpret_cast<const uint4*>(smem + L::WG_OFF + s * TC_BK * 2);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 wr = wgs[c];
                    const uint4 xv = *reinterpret_cast<const uint4*>(xr + ((c ^ (row & 7)) << 4));
                    const uint32_t ww[4] = {wr.x, wr.y, wr.z, wr.w}, xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        pg = fmaf(__uint_as_float(xw[e] << 16), __uint_as_float(ww[e] << 16), pg);
                        pg = fmaf(__uint_as_float(xw[e] & 0xFFFF0000u), __uint_as_float(ww[e] & 0xFFFF0000u), pg);
                    }
                }
            } else if (kt < ksteps) {
                // 64 codes of weight row `row` of each sub-tile -> 32 TMEM columns of bf16 pairs
                // (q - z), natural order.
#pragma unroll
                for (int sb = 0; sb < SUB; ++sb) {
                    const uint4* prow =
                        reinterpret_cast<const uint4*>(smem + L::P_OFF + s * L::P_BYTES + sb * L::P_SUB + row * 32);
                    uint32_t o[32];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint4 w = prow[h];
                        cvt_w4_pairs_natural(w.x, zb[sb], o + 16 * h);
                        cvt_w4_pairs_natural(w.y, zb[sb], o + 16 * h + 4);
                        cvt_w4_pairs_natural(w.z, zb[sb], o + 16 * h + 8);
                        cvt_w4_pairs_natural(w.w, zb[sb], o + 16 * h + 12);
                    }
                    tmem_st32(tmem_a + lane_base + (s * SUB + sb) * 32, o);
                }
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
            }
            mbar_arrive(&cvt[s]);
        }

        const bool acc_ok = ok && mbar_wait(acc_full, 0);
        if (!acc_ok) atomicOr(a.err, 4u);
        epi_ok = acc_ok;
        pg_part = pg;
        tc_fence_after();
        if (is_ec && SE > 1) {
            // K-split EC tile: the partial t and gate pre-activations meet after the block barrier.
        } else if (is_ec) {
            if (a.mlp.w1 != nullptr) {
                // Bottleneck-MLP gate: t is staged as [token][j] in the idle stages, then thread row
                // takes token m0 + row: h = relu(W1 t + b1), u[m, j] = alpha sigmoid(W2 h + b2)_j t_j.
                const int r = a.rank, H = a.mlp.hidden;
                // Odd row strides: each thread walks its own row, so rows must start in different banks.
                const int rs = r + 1, hsd = H + 1;
                float* ts = reinterpret_cast<float*>(smem + L::X_OFF);            // [TC_EB][r + 1]
                float* hs = ts + TC_EB * rs;                                       // [TC_EB][H + 1]
                for (int c0 = 0; c0 < TC_EB; c0 += 16) {
                    float v[16];
                    tmem_ld16(tmem_d + lane_base + (uint32_t)c0, v);
                    if (row < r) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) ts[(c0 + i) * rs + row] = v[i];
                    }
                }
                named_bar_epi();
                const int64_t m = m0 + row;
                if (acc_ok && m < a.M) {
                    const float* tr = ts + row * rs;
                    float* hr = hs + row * hsd;
                    for (int i = 0; i < H; ++i) {
                        const float* w1 = a.mlp.w1 + (int64_t)i * r;
                        float pre = __ldg(a.mlp.b1 + i);
#pragma unroll 8
                        for (int j = 0; j < r; ++j) pre = fmaf(__ldg(w1 + j), tr[j], pre);
                        hr[i] = fmaxf(pre, 0.0f);
                    }
                    for (int j = 0; j < r; ++j) {
                        const float* w2 = a.mlp.w2 + (int64_t)j * H;
                        float pre = __ldg(a.mlp.b2 + j);
#pragma unroll 8
                        for (int i = 0; i < H; ++i) pre = fmaf(__ldg(w2 + i), hr[i], pre);
                        a.u[m * r + j] = __float2bfloat16_rn(a.mlp.alpha * tr[j] / (1.0f + expf(-pre)));
                    }
                }
            } else {
            // g[m] = sigmoid(p[m] + b_g); u[m, j] = g[m] t[j, m] for j = row < r, as bf16.
            s_gate[row] = 1.0f / (1.0f + expf(-(pg + a.b_g)));
            named_bar_epi();
            const int j = row;
            for (int c0 = 0; c0 < TC_EB; c0 += 16) {
                float v[16];
                tmem_ld16(tmem_d + lane_base + (uint32_t)c0, v);
                if (!acc_ok || j >= a.rank) continue;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int64_t m = m0 + c0 + i;
                    if (m < a.M) a.u[m * a.rank + j] = __float2bfloat16_rn(s_gate[c0 + i] * v[i]);
                }
            }
            }
            asm volatile("fence.proxy.async.global;" ::: "memory");   // u is read by other CTAs' TMA
            __threadfence();
            named_bar_epi();
            // EC tiles launched alone (the semi-fused path) have no main tiles to signal.
            if (row == 0 && acc_ok && !a.ec_only)
                asm volatile("st.release.gpu.global.u32 [%0], 1;" ::"l"(&a.ec_ready[mb]) : "memory");
        } else if (S == 1) {
            // y[m, n] = s[n] D[n, m] (+ E[n, m]), sub-tile by sub-tile.  bf16 output: the tile is
            // staged in the (now idle) x stages as y[m][n] rows and leaves in one TMA store,
            // which also drops the rows past M; fp32 debug output is stored directly.
            constexpr int YROWS = TC_BM * SUB;
            __nv_bfloat16* ys = reinterpret_cast<__nv_bfloat16*>(smem + L::X_OFF);   // [BN][YROWS]
            for (int sb = 0; sb < SUB; ++sb) {
            const float sc = __half2float(a.scale[n0 + sb * TC_BM + row]);
            const int64_t n = n0 + sb * TC_BM + row;
            for (int c0 = 0; c0 < BN; c0 += 16) {
                float v[16], e[16];
                tmem_ld16(tmem_d + (uint32_t)(sb * BN) + lane_base + (uint32_t)c0, v);
                if (has_ec) tmem_ld16(tmem_e + (uint32_t)(sb * BN) + lane_base + (uint32_t)c0, e);
                if (!acc_ok) continue;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int64_t m = m0 + c0 + i;
                    const float yv = has_ec ? fmaf(sc, v[i], e[i]) : sc * v[i];
                    if (a.y_fp32) {
                        if (m < a.M) reinterpret_cast<float*>(a.y)[m * a.N + n] = yv;
                    } else {
                        ys[(c0 + i) * YROWS + sb * TC_BM + row] = __float2bfloat16_rn(yv);
                    }
                }
            }
            }
            if (!a.y_fp32 && acc_ok) {
                fence_proxy_async_smem();            // generic-proxy writes -> visible to the TMA
                named_bar_epi();
                if (row == 0) {
                    tma_store_2d(&tmap_y, ys, (int32_t)n0, (int32_t)m0);
                    tma_store_wait_read();
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (KS > 1) {
        // K split: the KS CTAs of this cluster hold partial sums of one tile.  Each has seen its
        // accumulators complete (before the block barrier above), so its stage area is idle; after
        // one cluster barrier it receives the partial tiles of the columns it owns: rank ks owns
        // columns [ks C / KS, (ks + 1) C / KS) of the tile's C token columns and sums the KS
        // partials in rank order (fixed order, so the result does not depend on timing).
        //   main tile: a partial is s[n] D + E (E on rank 0 only), summed into y;
        //   EC tile:   a partial is t[j, m] plus the gate pre-activation of token m, summed into
        //              u = sigmoid(p + b_g) t, after which the rank adds 1 to the block's ready flag.
        const int cols = is_ec ? TC_EB : BN;
        const int bno = cols / KS, rstride = bno + 4;    // padded rows: conflict-free float4 access
        float* recv = reinterpret_cast<float*>(smem + L::X_OFF);   // [KS][128 rows][bno + 4]
        float* recv_p = recv + KS * TC_BM * rstride;               // EC: [KS][128 tokens]
        __syncwarp();
        cluster_sync_all();
        tc_fence_after();
        if (warp >= 2) {
            const int row = (warp & 3) * 32 + lane;
            const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
            const float sc = is_ec ? 1.0f : __half2float(a.scale[n0 + row]);
            const bool with_e = ec_chunks > 0;
            // Rank ks starts with the columns of owner ks + 1, so that at any time each owner
            // receives from one rank rather than all ranks at once.
            for (int q = 0; q < cols; q += 16) {
                const int c0 = (q + (ks + 1) * bno) % cols;
                float v[16], e[16];
                tmem_ld16(tmem_d + lane_base + (uint32_t)c0, v);
                if (with_e) tmem_ld16(tmem_e + lane_base + (uint32_t)c0, e);
                const int owner = c0 / bno;                // bno is a multiple of 16
                float* dst = recv + (ks * TC_BM + row) * rstride + (c0 - owner * bno);
#pragma unroll
                for (int i = 0; i < 16; i += 4) {
                    const float4 w = with_e ? make_float4(fmaf(sc, v[i], e[i]), fmaf(sc, v[i + 1], e[i + 1]),
                                                          fmaf(sc, v[i + 2], e[i + 2]), fmaf(sc, v[i + 3], e[i + 3]))
                                            : make_float4(sc * v[i], sc * v[i + 1], sc * v[i + 2], sc * v[i + 3]);
                    st_dsmem_f4(reinterpret_cast<float4*>(dst + i), (unsigned)owner, w);
                }
            }
            if (is_ec) st_dsmem_f32(recv_p + ks * TC_BM + row, (unsigned)(row / bno), pg_part);
        }
        tc_fence_before();
        __syncwarp();
        cluster_sync_all();
        if (warp >= 2) {
            const int row = (warp & 3) * 32 + lane;
            if (is_ec) {
                // Thread row = EC column j; tokens of this rank's share one by one.
                const int j = row;
                for (int c = 0; c < bno; ++c) {
                    const int ml = ks * bno + c;
                    float p = recv_p[ml];
                    float tv = recv[j * rstride + c];
                    for (int src = 1; src < KS; ++src) {
                        p += recv_p[src * TC_BM + ml];
                        tv += recv[(src * TC_BM + j) * rstride + c];
                    }
                    const int64_t m = m0 + ml;
                    if (epi_ok && j < a.rank && m < a.M)
                        a.u[m * a.rank + j] = __float2bfloat16_rn(tv / (1.0f + expf(-(p + a.b_g))));
                }
                asm volatile("fence.proxy.async.global;" ::: "memory");   // u is read by other CTAs' TMA
                __threadfence();
                named_bar_epi();
                if (row == 0 && epi_ok)
                    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&a.ec_ready[mb]) : "memory");
            } else if (epi_ok) {
                const int64_t n = n0 + row;
                for (int c = 0; c < bno; c += 4) {
                    float4 sum = *reinterpret_cast<const float4*>(recv + row * rstride + c);
                    for (int src = 1; src < KS; ++src) {
                        const float4 o = *reinterpret_cast<const float4*>(recv + (src * TC_BM + row) * rstride + c);
                        sum.x += o.x;
                        sum.y += o.y;
                        sum.z += o.z;
                        sum.w += o.w;
                    }
                    const float sv[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int64_t m = m0 + (int64_t)ks * bno + c + i;
                        if (m >= a.M) continue;
                        if (a.y_fp32)
                            reinterpret_cast<float*>(a.y)[m * a.N + n] = sv[i];
                        else
                            reinterpret_cast<__nv_bfloat16*>(a.y)[m * a.N + n] = __float2bfloat16_rn(sv[i]);
                    }
                }
            }
        }
        tc_fence_after();
    }
    pdl_launch_dependents();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_d), "r"(L::TMEM_COLS) : "memory");
    }
}

// ---------------------------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once per process (thread-safe).
static EncodeTiledFn encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, []() {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

bool make_map_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem, uint64_t cols,
                 uint64_t rows, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * (uint64_t)elem};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, const uint64_t dims[3],
                 const uint64_t strides_bytes[2], const uint32_t box[3], CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
    const cuuint64_t st[2] = {strides_bytes[0], strides_bytes[1]};
    const cuuint32_t b[3] = {box[0], box[1], box[2]};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, dtype, 3, const_cast<void*>(base), d, st, b, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t opt_in_smem_at_least(const void* func, size_t bytes, std::mutex& mu, size_t* opted) {
    if (bytes == 0) return cudaSuccess;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (bytes <= opted[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) opted[dev] = bytes;
    return e;
}

cudaError_t opt_in_smem(const void* func, size_t bytes, std::once_flag* once, cudaError_t* status) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&]() {
        status[dev] = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    });
    return status[dev];
}

// A K split of S: the tile's token columns split into S owners' shares of a multiple of 16, the
// partial tiles fit in the stage area ([S][128][BN / S + 4] fp32; an EC tile's [S][128][128 / S + 4]
// plus [S][128] gate pre-activations), and every split has the same number of 64-wide K stages.
template <int BN, int STAGES, int SUB>
static bool split_fits(int split, int64_t K) {
    using L = TcSmem<BN, STAGES, SUB>;
    if (split == 1) return true;
    if (!(split == 2 || split == 4 || split == 8) || SUB != 1) return false;
    if (BN % (16 * split) != 0 || (K / TC_BK) % split != 0) return false;
    const int64_t stage_area = L::WG_OFF - L::X_OFF;
    const int64_t ec_part = (int64_t)split * TC_BM * (TC_EB / split + 4) * 4 + (int64_t)split * TC_BM * 4;
    return (int64_t)split * TC_BM * (BN / split + 4) * 4 <= stage_area && ec_part <= stage_area;
}

template <int BN, int STAGES, int SUB>
static cudaError_t launch_tc_t(const TcArgs& a_in, cudaStream_t stream, bool pdl, int priority, int split) {
    using L = TcSmem<BN, STAGES, SUB>;
    if (!split_fits<BN, STAGES, SUB>(split, a_in.K) || (split > 1 && a_in.ec_only)) return cudaErrorInvalidValue;
    TcArgs a = a_in;
    a.split = split;
    CUtensorMap mx, mw, ma, mb, mu, mg, mx128;
    if (!make_map_2d(&mx, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.K, (uint64_t)a.M, TC_BK, BN,
                     CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!make_map_2d(&mw, a.packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)(a.K / 2), (uint64_t)a.N, TC_BK / 2,
                     TC_BM, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    if (!make_map_2d(&mx128, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.K, (uint64_t)a.M, TC_BK, TC_EB,
                     CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    CUtensorMap my;
    if (!a.y_fp32) {
        // y [M, N] bf16 written as BN (m) x 128 SUB (n) boxes.
        if (!make_map_2d(&my, a.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.N, (uint64_t)a.M, TC_BM * SUB, BN,
                         CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    } else {
        my = mx;                                 // unused: fp32 output is stored directly
    }
    const bool has_ec = a.rank > 0;
    if (has_ec) {
        // A [K, r] read as 64 (j) x 64 (k) boxes; B [r, N] as 64 (n) x 64 (j); u [M, r] as 64 (j) x BN (m).
        if (!make_map_2d(&ma, a.A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.rank, (uint64_t)a.K, 64, TC_BK,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map_2d(&mb, a.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.N, (uint64_t)a.rank, 64, 64,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map_2d(&mu, a.u, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.rank, (uint64_t)a.M, 64, BN,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map_2d(&mg, a.wg, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.K, 1, TC_BK, 1,
                         CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    } else {
        ma = mx; mb = mx; mu = mx; mg = mx;      // unused
    }
    static std::once_flag once[kMaxDevices];
    static cudaError_t opt_status[kMaxDevices];
    cudaError_t oe = opt_in_smem((const void*)w4_tc05_kernel<BN, STAGES, SUB>, L::TOTAL, once, opt_status);
    if (oe != cudaSuccess) return oe;
    const unsigned mblocks = (unsigned)((a.M + BN - 1) / BN);
    const unsigned eblocks = (unsigned)((a.M + TC_EB - 1) / TC_EB);
    // EC CTAs first (split like the main tiles unless the MLP gate is on; padded to whole clusters),
    // then the split CTAs of each main tile side by side.
    const unsigned ec_ctas = has_ec ? eblocks * (a.mlp.w1 != nullptr ? 1u : (unsigned)split) : 0u;
    const unsigned ec_pad = (ec_ctas + split - 1) / split * split;
    const unsigned tiles =
        a.ec_only ? eblocks : (unsigned)(a.N / (TC_BM * SUB)) * mblocks * (unsigned)split + ec_pad;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(tiles);
    cfg.blockDim = dim3(TC_THREADS);
    cfg.dynamicSmemBytes = L::TOTAL;
    cfg.stream = stream;
    cudaLaunchAttribute attr[3];
    unsigned na = 0;
    if (split > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)split;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (priority != 0) {
        attr[na].id = cudaLaunchAttributePriority;
        attr[na].val.priority = priority;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, w4_tc05_kernel<BN, STAGES, SUB>, mx, mw, ma, mb, mu, mg, mx128, my, a);
}

cudaError_t launch_tc05(const TcArgs& a, int bn, int rows, cudaStream_t stream, bool pdl, int priority, int split) {
    if (rows == 256) return bn == 128 ? launch_tc_t<128, 4, 2>(a, stream, pdl, priority, split) : cudaErrorInvalidValue;
    if (rows != 128) return cudaErrorInvalidValue;
    if (bn == 128) return launch_tc_t<128, 3, 1>(a, stream, pdl, priority, split);
    if (bn == 160) return launch_tc_t<160, 4, 1>(a, stream, pdl, priority, split);
    if (bn == 192) return launch_tc_t<192, 3, 1>(a, stream, pdl, priority, split);
    if (bn == 256) return launch_tc_t<256, 4, 1>(a, stream, pdl, priority, split);
    return cudaErrorInvalidValue;
}

bool tc05_split_supported(int bn, int rows, int split, int64_t K) {
    if (rows == 256) return bn == 128 && split_fits<128, 4, 2>(split, K);
    if (rows != 128) return false;
    if (bn == 128) return split_fits<128, 3, 1>(split, K);
    if (bn == 160) return split_fits<160, 4, 1>(split, K);
    if (bn == 192) return split_fits<192, 3, 1>(split, K);
    if (bn == 256) return split_fits<256, 4, 1>(split, K);
    return false;
}

}  // namespace spear
