// stream_common.cuh -- pieces shared by the two stream-K kernels of stream.cu (tcgen05 MMA with the
// converted weights in TMEM) and stream_rk.cu (mma.sync with the converted weights in registers):
// wait bounds and error sites, the stream-K schedule, the compensator's slice and its u.
#pragma once

#include "kernels.h"
#include "tcgen05.cuh"

namespace spear {

constexpr int SK_ROWS = 128;                  // weight rows per tile = TMEM lanes
// Every wait of this kernel is bounded in time.  Each role first waits for the previous kernel
// in the stream (programmatic dependent launch) before any wait that could otherwise span it, so
// a wait here only spans this kernel's own work: microseconds normally, a second means a bug.
constexpr uint64_t SK_WAIT_NS = 1000000000ull;
constexpr float SK_FIX_ONE = 4294967296.0f;   // 2^32: fixed-point resolution of the EC accumulators
constexpr int SK_FIX_COUNT_BITS = 8;          // low bits of each word: K slices added so far
constexpr float SK_FIX_TOTAL = 8388608.0f;    // 2^23: bound on |t| and |p|

// Error-word bits of this kernel.
constexpr unsigned SK_ERR_RANGE = 2u;         // an EC partial sum was outside the fixed-point range
constexpr unsigned SK_ERR_MBAR = 16u;         // an mbarrier wait gave up
constexpr unsigned SK_ERR_FLAG = 32u;         // a wait for another CTA (partial sum or EC words) gave up


// Where a wait gave up: the first one is recorded in error word 1 as (site << 24) | (sequence
// number & 0xFFFFFF), beside the error bit in word 0; word 2 collects the sites as a bitmap and
// word 3 holds 1 + the index of the first CTA that gave up.
enum SkSite : unsigned {
    SITE_PROD_SEMPTY = 1, SITE_MMA_XFULL, SITE_MMA_AFULL, SITE_MMA_DEMPTY, SITE_MMA_UREADY, SITE_MMA_EEMPTY,
    SITE_MMA_BUNIT, SITE_CVT_WFULL, SITE_CVT_AEMPTY, SITE_EPI_DFULL, SITE_EPI_EFULL, SITE_EPI_FLAG,
    SITE_EC_BAR, SITE_EC_TACC, SITE_EXIT
};
SPEAR_DEVI void sk_fail(unsigned* err, unsigned bit, unsigned site, int seq) {
    atomicOr(err, bit);
    atomicCAS(err + 1, 0u, (site << 24) | ((unsigned)seq & 0xFFFFFFu));
    atomicOr(err + 2, 1u << site);                  // every site that gave up
    atomicCAS(err + 3, 0u, blockIdx.x + 1);         // the first CTA that did
}
// Poll a global word until pred(word) holds, for at most SK_WAIT_NS; false on timeout.
template <typename T, typename Pred>
SPEAR_DEVI bool poll_until(T (*load)(const T*), const T* p, Pred pred, T& v) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
        v = load(p);
        if (pred(v)) return true;
        if (it > 32) __nanosleep(64);
        if ((it & 15) == 0 && globaltimer_ns() - t0 > SK_WAIT_NS) return false;
    }
}

SPEAR_DEVI void red_add_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("red.relaxed.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
SPEAR_DEVI unsigned long long ld_relaxed_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
SPEAR_DEVI uint32_t lds_u32(const void* p) { return *reinterpret_cast<const uint32_t*>(p); }

// Byte offset of logical (row, 16-byte chunk) in a TMA tile of `pitch`-byte rows stored with the
// swizzle that matches the pitch (32, 64 or 128 bytes): chunk bits ^= row-group bits.
SPEAR_DEVI uint32_t swz_off(uint32_t row, uint32_t chunk, uint32_t pitch) {
    const uint32_t a = row * pitch + chunk * 16;
    const uint32_t mask = pitch == 128 ? 7u : (pitch == 64 ? 3u : 1u);
    return a ^ (((a >> 7) & mask) << 4);
}

// Units of CTA c: [u0, u1).
SPEAR_DEVI int sk_u0(const StreamArgs& a, int c) { return (int)((int64_t)a.units * c / a.grid); }
// The CTA whose range holds unit u.
SPEAR_DEVI int sk_cta_of(const StreamArgs& a, int u) {
    int c = (int)(((int64_t)u * a.grid) / a.units);
    while (c + 1 < a.grid && sk_u0(a, c + 1) <= u) ++c;
    while (c > 0 && sk_u0(a, c) > u) --c;
    return c;
}

struct SkSeg {
    int tile, kb, ke;      // tile and its chunks [kb, ke)
    bool fin;              // ends at the tile's last chunk: this CTA finalises the tile
};
// Segment i in processing order (0 = the range's last segment).
SPEAR_DEVI SkSeg sk_seg(const StreamArgs& a, int u0, int u1, int i) {
    const int t_first = u0 / a.nch, t_last = (u1 - 1) / a.nch;
    SkSeg s;
    s.tile = t_last - i;
    s.kb = s.tile == t_first ? u0 - s.tile * a.nch : 0;
    s.ke = s.tile == t_last ? u1 - s.tile * a.nch : a.nch;
    s.fin = s.ke == a.nch;
    return s;
}

// ---------------------------------------------------------------------------------------------
// The compensator's accumulators: int64 words [M][r + 1] (t, then the gate pre-activation), each
// word in a 32-byte sector of its own, so that the slices' additions to different words do not
// queue behind one another in one sector.  64 tokens x 257 words x 32 bytes fit the workspace's
// accumulator area.
// ---------------------------------------------------------------------------------------------
constexpr int SK_TACC_PAD = 4;
static_assert(64 * 257 * SK_TACC_PAD * 8 <= TACC_BYTES, "accumulator area");
constexpr int SK_EC_KR_MAX = 128;             // rows of A per compensator slice, at most
SPEAR_DEVI unsigned long long* tacc_word(unsigned long long* tacc, const StreamArgs& a, int64_t m, int j) {
    return tacc + ((int64_t)m * (a.rank + 1) + j) * SK_TACC_PAD;
}
SPEAR_DEVI const unsigned long long* tacc_word(const unsigned long long* tacc, const StreamArgs& a, int64_t m, int j) {
    return tacc + ((int64_t)m * (a.rank + 1) + j) * SK_TACC_PAD;
}
// Rows of A per slice: about K / 64 (rounded up to 32), at most SK_EC_KR_MAX and 16 KiB of A, and
// few enough slices for the 8-bit count and the grid.  0 if no such size exists.
inline int sk_ec_rows(int64_t K, int rank, int grid) {
    auto up32 = [](int64_t v) { return (v + 31) / 32 * 32; };
    int64_t kr = up32((K + 63) / 64);
    int64_t kr_max = (16384 / (2 * rank)) / 32 * 32;
    if (kr_max > SK_EC_KR_MAX) kr_max = SK_EC_KR_MAX;
    if (kr_max < 32) kr_max = 32;
    if (kr > kr_max) kr = kr_max;
    if (kr < 32) kr = 32;
    const int64_t slices_max = grid < 255 ? grid : 255;
    const int64_t need = up32((K + slices_max - 1) / slices_max);
    if (kr < need) kr = need;
    return kr <= SK_EC_KR_MAX ? (int)kr : 0;
}

// ---------------------------------------------------------------------------------------------
// The compensator's slice (one warp): t and p over rows [k0, k0 + rows) of A, for every token.
// Tokens are the M = 16 operand of mma.sync m16n8k16, columns of A the N = 8 operand; the 16
// columns of a group form two n8 tiles (even and odd columns) so that one 32-bit shared-memory
// word (two adjacent columns of a row) feeds both.  The gate is one more n8 tile with w_g in
// column 0.  The x fragments of a 16-token block are loaded once, all at the same time.
// ---------------------------------------------------------------------------------------------
SPEAR_DEVI void ec_slice(const StreamArgs& a, const uint16_t* As, const uint16_t* wgs, int64_t k0, int rows,
                         unsigned long long* tacc) {
    constexpr int KS = SK_EC_KR_MAX / 16;
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int r = a.rank, NG = r / 16;
    const float lim = SK_FIX_TOTAL / (float)a.ec_slices;
    const int ksteps = rows / 16;
    for (int m0 = 0; m0 < a.M; m0 += 16) {
        const int64_t ma = m0 + g, mb = m0 + g + 8;
        uint32_t xa[KS][4];
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            const int64_t k = k0 + 16 * kk + 2 * t;
            const bool in = kk < ksteps;
            xa[kk][0] = in && ma < a.M ? __ldcg(reinterpret_cast<const unsigned*>(a.x + ma * a.K + k)) : 0u;
            xa[kk][1] = in && mb < a.M ? __ldcg(reinterpret_cast<const unsigned*>(a.x + mb * a.K + k)) : 0u;
            xa[kk][2] = in && ma < a.M ? __ldcg(reinterpret_cast<const unsigned*>(a.x + ma * a.K + k + 8)) : 0u;
            xa[kk][3] = in && mb < a.M ? __ldcg(reinterpret_cast<const unsigned*>(a.x + mb * a.K + k + 8)) : 0u;
        }
        for (int P = 0; P <= NG; ++P) {
            const bool gate = P == NG;
            float de[4] = {0.f, 0.f, 0.f, 0.f}, dod[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                if (kk >= ksteps) break;
                const int kr = 16 * kk + 2 * t;    // row of the slice
                if (!gate) {
                    const uint16_t* p = As + (int64_t)kr * r + 16 * P + 2 * g;
                    const uint32_t w0 = lds_u32(p), w1 = lds_u32(p + r), w2 = lds_u32(p + 8 * r), w3 = lds_u32(p + 9 * r);
                    mma_bf16_16816(de, xa[kk], prmt(w0, w1, 0x5410u), prmt(w2, w3, 0x5410u));
                    mma_bf16_16816(dod, xa[kk], prmt(w0, w1, 0x7632u), prmt(w2, w3, 0x7632u));
                } else {
                    const uint32_t b0 = g == 0 ? lds_u32(wgs + kr) : 0u;
                    const uint32_t b1 = g == 0 ? lds_u32(wgs + kr + 8) : 0u;
                    mma_bf16_16816(de, xa[kk], b0, b1);
                }
            }
            // Lane (g, t) holds columns 16P + 4t + {0, 1, 2, 3} (even tile: +0, +2; odd: +1, +3)
            // of tokens ma (entries 0, 1) and mb (entries 2, 3); the gate tile's column 0 is in t == 0.
            auto add = [&](int64_t m, int col, float v) {
                if (m >= a.M) return;
                if (!(fabsf(v) < lim)) {
                    atomicOr(a.err, SK_ERR_RANGE);
                    v = 0.0f;
                }
                const unsigned long long fx = (unsigned long long)__float2ll_rn(v * SK_FIX_ONE);
                red_add_u64(tacc_word(tacc, a, m, col), (fx << SK_FIX_COUNT_BITS) | 1ull);
            };
            if (!gate) {
                const int c = 16 * P + 4 * t;
                add(ma, c, de[0]); add(ma, c + 1, dod[0]); add(ma, c + 2, de[1]); add(ma, c + 3, dod[1]);
                add(mb, c, de[2]); add(mb, c + 1, dod[2]); add(mb, c + 2, de[3]); add(mb, c + 3, dod[3]);
            } else if (t == 0) {
                add(ma, r, de[0]);
                add(mb, r, de[2]);
            }
        }
    }
}


// The compensator warp of a CTA that finalises tiles: read every accumulator word once all slices
// are in (bounded wait), form u[m][j] = sigmoid(p[m] + b_g) t[m][j] for m < rows and j < width
// (zero past M and past the rank) and hand each value to store(m, j, u).  gs: `rows` floats of
// shared memory for the gate.
template <typename Store>
SPEAR_DEVI void ec_compute_u(const StreamArgs& a, const unsigned long long* tacc, float* gs, int rows, int width,
                             Store store) {
    const int lane = threadIdx.x & 31;
    const int r = a.rank;
    const unsigned long long want = (unsigned long long)a.ec_slices;
    auto complete = [want](unsigned long long x) { return (x & 0xFFull) == want; };
    for (int m = lane; m < rows; m += 32) {
        float gv = 0.0f;
        if (m < a.M) {
            unsigned long long v;
            if (!poll_until<unsigned long long>(ld_relaxed_u64, tacc_word(tacc, a, m, r), complete, v))
                sk_fail(a.err, SK_ERR_FLAG, SITE_EC_TACC, m * (r + 1) + r);
            const float p = __ll2float_rn((long long)v >> SK_FIX_COUNT_BITS) * (1.0f / SK_FIX_ONE);
            gv = 1.0f / (1.0f + expf(-(p + a.b_g)));
        }
        gs[m] = gv;
    }
    __syncwarp();
    for (int e = lane; e < rows * width; e += 32) {
        const int m = e / width, j = e % width;
        float uv = 0.0f;
        if (m < a.M && j < r) {
            unsigned long long v;
            if (!poll_until<unsigned long long>(ld_relaxed_u64, tacc_word(tacc, a, m, j), complete, v))
                sk_fail(a.err, SK_ERR_FLAG, SITE_EC_TACC, m * (r + 1) + j);
            uv = __ll2float_rn((long long)v >> SK_FIX_COUNT_BITS) * (1.0f / SK_FIX_ONE) * gs[m];
        }
        store(m, j, uv);
    }
}

// After a compensator warp has read the accumulators: the last of the a.finalizers readers clears
// them (and the reader count) for the next call.  Whole warp.
SPEAR_DEVI void ec_retire(const StreamArgs& a, unsigned long long* tacc) {
    const int lane = threadIdx.x & 31;
    unsigned last = 0u;
    if (lane == 0) {
        __threadfence();
        last = atomicAdd(a.ec_readers, 1u) == (unsigned)a.finalizers - 1 ? 1u : 0u;
    }
    last = __shfl_sync(0xFFFFFFFFu, last, 0);
    if (last) {
        __threadfence();
        for (int64_t w = lane; w < a.M * (int64_t)(a.rank + 1); w += 32) tacc[w * SK_TACC_PAD] = 0ull;
        __threadfence();
        __syncwarp();
        if (lane == 0) *a.ec_readers = 0u;
    }
}

}  // namespace spear
