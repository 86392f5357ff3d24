// slo.cu -- the EC-aware, SLO-constrained prefill chunk picker over kernel-latency lookup tables.
//
// SPEAR technical summary, section 2.2C: because compensators sit only on selected layers, the
// cost of a step depends on where they are, and a fixed prefill chunk size either breaks the
// inter-token-latency (ITL) objective or wastes it.  The scheduler therefore picks, step by step,
// the largest prefill chunk whose predicted step latency meets the ITL target, from precomputed
// tables of kernel latencies.
//
// Here a step runs every linear of the model once on M = decode tokens + chunk tokens (chunked
// prefill: the decode tokens and the chunk share each GEMM).  Its predicted latency is
//
//     fixed_us + sum over linears i of count_i * T(M, N_i, K_i, rank_i > 0)
//
// with T from a latency table of measured calls: per (N, K, compensator or not), the samples
// T(M_j) are made nondecreasing in M (running maximum), then read by linear interpolation between
// measured batch sizes, as T(M_min) below the smallest one (the weight stream sets the time
// there) and as T(M_max) * M / M_max above the largest (compute-bound: time in proportion to
// tokens).  The step latency is then nondecreasing in the chunk size, so the largest chunk that
// meets the target is found by bisection over multiples of the caller's granule.
//
// The default table is the library's own dispatcher table: for each shape measured on a B200, the
// device time of its fastest plan per call in a chained CUDA graph.  It keys a shape by whether it
// has a compensator, not by its rank.
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#include <algorithm>
#include <vector>

#include "../../include/spear.h"

namespace spear {
namespace {

struct TableRow {
    int64_t M, N, K;
    int has_ec, kernel_id, tile_n, split_k, tile_m, flags;
    double us;
};
const TableRow kTable[] = {
#include "plan_table.inc"
};
constexpr int32_t kTableLen = (int32_t)(sizeof(kTable) / sizeof(kTable[0]));
constexpr int64_t SLO_M_MAX = 65536;

struct Sample {
    int64_t M;
    double us;
};

// The samples of one (N, K, has_ec) from the table, sorted by M, made nondecreasing.
bool samples_for(const spear_latency_entry* lut, int32_t len, int64_t N, int64_t K, int has_ec,
                 std::vector<Sample>* out) {
    out->clear();
    for (int32_t i = 0; i < len; ++i)
        if (lut[i].N == N && lut[i].K == K && (lut[i].has_ec != 0) == (has_ec != 0))
            out->push_back({lut[i].M, lut[i].us});
    if (out->empty()) return false;
    std::sort(out->begin(), out->end(), [](const Sample& a, const Sample& b) { return a.M < b.M; });
    // Equal M: keep the larger time, then the running maximum.
    std::vector<Sample> s;
    for (const Sample& x : *out) {
        if (!s.empty() && s.back().M == x.M) s.back().us = std::max(s.back().us, x.us);
        else s.push_back(x);
    }
    for (size_t i = 1; i < s.size(); ++i) s[i].us = std::max(s[i].us, s[i - 1].us);
    *out = s;
    return true;
}

double interpolate(const std::vector<Sample>& s, int64_t M) {
    if (M <= 0) return 0.0;
    if (M <= s.front().M) return s.front().us;
    if (M >= s.back().M) return s.back().us * (double)M / (double)s.back().M;
    size_t hi = 1;
    while (s[hi].M < M) ++hi;
    const Sample& a = s[hi - 1];
    const Sample& b = s[hi];
    return a.us + (b.us - a.us) * (double)(M - a.M) / (double)(b.M - a.M);
}

// Per-linear sample lists resolved once, then the step time at any M.
struct Model {
    std::vector<std::vector<Sample>> samples;
    std::vector<int32_t> counts;
    double fixed_us = 0.0;
    double at(int64_t M) const {
        double t = fixed_us;
        for (size_t i = 0; i < samples.size(); ++i) t += counts[i] * interpolate(samples[i], M);
        return t;
    }
};

// The dispatcher's table holds one row per shape and code order (row order, and the tile order of
// spear_tile_w4 for the stream-K kernel); a layer that holds both orders runs the faster one, so
// the latency table keeps, per (M, N, K, compensator or not), the fastest row.
struct BuiltinTable {
    spear_latency_entry* rows = nullptr;
    int32_t len = 0;
};
const BuiltinTable& builtin() {
    static BuiltinTable t = [] {
        BuiltinTable b;
        b.rows = (spear_latency_entry*)calloc((size_t)kTableLen, sizeof(spear_latency_entry));
        for (int32_t i = 0; b.rows && i < kTableLen; ++i) {
            int32_t j = 0;
            while (j < b.len && !(b.rows[j].M == kTable[i].M && b.rows[j].N == kTable[i].N &&
                                  b.rows[j].K == kTable[i].K && b.rows[j].has_ec == kTable[i].has_ec))
                ++j;
            if (j == b.len) {
                b.rows[j].M = kTable[i].M;
                b.rows[j].N = kTable[i].N;
                b.rows[j].K = kTable[i].K;
                b.rows[j].has_ec = kTable[i].has_ec;
                b.rows[j].us = kTable[i].us;
                ++b.len;
            } else if (kTable[i].us < b.rows[j].us) {
                b.rows[j].us = kTable[i].us;
            }
        }
        return b;
    }();
    return t;
}

spear_status build_model(const spear_linear_desc* linears, int32_t n, const spear_latency_entry* lut, int32_t lut_len,
                         double fixed_us, Model* m) {
    if (!linears || n <= 0 || !(fixed_us >= 0.0) || !isfinite(fixed_us)) return SPEAR_ERR_INVALID_ARG;
    if (!lut) {
        lut = builtin().rows;
        lut_len = builtin().len;
        if (!lut) return SPEAR_ERR_INVALID_ARG;
    } else if (lut_len <= 0) {
        return SPEAR_ERR_INVALID_ARG;
    } else {
        for (int32_t i = 0; i < lut_len; ++i)
            if (lut[i].M <= 0 || !(lut[i].us >= 0.0) || !isfinite(lut[i].us)) return SPEAR_ERR_INVALID_ARG;
    }
    m->samples.assign((size_t)n, {});
    m->counts.assign((size_t)n, 0);
    m->fixed_us = fixed_us;
    for (int32_t i = 0; i < n; ++i) {
        const spear_linear_desc& d = linears[i];
        if (d.N <= 0 || d.K <= 0 || d.rank < 0 || d.count < 0) return SPEAR_ERR_INVALID_ARG;
        m->counts[(size_t)i] = d.count;
        if (d.count == 0) {
            m->samples[(size_t)i] = {{1, 0.0}};
            continue;
        }
        if (!samples_for(lut, lut_len, d.N, d.K, d.rank > 0 ? 1 : 0, &m->samples[(size_t)i]))
            return SPEAR_ERR_UNSUPPORTED_SHAPE;
    }
    return SPEAR_OK;
}

}  // namespace
}  // namespace spear

using namespace spear;

extern "C" {

spear_status spear_latency_table(spear_latency_entry* out, int32_t capacity, int32_t* len_out) {
    if (!len_out) return SPEAR_ERR_INVALID_ARG;
    const BuiltinTable& t = builtin();
    if (!t.rows) return SPEAR_ERR_INVALID_ARG;
    *len_out = t.len;
    if (!out) return SPEAR_OK;
    if (capacity < t.len) return SPEAR_ERR_INVALID_ARG;
    for (int32_t i = 0; i < t.len; ++i) out[i] = t.rows[i];
    return SPEAR_OK;
}

spear_status spear_predict_step_us(const spear_linear_desc* linears, int32_t n_linears, int64_t M, double fixed_us,
                                   const spear_latency_entry* lut, int32_t lut_len, double* us_out) {
    if (!us_out || M < 0 || M > SLO_M_MAX) return SPEAR_ERR_INVALID_ARG;
    Model m;
    spear_status st = build_model(linears, n_linears, lut, lut_len, fixed_us, &m);
    if (st != SPEAR_OK) return st;
    *us_out = m.at(M);
    return SPEAR_OK;
}

spear_status spear_pick_prefill_chunk(const spear_linear_desc* linears, int32_t n_linears, int64_t decode_tokens,
                                      int64_t max_chunk, int64_t granule, double slo_us, double fixed_us,
                                      const spear_latency_entry* lut, int32_t lut_len, int64_t* chunk_out,
                                      double* predicted_us_out) {
    if (!chunk_out || !predicted_us_out) return SPEAR_ERR_INVALID_ARG;
    if (decode_tokens < 0 || decode_tokens > SLO_M_MAX || max_chunk < 0 || granule <= 0) return SPEAR_ERR_INVALID_ARG;
    if (!(slo_us > 0.0) || !isfinite(slo_us)) return SPEAR_ERR_INVALID_ARG;
    Model m;
    spear_status st = build_model(linears, n_linears, lut, lut_len, fixed_us, &m);
    if (st != SPEAR_OK) return st;
    // Chunks c * granule for c in [0, hi]; the step time is nondecreasing in c.
    const int64_t room = std::min(max_chunk, SLO_M_MAX - decode_tokens);
    int64_t lo = 0, hi = room / granule;
    if (m.at(decode_tokens) > slo_us) {
        *chunk_out = 0;                          // even the decode tokens alone miss the target
        *predicted_us_out = m.at(decode_tokens);
        return SPEAR_OK;
    }
    while (lo < hi) {                            // invariant: chunk lo * granule meets the target
        const int64_t mid = lo + (hi - lo + 1) / 2;
        if (m.at(decode_tokens + mid * granule) <= slo_us) lo = mid;
        else hi = mid - 1;
    }
    *chunk_out = lo * granule;
    *predicted_us_out = m.at(decode_tokens + lo * granule);
    return SPEAR_OK;
}

}  // extern "C"
