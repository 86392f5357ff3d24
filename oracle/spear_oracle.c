/*
 * spear_oracle.c -- plain, slow CPU oracle for the W4 + per-token-gated
 * error-compensator linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  It shares no code,
 * header or constant with the CUDA library, and neither one includes the other.
 *
 * What it computes (SPEAR: A System for Post-Quantization Error-Adaptive
 * Recovery, technical summary section 2.1A "Input-adaptive Error Compensators",
 * and the English abstract):
 *
 *   y[m,n] = sum_k x[m,k] * What[n,k]  +  g[m] * sum_j t[m,j] * B[j,n]
 *   What[n,k] = (q[n,k] - z[n]) * s[n]                (per-channel asymmetric W4)
 *   t[m,j]    = sum_k x[m,k] * A[k,j]                  (EC down-projection)
 *   g[m]      = 1 / (1 + exp(-(sum_k x[m,k] * w_g[k] + b_g)))   (scalar gate)
 *
 * The pages' effective-weight form W + alpha * B diag(gamma(Ax)) A is taken with
 * alpha = 1 and gamma a scalar sigmoid gate over x (the scalar gate is the linear
 * special case of the pages' bottleneck gate).  A is stored [K, r] and B [r, N],
 * i.e. the transposes of the pages' r x K and N x r factors.
 *
 * Quantisation (round-to-nearest, per output channel; the RTN backend the
 * summary's Llama-3.2-1B example uses, section 3.1) is defined here in IEEE
 * fp32 operations, each correctly rounded, because it decides integers that must
 * come out bit-identical on any conforming implementation:
 *
 *   lo = min(min_k W[n,k], 0),  hi = max(max_k W[n,k], 0)
 *   if hi == lo:               lo = -1, hi = 1
 *   s32 = fl32(fl32(hi - lo) / 15);  s = fp16_rne(s32)
 *   if s == 0:  the row is treated as all-zero (lo = -1, hi = 1, recompute s)
 *   z = clamp(rint_even(fl32(-lo / s)), 0, 15)
 *   q[n,k] = clamp(rint_even(fl32(W[n,k] / s)) + z, 0, 15)
 *
 * Packing: byte b of row n holds q[n,2b] in bits 0..3 and q[n,2b+1] in bits 4..7.
 * s and z are stored as IEEE binary16 bit patterns (z is an exact integer).
 *
 * Also here: the group-wise variant (scale and zero-point per group of G consecutive k of a row,
 * the per-channel steps applied to each group; oracle_w4ec_gemm_grouped) and the pages'
 * bottleneck-MLP gate (oracle_w4ec_gemm_mlp).
 *
 * Everything after quantisation runs in fp64, sums in ascending index order.
 *
 * Build: gcc -O2 -std=c11 -fno-fast-math -ffp-contract=off -fopenmp -shared -fPIC.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------- */
/* Number formats, written from the IEEE 754 binary16 / bfloat16 definitions. */

/* fp32 -> binary16, round to nearest, ties to even; overflow -> inf. */
uint16_t oracle_f32_to_f16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t exp = (u >> 23) & 0xFFu;
    uint32_t man = u & 0x7FFFFFu;
    if (exp == 0xFFu) {                                /* inf or NaN */
        return (uint16_t)(sign | 0x7C00u | (man ? 0x200u : 0u));
    }
    /* Work with the exact value |f| = man24 * 2^(e2) where man24 includes the
     * hidden bit.  binary16: normal values 2^-14 .. 65504, subnormal quantum 2^-24. */
    int e = (int)exp - 127;                            /* unbiased exponent */
    uint32_t m24 = exp ? (man | 0x800000u) : man;      /* 24-bit significand */
    if (!exp) e = -126;                                /* fp32 subnormal */
    if (m24 == 0) return sign;
    /* Target quantum: 2^(e16 - 10) with e16 = max(e, -14). */
    int e16 = e < -14 ? -14 : e;
    /* value = m24 * 2^(e - 23); in units of the quantum: m24 * 2^(e - 23 - e16 + 10) */
    int sh = (e - 23) - (e16 - 10);                    /* <= 0 always (sh = -13 for normals) */
    uint32_t q;
    if (sh >= 0) {
        q = m24 << sh;
    } else {
        int rs = -sh;
        if (rs > 31) {
            q = 0;                                     /* far below half a quantum */
            return sign;
        }
        uint32_t kept = m24 >> rs;
        uint32_t rem = m24 & ((1u << rs) - 1u);
        uint32_t half = 1u << (rs - 1);
        q = kept;
        if (rem > half || (rem == half && (kept & 1u))) q += 1;
    }
    /* q is the significand in quanta of 2^(e16-10); renormalise. */
    if (q == 0) return sign;
    if (e16 == -14 && q < 1024u) {                     /* subnormal result */
        return (uint16_t)(sign | q);
    }
    /* q in [1024, 2048]: normal; 2048 means carry into the next binade. */
    int E = e16;
    if (q >= 2048u) { q >>= 1; E += 1; }
    if (E > 15) return (uint16_t)(sign | 0x7C00u);     /* overflow */
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)(q & 0x3FFu));
}

/* binary16 -> fp64 (exact). */
double oracle_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int exp = (h >> 10) & 0x1F;
    int man = h & 0x3FF;
    double v;
    if (exp == 0) v = ldexp((double)man, -24);
    else if (exp == 31) v = man ? NAN : INFINITY;
    else v = ldexp((double)(man | 0x400), exp - 25);
    return sign ? -v : v;
}

/* bfloat16 -> fp64 (exact): the top half of an fp32 pattern. */
double oracle_bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* ------------------------------------------------------------------------- */
/* RTN per-channel asymmetric W4 quantisation of one row (fp32 IEEE steps). */

static float clamp_0_15(float v) { return v < 0.0f ? 0.0f : (v > 15.0f ? 15.0f : v); }

static void quantize_row(const float* w, int64_t K, uint8_t* q, uint16_t* s_bits, uint16_t* z_bits)
{
    float lo = 0.0f, hi = 0.0f;                        /* the range always contains 0 */
    for (int64_t k = 0; k < K; ++k) {
        if (w[k] < lo) lo = w[k];
        if (w[k] > hi) hi = w[k];
    }
    if (hi == lo) { lo = -1.0f; hi = 1.0f; }
    float range = hi - lo;
    float s32 = range / 15.0f;
    uint16_t sb = oracle_f32_to_f16(s32);
    float s = (float)oracle_f16_to_f64(sb);
    if (s == 0.0f) {                                   /* scale underflows binary16 */
        lo = -1.0f; hi = 1.0f;
        range = hi - lo;
        s32 = range / 15.0f;
        sb = oracle_f32_to_f16(s32);
        s = (float)oracle_f16_to_f64(sb);
    }
    /* z is an integer zero-point: going through int makes a zero z the canonical +0. */
    float negl = -lo;
    float zf = (float)(int)clamp_0_15(rintf(negl / s));
    for (int64_t k = 0; k < K; ++k) {
        float r = rintf(w[k] / s);
        q[k] = (uint8_t)clamp_0_15(r + zf);
    }
    *s_bits = sb;
    *z_bits = oracle_f32_to_f16(zf);                   /* exact: an integer in [0, 15] */
}

/* W fp32 [N,K] -> q uint8 [N,K] (values 0..15), s and z binary16 bits [N]. */
void oracle_quantize_rtn(const float* W, int64_t N, int64_t K,
                         uint8_t* q, uint16_t* s_bits, uint16_t* z_bits)
{
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        quantize_row(W + n * K, K, q + n * K, s_bits + n, z_bits + n);
}

/* q uint8 [N,K] -> packed [N, K/2]: low nibble = even k, high nibble = odd k. */
void oracle_pack_nibbles(const uint8_t* q, int64_t N, int64_t K, uint8_t* packed)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t b = 0; b < K / 2; ++b)
            packed[n * (K / 2) + b] = (uint8_t)((q[n * K + 2 * b] & 0xF) | ((q[n * K + 2 * b + 1] & 0xF) << 4));
}

/* packed [N, K/2] -> q uint8 [N,K]. */
void oracle_unpack_nibbles(const uint8_t* packed, int64_t N, int64_t K, uint8_t* q)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t b = 0; b < K / 2; ++b) {
            uint8_t v = packed[n * (K / 2) + b];
            q[n * K + 2 * b] = v & 0xF;
            q[n * K + 2 * b + 1] = v >> 4;
        }
}

/* W fp32 -> packed + s + z (quantise then pack). */
void oracle_pack_w4(const float* W, int64_t N, int64_t K,
                    uint8_t* packed, uint16_t* s_bits, uint16_t* z_bits)
{
    uint8_t* q = (uint8_t*)malloc((size_t)(N * K));
    oracle_quantize_rtn(W, N, K, q, s_bits, z_bits);
    oracle_pack_nibbles(q, N, K, packed);
    free(q);
}

/* Dequantised row n in fp64: What[n,k] = (q - z) * s (exact in fp64). */
static void dequant_row(const uint8_t* packed_row, int64_t K, uint16_t s_bits, uint16_t z_bits, double* out)
{
    double s = oracle_f16_to_f64(s_bits);
    double z = oracle_f16_to_f64(z_bits);
    for (int64_t b = 0; b < K / 2; ++b) {
        uint8_t v = packed_row[b];
        out[2 * b] = ((double)(v & 0xF) - z) * s;
        out[2 * b + 1] = ((double)(v >> 4) - z) * s;
    }
}

void oracle_dequant_w4(const uint8_t* packed, const uint16_t* s_bits, const uint16_t* z_bits,
                       int64_t N, int64_t K, double* What)
{
    for (int64_t n = 0; n < N; ++n)
        dequant_row(packed + n * (K / 2), K, s_bits[n], z_bits[n], What + n * K);
}

/* ------------------------------------------------------------------------- */
/* Error compensator: t = x A, p = x w_g + b_g, g = sigmoid(p), all fp64.     */

static double sigmoid(double p) { return 1.0 / (1.0 + exp(-p)); }

/* x bf16 [M,K], A bf16 [K,r], w_g bf16 [K] -> t fp64 [M,r], p fp64 [M], g fp64 [M]. */
void oracle_ec_gate(const uint16_t* x, int64_t M, int64_t K,
                    const uint16_t* A, int32_t r, const uint16_t* wg, float b_g,
                    double* t, double* p, double* g)
{
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int32_t j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += oracle_bf16_to_f64(x[m * K + k]) * oracle_bf16_to_f64(A[k * r + j]);
            t[m * r + j] = acc;
        }
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k)
            acc += oracle_bf16_to_f64(x[m * K + k]) * oracle_bf16_to_f64(wg[k]);
        acc += (double)b_g;
        p[m] = acc;
        g[m] = sigmoid(acc);
    }
}

/* ------------------------------------------------------------------------- */
/* The full layer in fp64.                                                    */

/* y[m,n] = sum_k x[m,k] What[n,k] + g[m] sum_j t[m,j] B[j,n].
 * A == NULL or r == 0 -> plain W4 layer (no compensator).  y is fp64 [M,N]. */
void oracle_w4ec_gemm(const uint16_t* x, int64_t M, int64_t N, int64_t K,
                      const uint8_t* packed, const uint16_t* s_bits, const uint16_t* z_bits,
                      const uint16_t* A, const uint16_t* B, const uint16_t* wg, float b_g, int32_t r,
                      double* y)
{
    int has_ec = (A != NULL && B != NULL && wg != NULL && r > 0);
    double* xd = (double*)malloc(sizeof(double) * (size_t)(M * K));
    for (int64_t i = 0; i < M * K; ++i) xd[i] = oracle_bf16_to_f64(x[i]);
    double *t = NULL, *p = NULL, *g = NULL;
    if (has_ec) {
        t = (double*)malloc(sizeof(double) * (size_t)(M * r));
        p = (double*)malloc(sizeof(double) * (size_t)M);
        g = (double*)malloc(sizeof(double) * (size_t)M);
        oracle_ec_gate(x, M, K, A, r, wg, b_g, t, p, g);
    }
    #pragma omp parallel
    {
        double* wrow = (double*)malloc(sizeof(double) * (size_t)K);
        #pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            dequant_row(packed + n * (K / 2), K, s_bits[n], z_bits[n], wrow);
            for (int64_t m = 0; m < M; ++m) {
                const double* xr = xd + m * K;
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k) acc += xr[k] * wrow[k];
                if (has_ec) {
                    double e = 0.0;
                    for (int32_t j = 0; j < r; ++j) e += t[m * r + j] * oracle_bf16_to_f64(B[(int64_t)j * N + n]);
                    acc += g[m] * e;
                }
                y[m * N + n] = acc;
            }
        }
        free(wrow);
    }
    free(xd);
    free(t); free(p); free(g);
}

/* Group-wise scales (the GPTQ/AWQ-style backends the technical summary's section 3.1 lists as
 * compatible): every G consecutive k of a row have their own scale and zero-point, found by the
 * same RTN steps as above applied to that group alone, so the grouped format of W [N, K] is the
 * per-channel format of W viewed as [N * K/G, G]: packed [N, K/2] unchanged, s and z [N, K/G].
 *   What[n,k] = (q[n,k] - z[n, k/G]) * s[n, k/G]
 *   y[m,n]    = sum_k x[m,k] What[n,k] + g[m] sum_j t[m,j] B[j,n]
 * A == NULL or r == 0 -> no compensator.  y is fp64 [M,N]. */
void oracle_w4ec_gemm_grouped(const uint16_t* x, int64_t M, int64_t N, int64_t K, int64_t G,
                              const uint8_t* packed, const uint16_t* s_bits, const uint16_t* z_bits,
                              const uint16_t* A, const uint16_t* B, const uint16_t* wg, float b_g, int32_t r,
                              double* y)
{
    int has_ec = (A != NULL && B != NULL && wg != NULL && r > 0);
    int64_t ng = K / G;
    double *t = NULL, *p = NULL, *g = NULL;
    if (has_ec) {
        t = (double*)malloc(sizeof(double) * (size_t)(M * r));
        p = (double*)malloc(sizeof(double) * (size_t)M);
        g = (double*)malloc(sizeof(double) * (size_t)M);
        oracle_ec_gate(x, M, K, A, r, wg, b_g, t, p, g);
    }
    #pragma omp parallel
    {
        double* what = (double*)malloc(sizeof(double) * (size_t)K);
        #pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            for (int64_t k = 0; k < K; ++k) {
                uint8_t v = packed[n * (K / 2) + k / 2];
                double q = (double)((k & 1) ? (v >> 4) : (v & 0xF));
                int64_t grp = k / G;
                what[k] = (q - oracle_f16_to_f64(z_bits[n * ng + grp])) * oracle_f16_to_f64(s_bits[n * ng + grp]);
            }
            for (int64_t m = 0; m < M; ++m) {
                double sum = 0.0;
                for (int64_t k = 0; k < K; ++k) sum += oracle_bf16_to_f64(x[m * K + k]) * what[k];
                if (has_ec) {
                    double ec = 0.0;
                    for (int32_t j = 0; j < r; ++j)
                        ec += t[m * r + j] * oracle_bf16_to_f64(B[(int64_t)j * N + n]);
                    sum += g[m] * ec;
                }
                y[m * N + n] = sum;
            }
        }
        free(what);
    }
    free(t); free(p); free(g);
}

/* The pages' gate form (technical summary section 2.1A): effective weight
 * W + alpha * B diag(gamma(Ax)) A, gamma a bottleneck MLP.  The pages do not
 * spell the MLP out; this follows the plainest reading of "bottleneck MLP" over
 * the rank-r projection t = x A, one output per rank component:
 *   h[m,i]     = max(0, sum_j W1[i,j] t[m,j] + b1[i])          i < H   (W1 [H, r])
 *   gamma[m,j] = 1 / (1 + exp(-(sum_i W2[j,i] h[m,i] + b2[j])))   (W2 [r, H])
 *   u[m,j]     = alpha * gamma[m,j] * t[m,j]
 *   y[m,n]     = sum_k x[m,k] What[n,k] + sum_j u[m,j] B[j,n]
 * W1, b1, W2, b2 are fp32; everything is evaluated in fp64.  y is fp64 [M,N]. */
void oracle_w4ec_gemm_mlp(const uint16_t* x, int64_t M, int64_t N, int64_t K,
                          const uint8_t* packed, const uint16_t* s_bits, const uint16_t* z_bits,
                          const uint16_t* A, const uint16_t* B, int32_t r,
                          const float* W1, const float* b1, const float* W2, const float* b2, int32_t H,
                          float alpha, double* y)
{
    /* t = x A from the scalar-gate path (its gate outputs are not used here). */
    uint16_t* wg0 = (uint16_t*)calloc((size_t)K, sizeof(uint16_t));
    double* t = (double*)malloc(sizeof(double) * (size_t)(M * r));
    double* p = (double*)malloc(sizeof(double) * (size_t)M);
    double* g = (double*)malloc(sizeof(double) * (size_t)M);
    oracle_ec_gate(x, M, K, A, r, wg0, 0.0f, t, p, g);
    double* u = (double*)malloc(sizeof(double) * (size_t)(M * r));
    double* h = (double*)malloc(sizeof(double) * (size_t)H);
    for (int64_t m = 0; m < M; ++m) {
        const double* tm = t + m * r;
        for (int32_t i = 0; i < H; ++i) {
            double pre = (double)b1[i];
            for (int32_t j = 0; j < r; ++j) pre += (double)W1[(int64_t)i * r + j] * tm[j];
            h[i] = pre > 0.0 ? pre : 0.0;
        }
        for (int32_t j = 0; j < r; ++j) {
            double pre = (double)b2[j];
            for (int32_t i = 0; i < H; ++i) pre += (double)W2[(int64_t)j * H + i] * h[i];
            u[m * r + j] = (double)alpha * (1.0 / (1.0 + exp(-pre))) * tm[j];
        }
    }
    /* Main term: the plain layer; then the compensator term. */
    oracle_w4ec_gemm(x, M, N, K, packed, s_bits, z_bits, NULL, NULL, NULL, 0.0f, 0, y);
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t m = 0; m < M; ++m) {
            double e = 0.0;
            for (int32_t j = 0; j < r; ++j) e += u[m * r + j] * oracle_bf16_to_f64(B[(int64_t)j * N + n]);
            y[m * N + n] += e;
        }
    free(wg0); free(t); free(p); free(g); free(u); free(h);
}

/* Same layer, evaluated only at `count` sampled outputs (mi[c], ni[c]) -> y[c].
 * Used where the full product is too large for the CPU (the full-size workloads). */
void oracle_w4ec_gemm_sampled(const uint16_t* x, int64_t M, int64_t N, int64_t K,
                              const uint8_t* packed, const uint16_t* s_bits, const uint16_t* z_bits,
                              const uint16_t* A, const uint16_t* B, const uint16_t* wg, float b_g, int32_t r,
                              const int64_t* mi, const int64_t* ni, int64_t count, double* y)
{
    (void)M;
    int has_ec = (A != NULL && B != NULL && wg != NULL && r > 0);
    #pragma omp parallel
    {
        double* wrow = (double*)malloc(sizeof(double) * (size_t)K);
        double* t = has_ec ? (double*)malloc(sizeof(double) * (size_t)r) : NULL;
        #pragma omp for schedule(dynamic, 16)
        for (int64_t c = 0; c < count; ++c) {
            int64_t m = mi[c], n = ni[c];
            dequant_row(packed + n * (K / 2), K, s_bits[n], z_bits[n], wrow);
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += oracle_bf16_to_f64(x[m * K + k]) * wrow[k];
            if (has_ec) {
                double pm, gm;
                oracle_ec_gate(x + m * K, 1, K, A, r, wg, b_g, t, &pm, &gm);
                double e = 0.0;
                for (int32_t j = 0; j < r; ++j) e += t[j] * oracle_bf16_to_f64(B[(int64_t)j * N + n]);
                acc += gm * e;
            }
            y[c] = acc;
        }
        free(wrow);
        free(t);
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
