// pack.cu -- RTN per-output-channel asymmetric int4 packer and the unpack test hook.
//
// SPEAR (Post-Quantization Error-Adaptive Recovery), technical summary section 3.1: weights
// are quantised to 4 bits per output channel with round-to-nearest.  The steps are IEEE fp32
// operations with explicit round-to-nearest intrinsics, so the codes, scales and zero-points are
// bit-identical to any other conforming evaluation of the same rule (see include/spear.h).
//
// One warp per output row: a min/max pass over the row, the scalar scale/zero computation in
// lane 0's registers (all lanes compute it redundantly), then a quantise-and-pack pass in which
// each lane turns 8 consecutive weights into one 32-bit word of nibbles.
#include "common.cuh"

namespace spear {

template <typename T>
SPEAR_DEVI float load_w(const T* p);
template <>
SPEAR_DEVI float load_w<float>(const float* p) { return *p; }
template <>
SPEAR_DEVI float load_w<uint16_t>(const uint16_t* p) { return bf16_bits_to_f32(*p); }

template <typename T>
SPEAR_DEVI void load8(const T* p, float v[8]);
template <>
SPEAR_DEVI void load8<float>(const float* p, float v[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0];
    const float4 b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
SPEAR_DEVI void load8<uint16_t>(const uint16_t* p, float v[8]) {
    const uint4 a = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

SPEAR_DEVI float clamp_0_15(float v) { return v < 0.0f ? 0.0f : (v > 15.0f ? 15.0f : v); }

SPEAR_DEVI uint32_t code_of(float w, float s, float zf) {
    const float r = rintf(__fdiv_rn(w, s));
    return (uint32_t)clamp_0_15(__fadd_rn(r, zf));
}

template <typename T>
__global__ void __launch_bounds__(256) pack_w4_kernel(const T* __restrict__ W, int64_t N, int64_t K,
                                                      uint8_t* __restrict__ packed,
                                                      __half* __restrict__ scale, __half* __restrict__ zero) {
    const int lane = threadIdx.x & 31;
    const int64_t n = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (n >= N) return;
    const T* row = W + n * K;
    const bool vec = (K % 8) == 0;

    // Range of the row, always containing 0 (min/max are exact in any order).
    float lo = 0.0f, hi = 0.0f;
    if (vec) {
        for (int64_t k = (int64_t)lane * 8; k < K; k += 256) {
            float v[8];
            load8<T>(row + k, v);
#pragma unroll
            for (int i = 0; i < 8; ++i) { lo = fminf(lo, v[i]); hi = fmaxf(hi, v[i]); }
        }
    } else {
        for (int64_t k = lane; k < K; k += 32) {
            const float v = load_w<T>(row + k);
            lo = fminf(lo, v); hi = fmaxf(hi, v);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
    }
    if (hi == lo) { lo = -1.0f; hi = 1.0f; }
    __half sh = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
    float s = __half2float(sh);
    if (s == 0.0f) {  // the scale underflows binary16: treat the row as all-zero
        lo = -1.0f; hi = 1.0f;
        sh = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
        s = __half2float(sh);
    }
    // z is an integer; going through int gives +0 rather than -0 when lo == 0.
    const float zf = (float)(int)clamp_0_15(rintf(__fdiv_rn(-lo, s)));
    if (lane == 0) {
        scale[n] = sh;
        zero[n] = __float2half_rn(zf);
    }

    uint8_t* prow = packed + n * (K / 2);
    if (vec) {
        for (int64_t k = (int64_t)lane * 8; k < K; k += 256) {
            float v[8];
            load8<T>(row + k, v);
            uint32_t word = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) word |= code_of(v[i], s, zf) << (4 * i);
            *reinterpret_cast<uint32_t*>(prow + k / 2) = word;
        }
    } else {
        for (int64_t b = lane; b < K / 2; b += 32) {
            const uint32_t q0 = code_of(load_w<T>(row + 2 * b), s, zf);
            const uint32_t q1 = code_of(load_w<T>(row + 2 * b + 1), s, zf);
            prow[b] = (uint8_t)(q0 | (q1 << 4));
        }
    }
}

// Test hook: codes and the exact bf16 (q - z) values produced by the kernels' converter.
__global__ void __launch_bounds__(256) unpack_w4_kernel(const uint8_t* __restrict__ packed,
                                                        const __half* __restrict__ zero, int64_t N, int64_t K,
                                                        uint8_t* __restrict__ q_out,
                                                        uint16_t* __restrict__ qz_out) {
    // One thread per 8 codes (K % 8 == 0) or per 2 codes otherwise.
    const int64_t words_per_row = (K % 8 == 0) ? K / 8 : 0;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (words_per_row) {
        if (idx >= N * words_per_row) return;
        const int64_t n = idx / words_per_row, kw = idx % words_per_row;
        const uint32_t w = *reinterpret_cast<const uint32_t*>(packed + n * (K / 2) + kw * 4);
        const uint32_t z = (uint32_t)__half2float(zero[n]);
        if (q_out) {
#pragma unroll
            for (int i = 0; i < 8; ++i) q_out[n * K + kw * 8 + i] = (uint8_t)((w >> (4 * i)) & 0xF);
        }
        if (qz_out) {
            uint32_t nat[4];
            cvt_w4_pairs_natural(w, zero_bias_bf16x2(z), nat);
            uint32_t* dst = reinterpret_cast<uint32_t*>(qz_out + n * K + kw * 8);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = nat[i];
        }
    } else {
        if (idx >= N * (K / 2)) return;
        const int64_t n = idx / (K / 2), b = idx % (K / 2);
        const uint32_t v = packed[n * (K / 2) + b];
        const uint32_t z = (uint32_t)__half2float(zero[n]);
        if (q_out) {
            q_out[n * K + 2 * b] = (uint8_t)(v & 0xF);
            q_out[n * K + 2 * b + 1] = (uint8_t)(v >> 4);
        }
        if (qz_out) {
            uint32_t nat[4];
            cvt_w4_pairs_natural(v, zero_bias_bf16x2(z), nat);
            *reinterpret_cast<uint32_t*>(qz_out + n * K + 2 * b) = nat[0];
        }
    }
}

// Tile order of the register-path stream kernel: one thread per 32-bit word of the output.
// Output word d = ((T * K/128 + B) * 128 + r) * 16 + i, i = 4c + w, comes from row 128 T + r, word
// 16 B + s of the row order with s = 2c + w (w < 2) or 8 + 2c + w - 2 (w >= 2); code j of the word
// moves from nibble j to nibble (j / 2) + 4 (j % 2).
__global__ void __launch_bounds__(256) tile_w4_kernel(const uint32_t* __restrict__ packed, int64_t N, int64_t K,
                                                      uint32_t* __restrict__ tiled) {
    const int64_t d = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t words = N * (K / 8);
    if (d >= words) return;
    const int64_t nblk = K / 128;
    const int64_t i = d & 15, r = (d >> 4) & 127, tb = d >> 11;
    const int64_t T = tb / nblk, B = tb % nblk;
    const int64_t c = i >> 2, wi = i & 3;
    const int64_t src = wi < 2 ? 2 * c + wi : 8 + 2 * c + (wi - 2);
    const uint32_t w = packed[(T * 128 + r) * (K / 8) + B * 16 + src];
    uint32_t o = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) o |= ((w >> (4 * j)) & 0xFu) << (4 * ((j >> 1) + 4 * (j & 1)));
    tiled[d] = o;
}

cudaError_t launch_tile_w4(const void* packed, int64_t N, int64_t K, void* tiled, cudaStream_t stream) {
    const int64_t words = N * (K / 8);
    const dim3 grid((unsigned)((words + 255) / 256));
    cudaGetLastError();   // report this launch only, not an earlier call's error
    tile_w4_kernel<<<grid, 256, 0, stream>>>((const uint32_t*)packed, N, K, (uint32_t*)tiled);
    return cudaGetLastError();
}

cudaError_t launch_pack_w4(const void* W, bool w_is_bf16, int64_t N, int64_t K, void* packed, void* scale,
                           void* zero, cudaStream_t stream) {
    const int rows_per_block = 8;
    const dim3 grid((unsigned)((N + rows_per_block - 1) / rows_per_block));
    cudaGetLastError();   // report this launch only, not an earlier call's error
    if (w_is_bf16)
        pack_w4_kernel<uint16_t><<<grid, 256, 0, stream>>>((const uint16_t*)W, N, K, (uint8_t*)packed,
                                                           (__half*)scale, (__half*)zero);
    else
        pack_w4_kernel<float><<<grid, 256, 0, stream>>>((const float*)W, N, K, (uint8_t*)packed,
                                                        (__half*)scale, (__half*)zero);
    return cudaGetLastError();
}

cudaError_t launch_unpack_w4(const void* packed, const void* zero, int64_t N, int64_t K, void* q_out,
                             void* qz_out, cudaStream_t stream) {
    const int64_t items = (K % 8 == 0) ? N * (K / 8) : N * (K / 2);
    const dim3 grid((unsigned)((items + 255) / 256));
    cudaGetLastError();   // report this launch only, not an earlier call's error
    unpack_w4_kernel<<<grid, 256, 0, stream>>>((const uint8_t*)packed, (const __half*)zero, N, K,
                                               (uint8_t*)q_out, (uint16_t*)qz_out);
    return cudaGetLastError();
}

}  // namespace spear
