// common.cuh -- device helpers shared by the sm_100a kernels of the W4 + gated-EC layer.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/spear.h"

#define SPEAR_DEVI __device__ __forceinline__

namespace spear {

// ---------------------------------------------------------------------------------------------
// int4 -> bf16 conversion.
//
// A nibble q in [0, 15] placed in the low mantissa bits of bf16 128.0 (bits 0x4300) encodes the
// value 128 + q exactly (bf16 keeps 7 fraction bits; 128..143 needs 4).  Subtracting the bf16
// value 128 + z (also exact) leaves q - z in [-15, 15], exact in bf16.  The per-channel scale s[n]
// is applied later, to the fp32 accumulator, so the tensor-core operand is the exact integer q - z.
// ---------------------------------------------------------------------------------------------

// bf16x2 pattern holding (128 + z, 128 + z) for an integer zero-point z in [0, 15].
SPEAR_DEVI uint32_t zero_bias_bf16x2(uint32_t z) { return 0x43004300u | z | (z << 16); }

SPEAR_DEVI uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

SPEAR_DEVI uint32_t lop_and_or(uint32_t a, uint32_t mask, uint32_t orv) {
    // (a & mask) | orv in one LOP3.
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(orv));
    return d;
}

SPEAR_DEVI uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// 8 codes of one 32-bit packed word (code i in bits 4i..4i+3, i.e. k = k0 + i) ->
// out[i] = bf16x2 (q[i] - z, q[i+4] - z) for i = 0..3.  The pairing (i, i+4) is the one a
// single mask per shift produces; the caller permutes the other MMA operand to match.
SPEAR_DEVI void cvt_w4_pairs_i_i4(uint32_t w, uint32_t zb, uint32_t out[4]) {
    out[0] = bf16x2_sub(lop_and_or(w, 0x000F000Fu, 0x43004300u), zb);
    out[1] = bf16x2_sub(lop_and_or(w >> 4, 0x000F000Fu, 0x43004300u), zb);
    out[2] = bf16x2_sub(lop_and_or(w >> 8, 0x000F000Fu, 0x43004300u), zb);
    out[3] = bf16x2_sub(lop_and_or(w >> 12, 0x000F000Fu, 0x43004300u), zb);
}

// Same codes in natural order: out[i] = bf16x2 (q[2i] - z, q[2i+1] - z) (low half = even k).
SPEAR_DEVI void cvt_w4_pairs_natural(uint32_t w, uint32_t zb, uint32_t out[4]) {
    const uint32_t w4 = w >> 4;
    // byte j of w holds (q[2j] | q[2j+1] << 4); byte j of w4 holds q[2j+1] in its low nibble.
    // Selector: result byte 0 <- w.byte j (keeps q[2j]), result byte 2 <- w4.byte j (keeps q[2j+1]).
    out[0] = bf16x2_sub(lop_and_or(prmt(w, w4, 0x4400u), 0x000F000Fu, 0x43004300u), zb);
    out[1] = bf16x2_sub(lop_and_or(prmt(w, w4, 0x5511u), 0x000F000Fu, 0x43004300u), zb);
    out[2] = bf16x2_sub(lop_and_or(prmt(w, w4, 0x6622u), 0x000F000Fu, 0x43004300u), zb);
    out[3] = bf16x2_sub(lop_and_or(prmt(w, w4, 0x7733u), 0x000F000Fu, 0x43004300u), zb);
}

// ---------------------------------------------------------------------------------------------
// Warp-level tensor-core MMA (m16n8k16, bf16 in, fp32 accumulate).
// ---------------------------------------------------------------------------------------------
SPEAR_DEVI void mma_bf16_16816(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------------------------
// Global loads.
// ---------------------------------------------------------------------------------------------
SPEAR_DEVI uint4 ldg_stream_u4(const void* p) {
    // Weight stream: read once, keep it out of L1.
    uint4 v;
    asm volatile("ld.global.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

SPEAR_DEVI uint4 ldg_u4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

SPEAR_DEVI uint32_t ldg_u32_nc(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// ---------------------------------------------------------------------------------------------
// Programmatic dependent launch controls (no-ops when the grid was launched without PDL).
// ---------------------------------------------------------------------------------------------
SPEAR_DEVI void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
SPEAR_DEVI void pdl_wait_primary() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

SPEAR_DEVI int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }

SPEAR_DEVI float bf16_bits_to_f32(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }

// ---------------------------------------------------------------------------------------------
// Cluster helpers (distributed shared memory).
// ---------------------------------------------------------------------------------------------
// Split form of the cluster barrier: the arrive at kernel start and the wait before the first
// remote store make sure every CTA of the cluster is running before its shared memory is written.
SPEAR_DEVI void cluster_arrive_relaxed() { asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory"); }
SPEAR_DEVI void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }
SPEAR_DEVI void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Store to the same shared-memory offset in cluster rank `rank`.
SPEAR_DEVI void st_dsmem_f32(float* local, unsigned rank, float v) {
    uint32_t la = (uint32_t)__cvta_generic_to_shared(local), ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(la), "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}
SPEAR_DEVI void st_dsmem_f4(float4* local, unsigned rank, float4 v) {
    uint32_t la = (uint32_t)__cvta_generic_to_shared(local), ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(la), "r"(rank));
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(ra), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

}  // namespace spear
