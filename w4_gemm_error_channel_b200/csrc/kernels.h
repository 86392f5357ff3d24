// kernels.h -- internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stddef.h>
#include <stdint.h>

namespace spear {

// Workspace control block: the first CTRL_BYTES of every workspace.  Must start zeroed; every
// call leaves the tickets zeroed again.  Layout: [0] device error word, then ticket arrays.
constexpr size_t CTRL_BYTES = 128 * 1024;
constexpr size_t CTRL_HEADER_BYTES = 256;
constexpr size_t EC_TICKETS_MAX = 4096;                          // token chunks of 16 -> M <= 65536
constexpr size_t GEMM_TICKETS_MAX = (CTRL_BYTES - CTRL_HEADER_BYTES) / 4 - EC_TICKETS_MAX;
constexpr int64_t M_MAX = 65536;

struct EcPrepassArgs {
    const uint16_t* x;      // bf16 [M, K]
    const uint16_t* A;      // bf16 [K, r]
    const uint16_t* wg;     // bf16 [K]
    float b_g;
    int64_t M, K;
    int rank;
    int64_t k_per_cta;
    float* ec_part;         // [S_ec][M][r + 1]
    float* u;               // [M][r]   u = g * t
    unsigned* tickets;      // [ceil(M / 16)]
};

struct SplitKArgs {
    const uint16_t* x;      // bf16 [M, K]
    const uint8_t* packed;  // [N, K/2]
    const __half* scale;    // [N]
    const __half* zero;     // [N]
    const uint16_t* B;      // bf16 [r, N] (unused when u == nullptr)
    const float* u;         // [M][r] or nullptr (no EC)
    int rank;
    void* y;
    int y_fp32;
    int64_t M, N, K, k_slice;
    float* part;            // [S][M][N] when S > 1
    unsigned* tickets;      // [(N / RT) * ceil(M / TM)]
};

cudaError_t launch_pack_w4(const void* W, bool w_is_bf16, int64_t N, int64_t K, void* packed, void* scale,
                           void* zero, cudaStream_t stream);
cudaError_t launch_unpack_w4(const void* packed, const void* zero, int64_t N, int64_t K, void* q_out,
                             void* qz_out, cudaStream_t stream);

int64_t ec_prepass_token_chunks(int64_t M);
int64_t ec_prepass_k_per_cta(int64_t M, int64_t K, int num_sms);
int64_t ec_prepass_splits(int64_t K, int64_t k_per_cta);
size_t ec_prepass_smem_bytes(int rank);
size_t ec_prepass_max_smem_bytes();
const void* ec_prepass_kernel_ptr();
cudaError_t launch_ec_prepass(const EcPrepassArgs& a, cudaStream_t stream);

// nb in {1,2,4} (tokens per CTA = 8*nb), g in {1,2,4,8} (rows per CTA = 16*g; g=8 needs nb<=2).
cudaError_t launch_splitk(const SplitKArgs& a, int nb, int g, int split, cudaStream_t stream, bool pdl);

}  // namespace spear
