// internal.h -- launchers shared between the C ABI (capi.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace nvfp4 {

// One quantize pass.  Outputs with a null data pointer are not written.
struct QuantParams {
    const uint16_t* x;  // bf16 [rows][cols]
    int64_t rows, cols;
    uint8_t* row_data;  // [rows][cols/2]
    uint8_t* row_sf;    // swizzled scales of the rows x cols operand
    float* row_g;       // tensor scale of the row orientation
    uint8_t* col_data;  // [cols][rows/2]
    uint8_t* col_sf;    // swizzled scales of the cols x rows operand
    float* col_g;
    const uint32_t* amax_words;  // [0] max|x| bits, [1] max|RHT(col)| bits
    int* status;
    uint64_t seed;
    int row_sr, col_sr, col_rht;
    uint32_t sign_mask;  // bit i set: rotation sign i is -1
    uint32_t rk[20];     // Philox4x32-10 round keys of `seed` (filled by the launchers)
};

// Philox4x32-10 key schedule of a 64-bit seed: round r uses
// (lo(seed) + r * 0x9E3779B9, hi(seed) + r * 0xBB67AE85), mod 2^32.
inline void philox_round_keys(uint64_t seed, uint32_t (&rk)[20]) {
    uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
    for (int r = 0; r < 10; ++r) {
        rk[2 * r] = k0;
        rk[2 * r + 1] = k1;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
}

cudaError_t launch_amax(const uint16_t* x, int64_t rows, int64_t cols, bool col_rht,
                        uint32_t sign_mask, uint32_t* words, int sm_count, cudaStream_t st);
cudaError_t launch_quant_rows(const QuantParams& p, int sm_count, cudaStream_t st);
cudaError_t launch_quant_tile(const QuantParams& p, bool two_d, cudaStream_t st);
cudaError_t launch_sf_pad(uint8_t* sf, int64_t rows, int64_t nb, int sm_count, cudaStream_t st);
cudaError_t launch_rht(const uint16_t* x, float* y, int64_t rows, int64_t cols, int axis,
                       uint32_t sign_mask, int sm_count, cudaStream_t st);

cudaError_t launch_moe_gather(const uint16_t* src, const int32_t* idx, uint16_t* dst, int64_t rows,
                              int64_t cols, int sm_count, cudaStream_t st);
cudaError_t launch_moe_combine(const uint16_t* src, const int32_t* slot, uint16_t* dst,
                               int64_t tokens, int64_t cols, int topk, int sm_count, cudaStream_t st);

struct GemmParams {
    const uint8_t* A;    // [M][K/2]
    const uint8_t* sfA;  // swizzled
    const uint8_t* B;    // [N][K/2]
    const uint8_t* sfB;
    const float* scale_a;
    const float* scale_b;
    float alpha;
    int64_t M, N, K;
    void* D_bf16;
    float* D_f32;
    int* status;
};
cudaError_t launch_gemm(const GemmParams& p, int sm_count, cudaStream_t st);

}  // namespace nvfp4
