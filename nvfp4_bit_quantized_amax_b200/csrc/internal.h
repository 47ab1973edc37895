// internal.h -- launchers shared between the C ABI (capi.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace nvfp4 {

// Sign flips of the 16 rotation inputs, as constants the kernels read from their
// parameters: pair[i] flips both bf16 of a packed word (0x80008000 or 0), lo[i] is
// the same flip for the low value once shifted into an fp32 (0x80000000 or 0).
struct RhtFlips {
    uint32_t pair[16];
    uint32_t lo[16];
};
inline void rht_flips(uint32_t sign_mask, RhtFlips& f) {
    for (int i = 0; i < 16; ++i) {
        const bool neg = (sign_mask >> i) & 1u;
        f.pair[i] = neg ? 0x80008000u : 0u;
        f.lo[i] = neg ? 0x80000000u : 0u;
    }
}

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
    int row_rht;         // rotate the row orientation too (tile kernel, ungrouped, 1x16)
    uint32_t sign_mask;  // bit i set: rotation sign i is -1
    RhtFlips flips;      // the same signs as flip constants (filled by the launchers)
    uint32_t rk[20];     // Philox4x32-10 round keys of `seed` (filled by the launchers)
    // Grouped tensors (mixture of experts): row r belongs to group
    // row_group[r / 128] (table) or r / group_rows_uniform; group g owns rows
    // [row0_g, row0_g + rows_g) and has its own amax words (amax_words + 2g), tensor
    // scales (row_g[g], col_g[g]), Philox key seed + g, and element indices counted
    // inside its rows.  Groups are whole 128-row blocks.
    const int32_t* row_group;
    const int64_t* group_row0;
    const int64_t* group_nrows;
    int64_t group_rows_uniform;
    // Gathered input (nullable): row r of the quantized tensor is row row_src[r] of
    // x, which has src_rows rows; a negative entry reads as a zero row, one past the
    // source records kStatusIndex and also reads as zeros.
    const int32_t* row_src;
    int64_t src_rows;
};

// Rows one launch of the quantize tile kernel covers: 64-row tiles along the
// grid's y extent (at most 65535).  The entry points refuse larger tensors as a
// shape error.
constexpr int64_t kMaxTileRows = 65535ll * 64;

cudaError_t launch_amax_grouped(const QuantParams& p, int sm_count, cudaStream_t st);

// Group tables of a grouped tensor from its group sizes (host array of E <=
// kMaxGroups entries, multiples of 128): group of every 128-row block, first row
// and rows of every group, and (when pair_row0 is not null) the 256-row tiles of
// every group in order (first row, group, rows inside the group), written on `st`.
constexpr int kMaxGroups = 1024;
cudaError_t launch_group_tables(const int64_t* group_rows, int E, int32_t* block_group, int64_t* row0,
                                int64_t* nrows, cudaStream_t st, int64_t* pair_row0 = nullptr,
                                int32_t* pair_group = nullptr, int32_t* pair_rows = nullptr);

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
                        uint32_t sign_mask, uint32_t* words, int sm_count, cudaStream_t st,
                        bool row_rht = false, int* status = nullptr);
cudaError_t launch_quant_rows(const QuantParams& p, int sm_count, cudaStream_t st);
cudaError_t launch_quant_tile(const QuantParams& p, bool two_d, int sm_count, cudaStream_t st);
cudaError_t launch_sf_pad(uint8_t* sf, int64_t rows, int64_t nb, int sm_count, cudaStream_t st);
cudaError_t launch_mx_quant_rows(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* packed,
                                 uint8_t* sf, int sm_count, cudaStream_t st);
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
    // Grouped problems (mixture of experts), one launch for all groups:
    //  group_mode 1: A rows are grouped in 128-row tiles (mtile_group[m / 128] is the
    //    group of A row m); a tile of group g reads B rows g * b_group_rows + n.
    //  group_mode 2: group g reduces over k in [k_start[g], k_start[g] + k_len[g]) of
    //    A and B (both multiples of 128) and writes D rows g * M + m.
    //  scale_a / scale_b then hold one tensor scale per group; no fp32 output.
    //  In mode 1 a tile of group g also starts its reduction over B at column
    //  g * b_group_k, and B's rows are Kb wide (0: K).
    int group_mode;
    const int32_t* mtile_group;
    int64_t b_group_rows;
    int64_t b_group_k;
    int64_t Kb;
    const int64_t* k_start;
    const int64_t* k_len;
    int num_groups;
    // Mode 1 on the two-SM kernel: the 256-row tiles of every group (first row,
    // group, rows that belong to the group: 128 or 256), num_pair_tiles entries.
    const int64_t* pair_row0;
    const int32_t* pair_group;
    const int32_t* pair_rows;
    int64_t num_pair_tiles;
    int mx;  // MXFP4 operands: UE8M0 scales over 32-element blocks, no tensor scales
    // Ungrouped two-SM problems: tile order and band width (filled by the launcher).
    int tile_order;
    int64_t tile_band;
    // Clock cycles a pipeline wait may last before the kernel gives up and records
    // NVFP4_ERR_TIMEOUT (0: the default, 2^31, about a second).
    long long wait_cycles;
};
cudaError_t launch_gemm(const GemmParams& p, int sm_count, cudaStream_t st);

}  // namespace nvfp4
