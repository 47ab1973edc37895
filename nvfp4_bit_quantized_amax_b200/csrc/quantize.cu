// quantize.cu -- memory-bound kernels of the NVFP4 training path on sm_100a:
//   * amax prepass (tensor max |x|, and max |RHT(x)| of the column orientation)
//   * fused quantize: one read of a bf16 tile, row and/or column orientation,
//     1x16 or 16x16 blocks, RNE or Philox stochastic rounding, optional 16-point
//     random Hadamard transform in front of the column orientation
//   * standalone RHT, and the zero fill of the scale padding.
//
// Method: two-level NVFP4 scaling ("Nemotron NVFP4" explainer, "What NVFP4
// actually is"); 16x16 weight blocks, RHT on the wgrad inputs, SR on gradients
// ("NVIDIA's 4-bit floating point pushes AI training limits", artiverse.ca).
#include <cuda_bf16.h>

#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace nvfp4 {

// ============================================================================
// 16-point Hadamard butterfly in fp64.  The Sylvester H16 is symmetric, so
// x . diag(s) . H16 == H16 . (s * x); four radix-2 stages compute it.  Inputs
// are bf16 values (8 significant bits), so every partial sum is exact while the
// chunk's exponents span at most 41 binades; the fp32 rounding of the result is
// then the correctly rounded value of the exact sum.
// ============================================================================
__device__ __forceinline__ void fwht16(double (&y)[16]) {
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if ((i & h) == 0) {
                const double a = y[i], b = y[i + h];
                y[i] = a + b;
                y[i + h] = a - b;
            }
        }
    }
}

// 16-point rotation of a row chunk held by a lane pair (even lane: elements 0-7,
// odd lane: 8-15; both lanes of every pair call this together): three butterfly
// stages inside the lane, the last across the pair.  In fp64, exact like fwht16;
// y receives the lane's eight outputs.
__device__ __forceinline__ void rht16_lane_pair(const uint4& w, uint32_t sign_mask, int lane,
                                                double (&y)[8]) {
    const int base = (lane & 1) * 8;
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint32_t b = (k & 1) ? (ws[k >> 1] >> 16) : (ws[k >> 1] & 0xFFFFu);
        y[k] = (double)__uint_as_float((b ^ (((sign_mask >> (base + k)) & 1u) << 15)) << 16);
    }
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if ((k & h) == 0) {
                const double a = y[k], b = y[k + h];
                y[k] = a + b;
                y[k + h] = a - b;
            }
        }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const double o = __shfl_xor_sync(0xFFFFFFFFu, y[k], 1);
        y[k] = (lane & 1) ? o - y[k] : y[k] + o;
    }
}

// bf16 bit pattern with its sign flipped where the rotation sign is -1.
__device__ __forceinline__ double bf16_signed_to_f64(uint32_t bits16, uint32_t flip) {
    return (double)__uint_as_float((bits16 ^ (flip << 15)) << 16);
}

// ============================================================================
// amax prepass.  One warp handles a 16-row x 256-column unit, each lane 16 rows
// x 8 columns (sixteen 16-byte loads).  Word 0 receives max |x| (fp32 bits of a
// bf16 magnitude; NaN patterns sort above Inf), word 1 max |RHT16 down the
// rows| (column orientation), as fp32 bits.  Both are combined with atomicMax.
// ============================================================================
// Grouped (kGrouped): the rows of a unit lie in one group, whose words are
// words[2g] and words[2g+1]; each unit is folded into them by the warp.
// kRowRht: word 0 (or 2g) is max |RHT16 along the rows| instead of max |x| (the
// row orientation is rotated); a non-finite input still makes it non-finite.
template <bool kColRht, bool kGrouped, bool kRowRht>
__global__ void __launch_bounds__(256) amax_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                   int64_t cols, uint32_t sign_mask,
                                                   uint32_t* __restrict__ words,
                                                   const int32_t* __restrict__ row_group,
                                                   int64_t group_rows_uniform) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t col_units = (cols + 255) >> 8;
    const int64_t units = ((rows + 15) >> 4) * col_units;
    uint32_t m_row = 0;   // two packed 16-bit magnitudes
    double m_col = 0.0;
    double m_rrht = 0.0;  // kRowRht: max |rotated row|
    for (int64_t u = (int64_t)blockIdx.x * 8 + warp; u < units; u += (int64_t)gridDim.x * 8) {
        const int64_t r0 = (u / col_units) * 16;
        const int64_t c0 = (u % col_units) * 256 + lane * 8;
        if (kGrouped) {
            m_row = 0;
            m_col = 0.0;
        }
        if (kRowRht || c0 < cols) {
        uint4 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            v[i] = (c0 < cols && r0 + i < rows) ? ld_stream_v4(x + (r0 + i) * cols + c0)
                                                : make_uint4(0, 0, 0, 0);
        if (kRowRht) {  // every lane takes part (zeros past the columns)
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                double y[8];
                rht16_lane_pair(v[i], sign_mask, lane, y);
#pragma unroll
                for (int k = 0; k < 8; ++k) m_rrht = fmax(m_rrht, fabs(y[k]));
            }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            m_row = __vmaxu2(m_row, v[i].x & 0x7FFF7FFFu);
            m_row = __vmaxu2(m_row, v[i].y & 0x7FFF7FFFu);
            m_row = __vmaxu2(m_row, v[i].z & 0x7FFF7FFFu);
            m_row = __vmaxu2(m_row, v[i].w & 0x7FFF7FFFu);
        }
        if (kColRht) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                double y[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint32_t w = (c >> 1) == 0 ? v[i].x : (c >> 1) == 1 ? v[i].y
                                     : (c >> 1) == 2 ? v[i].z : v[i].w;
                    const uint32_t b = (c & 1) ? (w >> 16) : (w & 0xFFFFu);
                    y[i] = bf16_signed_to_f64(b, (sign_mask >> i) & 1u);
                }
                fwht16(y);
#pragma unroll
                for (int i = 0; i < 16; ++i) m_col = fmax(m_col, fabs(y[i]));
            }
        }
        }
        if (kGrouped) {
            const int64_t g = row_group ? (int64_t)row_group[r0 >> 7] : r0 / group_rows_uniform;
            uint32_t ur = max(m_row & 0xFFFFu, m_row >> 16) << 16;
            uint32_t uc = kColRht ? __float_as_uint(__double2float_rn(m_col)) : 0u;
            ur = __reduce_max_sync(0xFFFFFFFFu, ur);
            uc = __reduce_max_sync(0xFFFFFFFFu, uc);
            if (lane == 0) {
                if (ur) atomicMax(words + 2 * g, ur);
                if (kColRht && uc) atomicMax(words + 2 * g + 1, uc);
            }
        }
    }
    if (kGrouped) return;
    uint32_t a_row = max(m_row & 0xFFFFu, m_row >> 16) << 16;
    if (kRowRht && a_row < 0x7F800000u) a_row = __float_as_uint(__double2float_rn(m_rrht));
    uint32_t a_col = kColRht ? __float_as_uint(__double2float_rn(m_col)) : 0u;
    a_row = __reduce_max_sync(0xFFFFFFFFu, a_row);
    a_col = __reduce_max_sync(0xFFFFFFFFu, a_col);
    __shared__ uint32_t red[2][8];
    if (lane == 0) {
        red[0][warp] = a_row;
        red[1][warp] = a_col;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t r = 0, c = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            r = max(r, red[0][w]);
            c = max(c, red[1][w]);
        }
        if (r) atomicMax(words + 0, r);
        if (kColRht && c) atomicMax(words + 1, c);
    }
}

// ============================================================================
// Shared helpers of the quantize kernels.
// ============================================================================
__device__ __forceinline__ bool finite_bits(uint32_t b) { return (b & 0x7FFFFFFFu) < 0x7F800000u; }

// Eight values -> packed codes with RNE or SR (element index e0 .. e0+7 of the
// quantized tensor, e0 % 8 == 0); element i lands in bits [4i, 4i+4).
__device__ __forceinline__ uint32_t encode8(const float (&v)[8], float inv, bool sr,
                                            const uint32_t (&rk)[20], uint32_t stream,
                                            uint64_t e0) {
    if (!sr) {
        float q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(v[i], inv);
        return e2m1x8_rn(q);
    }
    float q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(v[i], inv);
    return sr_e2m1x8(q, sr_draws8(rk, stream, e0 >> 3));
}

__device__ __forceinline__ void unpack8(const uint4& w, float (&v)[8]) {
    v[0] = bf16_lo(w.x); v[1] = bf16_hi(w.x);
    v[2] = bf16_lo(w.y); v[3] = bf16_hi(w.y);
    v[4] = bf16_lo(w.z); v[5] = bf16_hi(w.z);
    v[6] = bf16_lo(w.w); v[7] = bf16_hi(w.w);
}

__device__ __forceinline__ float absmax8(const uint4& w) {
    uint32_t m = __vmaxu2(__vmaxu2(w.x & 0x7FFF7FFFu, w.y & 0x7FFF7FFFu),
                          __vmaxu2(w.z & 0x7FFF7FFFu, w.w & 0x7FFF7FFFu));
    return __uint_as_float(max(m & 0xFFFFu, m >> 16) << 16);
}

// Reads the tensor amax words; false (and the error recorded) if non-finite.
__device__ __forceinline__ bool load_tensor_scales(const QuantParams& p, TensorScale& tr,
                                                   TensorScale& tc) {
    const uint32_t wr = p.amax_words[0];
    const uint32_t wc = p.col_rht ? p.amax_words[1] : wr;
    const bool ok = finite_bits(wr) && finite_bits(wc);
    const bool first = blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0;
    if (!ok) {
        if (first) {
            set_status(p.status, kStatusNonFinite);
            if (p.row_g) *p.row_g = __uint_as_float(0x7FC00000u);
            if (p.col_g) *p.col_g = __uint_as_float(0x7FC00000u);
        }
        return false;
    }
    tr = tensor_scale_from_amax(__uint_as_float(wr));
    tc = tensor_scale_from_amax(__uint_as_float(wc));
    if (first) {
        if (p.row_g) *p.row_g = tr.g;
        if (p.col_g) *p.col_g = tc.g;
    }
    return true;
}

// ============================================================================
// Row orientation only, 1x16 blocks: every lane owns 8 consecutive elements
// (one 16-byte load); a block is a lane pair.  Grid-stride over 8-chunks.
// ============================================================================
__global__ void __launch_bounds__(256) quant_rows_kernel(QuantParams p) {
    TensorScale tr, tc;
    if (!load_tensor_scales(p, tr, tc)) return;
    const int64_t cpr = p.cols >> 3;  // 8-chunks per row (even)
    const int64_t nchunks = p.rows * cpr;
    const int64_t katoms = (p.cols / 16 + 3) >> 2;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    // warp-uniform trip count: every lane takes part in the pair shuffle
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); base < nchunks;
         base += stride) {
        const int64_t q = base + (threadIdx.x & 31);
        const bool valid = q < nchunks;
        const uint4 w = valid ? ld_stream_v4(p.x + q * 8) : make_uint4(0, 0, 0, 0);
        float amax = absmax8(w);
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
        uint32_t s;
        float inv;
        block_scale(amax, tr, s, inv);
        float v[8];
        unpack8(w, v);
        const uint32_t codes = encode8(v, inv, p.row_sr, p.rk, 0u, (uint64_t)q * 8);
        if (valid) {
            reinterpret_cast<uint32_t*>(p.row_data)[q] = codes;
            if ((q & 1) == 0) {
                const int64_t r = q / cpr, kb = (q % cpr) >> 1;
                p.row_sf[sf_offset(r, kb, katoms)] = (uint8_t)s;
            }
        }
    }
}

// ============================================================================
// Tile kernel: a CTA loads a 64 x 128 bf16 tile once (registers + shared
// memory) and writes the row orientation (from registers, lane pairs) and/or
// the column orientation (from shared memory, one lane per column, two
// 16-row chunks per lane).  k2D: 16x16 blocks, the tile scale is found by the
// column pass and shared by both orientations.  kRht: 16-point RHT in fp64
// down each column chunk before the column orientation is quantized.
// ============================================================================
constexpr int kTR = 64, kTC = 128, kPitch = kTC + 8;

// Grouped (kGrouped): the tile's rows lie in one group g (see QuantParams), which
// supplies the tensor scales, the Philox key seed + g and the origin of the
// element indices.
// kRowRht: the row orientation is rotated too (16-point RHT along each row block,
// the block's lane pair exchanging halves), e.g. dgrad operands under the Mosaic
// recipe.
// Resident CTAs per SM that the register budget is sized for.  A CTA loads its
// tile once and then only computes and stores, so more resident CTAs keep more
// loads in flight; the grouped RHT variant keeps three (at four it spills).
template <bool k2D, bool kRht, bool kGrouped>
constexpr int quant_tile_min_blocks() {
    return (kGrouped && kRht) ? 3 : 4;
}

template <bool k2D, bool kRht, bool kGrouped, bool kRowRht>
__global__ void __launch_bounds__(256, (quant_tile_min_blocks<k2D, kRht, kGrouped>()))
    quant_tile_kernel(QuantParams p) {
    __shared__ __align__(16) uint16_t tile[kTR][kPitch];
    __shared__ uint32_t tile_s[kTR / 16][kTC / 16];
    __shared__ float tile_inv[kTR / 16][kTC / 16];
    // The tile's scales, staged so that they leave in wide stores instead of one
    // byte each: the column orientation's 128 columns x 4 blocks are exactly one
    // 512-byte atom; the row orientation's 64 rows x 8 blocks are 8 bytes of each
    // of the 32 lines of two atoms.  Entries past the tensor hold 0 (the padding).
    __shared__ __align__(16) uint8_t col_atom[512];
    __shared__ __align__(16) uint8_t row_half_atoms[2][32][8];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t r0 = (int64_t)blockIdx.y * kTR, c0 = (int64_t)blockIdx.x * kTC;
    TensorScale tr, tc;
    int64_t g_row0 = 0, g_rows = p.rows;  // the rows the element indices count in
    uint32_t rkg[20];                     // the group's Philox round keys
    if (kGrouped) {
        const int64_t g = p.row_group ? (int64_t)p.row_group[r0 >> 7] : r0 / p.group_rows_uniform;
        g_row0 = p.row_group ? p.group_row0[g] : g * p.group_rows_uniform;
        g_rows = p.row_group ? p.group_nrows[g] : p.group_rows_uniform;
        const uint32_t wr = p.amax_words[2 * g];
        const uint32_t wc = p.col_rht ? p.amax_words[2 * g + 1] : wr;
        const bool first = r0 == g_row0 && c0 == 0 && tid == 0;
        if (!finite_bits(wr) || !finite_bits(wc)) {
            if (first) {
                set_status(p.status, kStatusNonFinite);
                if (p.row_g) p.row_g[g] = __uint_as_float(0x7FC00000u);
                if (p.col_g) p.col_g[g] = __uint_as_float(0x7FC00000u);
            }
            return;
        }
        tr = tensor_scale_from_amax(__uint_as_float(wr));
        tc = tensor_scale_from_amax(__uint_as_float(wc));
        if (first) {
            if (p.row_g) p.row_g[g] = tr.g;
            if (p.col_g) p.col_g[g] = tc.g;
        }
        uint32_t k0 = (uint32_t)(p.seed + (uint64_t)g), k1 = (uint32_t)((p.seed + (uint64_t)g) >> 32);
#pragma unroll
        for (int r = 0; r < 10; ++r) {
            rkg[2 * r] = k0;
            rkg[2 * r + 1] = k1;
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
    } else {
        if (!load_tensor_scales(p, tr, tc)) return;
    }
    const uint32_t (&rk)[20] = kGrouped ? rkg : p.rk;
    const bool want_row = p.row_data != nullptr;
    const bool want_col = p.col_data != nullptr;
    const bool use_smem = want_col || k2D;

    // ---- load: chunk q = k*256 + tid covers row q/16, columns (q%16)*8 .. +7
    uint4 reg[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int q = k * 256 + tid;
        const int lr = q >> 4, lc = (q & 15) * 8;
        const int64_t r = r0 + lr, c = c0 + lc;
        reg[k] = (r < p.rows && c < p.cols) ? ld_stream_v4(p.x + r * p.cols + c)
                                            : make_uint4(0, 0, 0, 0);
        if (use_smem) *reinterpret_cast<uint4*>(&tile[lr][lc]) = reg[k];
    }
    if (use_smem) __syncthreads();

    // ---- column pass: lane -> column lc, chunks j0, j0+1 (16 rows each)
    if (use_smem) {
        const int lc = 32 * (warp & 3) + lane;
        const int j0 = 2 * (warp >> 2);
        const int64_t c = c0 + lc;
        uint32_t out[4];
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            const int j = j0 + jj;
            float y[16];
            if (kRht) {
                double d[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    d[i] = bf16_signed_to_f64(tile[16 * j + i][lc], (p.sign_mask >> i) & 1u);
                fwht16(d);
#pragma unroll
                for (int i = 0; i < 16; ++i) y[i] = __double2float_rn(d[i]);
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) y[i] = __uint_as_float((uint32_t)tile[16 * j + i][lc] << 16);
            }
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(y[i]));
            uint32_t s;
            float inv;
            if (k2D) {
                // 16x16 tile: 16 lanes hold its 16 columns
#pragma unroll
                for (int o = 8; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
                block_scale(amax, tc, s, inv);
                if ((lane & 15) == 0) {
                    tile_s[j][lc >> 4] = s;
                    tile_inv[j][lc >> 4] = inv;
                }
            } else {
                block_scale(amax, tc, s, inv);
            }
            if (want_col) {
                const uint64_t e0 = (uint64_t)c * (uint64_t)g_rows + (uint64_t)(r0 - g_row0 + 16 * j);
                float lo8[8], hi8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    lo8[i] = y[i];
                    hi8[i] = y[8 + i];
                }
                out[2 * jj] = encode8(lo8, inv, p.col_sr, rk, 1u, e0);
                out[2 * jj + 1] = encode8(hi8, inv, p.col_sr, rk, 1u, e0 + 8);
                // atom byte of (column lc, block j): line lc % 32, group lc / 32
                col_atom[lane * 16 + (warp & 3) * 4 + j] =
                    (c < p.cols && r0 + 16 * j < p.rows) ? (uint8_t)s : (uint8_t)0;
            }
        }
        if (want_col && c < p.cols) {
            uint8_t* base = p.col_data + c * (p.rows >> 1) + ((r0 + 16 * j0) >> 1);
            const bool both = r0 + 16 * (j0 + 1) < p.rows;
            if (both && (reinterpret_cast<uintptr_t>(base) & 15u) == 0) {
                *reinterpret_cast<uint4*>(base) = make_uint4(out[0], out[1], out[2], out[3]);
            } else {
                if (r0 + 16 * j0 < p.rows) *reinterpret_cast<uint2*>(base) = make_uint2(out[0], out[1]);
                if (both) *reinterpret_cast<uint2*>(base + 8) = make_uint2(out[2], out[3]);
            }
        }
        if (k2D) __syncthreads();
    }

    // ---- row pass from registers: a 16-block is a lane pair
    if (want_row) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int q = k * 256 + tid;
            const int lr = q >> 4, lc = (q & 15) * 8;
            const int64_t r = r0 + lr, c = c0 + lc;
            uint32_t s;
            float inv;
            float v[8];
            if (kRowRht) {
                double y[8];
                rht16_lane_pair(reg[k], p.sign_mask, lane, y);
                float amax = 0.0f;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    v[i] = __double2float_rn(y[i]);
                    amax = fmaxf(amax, fabsf(v[i]));
                }
                amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
                block_scale(amax, tr, s, inv);
            } else if (k2D) {
                s = tile_s[lr >> 4][lc >> 4];
                inv = tile_inv[lr >> 4][lc >> 4];
                unpack8(reg[k], v);
            } else {
                float amax = absmax8(reg[k]);
                amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
                block_scale(amax, tr, s, inv);
                unpack8(reg[k], v);
            }
            const uint32_t codes =
                encode8(v, inv, p.row_sr, rk, 0u, (uint64_t)(r - g_row0) * (uint64_t)p.cols + (uint64_t)c);
            const bool inside = r < p.rows && c < p.cols;
            if (inside) *reinterpret_cast<uint32_t*>(p.row_data + r * (p.cols >> 1) + (c >> 1)) = codes;
            // (row lr, block lc / 16): half-atom lc / 64, line lr % 32, byte 4 * (lr / 32) + block % 4
            if ((lc & 15) == 0)
                row_half_atoms[lc >> 6][lr & 31][(lr >> 5) * 4 + ((lc >> 4) & 3)] = inside ? (uint8_t)s : (uint8_t)0;
        }
    }

    // ---- scale stores.  Every entry written lies inside the scale buffer: the
    // column atom is (128-column group c0 / 128, blocks r0 / 16 .. + 3) with r0 a
    // multiple of 64 below the rows; the row half-atoms cover 64 rows below
    // pad128(rows), and the second is skipped when its blocks start past the
    // padded block count.
    __syncthreads();
    if (want_col && warp == 0) {
        const int64_t katoms_c = (p.rows / 16 + 3) >> 2;
        const int64_t atom = (c0 >> 7) * katoms_c + (r0 >> 6);
        *reinterpret_cast<uint4*>(p.col_sf + atom * 512 + lane * 16) =
            *reinterpret_cast<const uint4*>(col_atom + lane * 16);
    }
    if (want_row && (warp == 2 || warp == 3)) {
        const int64_t katoms_r = (p.cols / 16 + 3) >> 2;
        const int a = warp - 2;
        if ((c0 >> 6) + a < katoms_r) {
            const int64_t atom = (r0 >> 7) * katoms_r + (c0 >> 6) + a;
            *reinterpret_cast<uint2*>(p.row_sf + atom * 512 + lane * 16 + ((r0 & 127) >> 5) * 4) =
                *reinterpret_cast<const uint2*>(row_half_atoms[a][lane]);
        }
    }
}

// ============================================================================
// MXFP4 (the comparison format): row orientation, E8M0 scale per 32 elements,
// round-to-nearest-even, one pass (no tensor scale, so no amax prepass).  Every
// lane owns 8 consecutive elements; a 32-block is a lane quad.  The scale is the
// smallest power of two 2^k with amax <= 6 * 2^k: for amax = (1 + f) * 2^E, k =
// E - 2 if f <= 1/2 else E - 1, code e = k + 127 (0 for a zero or subnormal
// amax, 255 when the block holds Inf / NaN); elements are x * 2^-k, exact.
// ============================================================================
__global__ void __launch_bounds__(256) mx_quant_rows_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                            int64_t cols, uint8_t* __restrict__ packed,
                                                            uint8_t* __restrict__ sf) {
    const int64_t cpr = cols >> 3;  // 8-chunks per row (a multiple of 4)
    const int64_t nchunks = rows * cpr;
    const int64_t katoms = (cols / 32 + 3) >> 2;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); base < nchunks;
         base += stride) {
        const int64_t q = base + (threadIdx.x & 31);
        const bool valid = q < nchunks;
        const uint4 w = valid ? ld_stream_v4(x + q * 8) : make_uint4(0, 0, 0, 0);
        float amax = absmax8(w);
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
        const uint32_t ab = __float_as_uint(amax);
        uint32_t e;
        if (ab >= 0x7F800000u)
            e = 255u;
        else if ((ab >> 23) == 0u)
            e = 0u;
        else
            e = (ab >> 23) - 2u + ((ab & 0x7FFFFFu) > 0x400000u ? 1u : 0u);
        // 2^-k = 2^(127 - e) (e <= 253 for finite bf16 input, so this is a normal float)
        const float mult = e == 255u ? __uint_as_float(0x7FC00000u) : __uint_as_float((254u - e) << 23);
        float v[8];
        unpack8(w, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], mult);
        const uint32_t codes = e2m1x8_rn(v);
        if (valid) {
            reinterpret_cast<uint32_t*>(packed)[q] = codes;
            if ((q & 3) == 0) {
                const int64_t r = q / cpr, kb = (q % cpr) >> 2;
                sf[sf_offset(r, kb, katoms)] = (uint8_t)e;
            }
        }
    }
}

static int grid_for(int64_t work_items, int per_block, int sm_count, int blocks_per_sm);

cudaError_t launch_mx_quant_rows(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* packed,
                                 uint8_t* sf, int sm_count, cudaStream_t st) {
    const int64_t nchunks = rows * (cols / 8);
    const int grid = grid_for(nchunks, 256, sm_count, 8);
    mx_quant_rows_kernel<<<grid, 256, 0, st>>>(x, rows, cols, packed, sf);
    return cudaGetLastError();
}

// ============================================================================
// Zero fill of the scale padding: rows [rows, pad128(rows)) and 16-blocks
// [nb, pad4(nb)) of an operand with `rows` rows and `nb` 16-blocks per row.
// ============================================================================
__global__ void sf_pad_kernel(uint8_t* __restrict__ sf, int64_t rows, int64_t nb) {
    const int64_t prow = (rows + 127) / 128 * 128, pnb = (nb + 3) / 4 * 4;
    const int64_t katoms = pnb / 4;
    const int64_t total = prow * pnb;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / pnb, kb = i % pnb;
        if (r >= rows || kb >= nb) sf[sf_offset(r, kb, katoms)] = 0;
    }
}

// ============================================================================
// Standalone RHT.  axis 1: a thread transforms 16 contiguous elements.
// axis 0: a thread transforms 8 columns x 16 rows (like the amax unit).
// ============================================================================
__global__ void __launch_bounds__(256) rht_axis1_kernel(const uint16_t* __restrict__ x, float* __restrict__ y,
                                                       int64_t nchunks, uint32_t sign_mask) {
    for (int64_t ch = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; ch < nchunks;
         ch += (int64_t)gridDim.x * blockDim.x) {
        const uint4 a = ld_stream_v4(x + ch * 16), b = ld_stream_v4(x + ch * 16 + 8);
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        double d[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            d[i] = bf16_signed_to_f64((i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xFFFFu),
                                      (sign_mask >> i) & 1u);
        fwht16(d);
        float4* out = reinterpret_cast<float4*>(y + ch * 16);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            out[i] = make_float4(__double2float_rn(d[4 * i]), __double2float_rn(d[4 * i + 1]),
                                 __double2float_rn(d[4 * i + 2]), __double2float_rn(d[4 * i + 3]));
    }
}

__global__ void __launch_bounds__(256) rht_axis0_kernel(const uint16_t* __restrict__ x, float* __restrict__ y,
                                                       int64_t rows, int64_t cols, uint32_t sign_mask) {
    const int64_t cunits = cols / 8;
    const int64_t units = (rows / 16) * cunits;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < units;
         u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r0 = (u / cunits) * 16, c0 = (u % cunits) * 8;
        uint4 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = ld_stream_v4(x + (r0 + i) * cols + c0);
#pragma unroll
        for (int half = 0; half < 2; ++half) {  // columns 4*half .. 4*half+3
            float o[16][4];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const int c = 4 * half + cc;
                double d[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint32_t w = (c >> 1) == 0 ? v[i].x : (c >> 1) == 1 ? v[i].y
                                     : (c >> 1) == 2 ? v[i].z : v[i].w;
                    d[i] = bf16_signed_to_f64((c & 1) ? (w >> 16) : (w & 0xFFFFu), (sign_mask >> i) & 1u);
                }
                fwht16(d);
#pragma unroll
                for (int i = 0; i < 16; ++i) o[i][cc] = __double2float_rn(d[i]);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i)
                *reinterpret_cast<float4*>(y + (r0 + i) * cols + c0 + 4 * half) =
                    make_float4(o[i][0], o[i][1], o[i][2], o[i][3]);
        }
    }
}

// ============================================================================
// Launchers
// ============================================================================
static int grid_for(int64_t work_items, int per_block, int sm_count, int blocks_per_sm) {
    int64_t g = (work_items + per_block - 1) / per_block;
    const int64_t cap = (int64_t)sm_count * blocks_per_sm;
    if (g > cap) g = cap;
    if (g < 1) g = 1;
    return (int)g;
}

cudaError_t launch_amax(const uint16_t* x, int64_t rows, int64_t cols, bool col_rht,
                        uint32_t sign_mask, uint32_t* words, int sm_count, cudaStream_t st,
                        bool row_rht) {
    const int64_t units = ((rows + 15) / 16) * ((cols + 255) / 256);
    const int grid = grid_for(units, 8, sm_count, 8);
    if (row_rht && col_rht)
        amax_kernel<true, false, true><<<grid, 256, 0, st>>>(x, rows, cols, sign_mask, words, nullptr, 0);
    else if (row_rht)
        amax_kernel<false, false, true><<<grid, 256, 0, st>>>(x, rows, cols, sign_mask, words, nullptr, 0);
    else if (col_rht)
        amax_kernel<true, false, false><<<grid, 256, 0, st>>>(x, rows, cols, sign_mask, words, nullptr, 0);
    else
        amax_kernel<false, false, false><<<grid, 256, 0, st>>>(x, rows, cols, sign_mask, words, nullptr, 0);
    return cudaGetLastError();
}

cudaError_t launch_amax_grouped(const QuantParams& p, int sm_count, cudaStream_t st) {
    const int64_t units = ((p.rows + 15) >> 4) * ((p.cols + 255) >> 8);
    const int grid = grid_for(units, 8, sm_count, 8);
    uint32_t* words = const_cast<uint32_t*>(p.amax_words);
    if (p.col_rht)
        amax_kernel<true, true, false><<<grid, 256, 0, st>>>(p.x, p.rows, p.cols, p.sign_mask, words, p.row_group,
                                                     p.group_rows_uniform);
    else
        amax_kernel<false, true, false><<<grid, 256, 0, st>>>(p.x, p.rows, p.cols, p.sign_mask, words, p.row_group,
                                                      p.group_rows_uniform);
    return cudaGetLastError();
}

// ============================================================================
// Group tables of a grouped tensor, built on the device from the group sizes
// (carried in the kernel's parameters): the group of every 128-row block, and
// each group's first row and row count.
// ============================================================================
struct GroupSizes {
    int64_t rows[kMaxGroups];
};
__global__ void group_tables_kernel(GroupSizes gs, int E, int32_t* __restrict__ block_group,
                                    int64_t* __restrict__ row0, int64_t* __restrict__ nrows) {
    __shared__ int64_t start[kMaxGroups + 1];
    if (threadIdx.x == 0) {
        int64_t r = 0;
        for (int e = 0; e < E; ++e) {
            start[e] = r;
            r += gs.rows[e];
        }
        start[E] = r;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        row0[e] = start[e];
        nrows[e] = gs.rows[e];
    }
    const int64_t blocks = start[E] / 128;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < blocks;
         b += (int64_t)gridDim.x * blockDim.x) {
        int lo = 0, hi = E - 1;  // last group whose start is <= the block's first row
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (start[mid] <= b * 128) lo = mid; else hi = mid - 1;
        }
        while (lo < E - 1 && start[lo + 1] <= b * 128) ++lo;
        block_group[b] = lo;
    }
}

cudaError_t launch_group_tables(const int64_t* group_rows, int E, int32_t* block_group, int64_t* row0,
                                int64_t* nrows, cudaStream_t st) {
    if (E < 1 || E > kMaxGroups) return cudaErrorInvalidValue;
    GroupSizes gs;
    memset(&gs, 0, sizeof gs);
    int64_t total = 0;
    for (int e = 0; e < E; ++e) {
        gs.rows[e] = group_rows[e];
        total += group_rows[e];
    }
    const int64_t blocks = total / 128;
    const int grid = (int)((blocks + 255) / 256 < 64 ? (blocks + 255) / 256 : 64);
    group_tables_kernel<<<grid > 0 ? grid : 1, 256, 0, st>>>(gs, E, block_group, row0, nrows);
    return cudaGetLastError();
}

cudaError_t launch_quant_rows(const QuantParams& params, int sm_count, cudaStream_t st) {
    QuantParams p = params;
    philox_round_keys(p.seed, p.rk);
    const int64_t nchunks = p.rows * (p.cols / 8);
    const int grid = grid_for(nchunks, 256, sm_count, 8);
    quant_rows_kernel<<<grid, 256, 0, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_quant_tile(const QuantParams& params, bool two_d, cudaStream_t st) {
    QuantParams p = params;
    philox_round_keys(p.seed, p.rk);
    const dim3 grid((unsigned)((p.cols + kTC - 1) / kTC), (unsigned)((p.rows + kTR - 1) / kTR));
    const bool grouped = p.row_group != nullptr || p.group_rows_uniform > 0;
    if (p.row_rht && (grouped || two_d)) return cudaErrorInvalidValue;
    const bool col_rht = p.col_rht && p.col_data;
    if (grouped) {
        if (two_d)
            quant_tile_kernel<true, false, true, false><<<grid, 256, 0, st>>>(p);
        else if (col_rht)
            quant_tile_kernel<false, true, true, false><<<grid, 256, 0, st>>>(p);
        else
            quant_tile_kernel<false, false, true, false><<<grid, 256, 0, st>>>(p);
    } else if (two_d)
        quant_tile_kernel<true, false, false, false><<<grid, 256, 0, st>>>(p);
    else if (p.row_rht && col_rht)
        quant_tile_kernel<false, true, false, true><<<grid, 256, 0, st>>>(p);
    else if (p.row_rht)
        quant_tile_kernel<false, false, false, true><<<grid, 256, 0, st>>>(p);
    else if (col_rht)
        quant_tile_kernel<false, true, false, false><<<grid, 256, 0, st>>>(p);
    else
        quant_tile_kernel<false, false, false, false><<<grid, 256, 0, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_sf_pad(uint8_t* sf, int64_t rows, int64_t nb, int sm_count, cudaStream_t st) {
    if (rows % 128 == 0 && nb % 4 == 0) return cudaSuccess;
    const int64_t total = (rows + 127) / 128 * 128 * ((nb + 3) / 4 * 4);
    sf_pad_kernel<<<grid_for(total, 256, sm_count, 4), 256, 0, st>>>(sf, rows, nb);
    return cudaGetLastError();
}

cudaError_t launch_rht(const uint16_t* x, float* y, int64_t rows, int64_t cols, int axis,
                       uint32_t sign_mask, int sm_count, cudaStream_t st) {
    if (axis == 1) {
        const int64_t n = rows * cols / 16;
        rht_axis1_kernel<<<grid_for(n, 256, sm_count, 8), 256, 0, st>>>(x, y, n, sign_mask);
    } else {
        const int64_t n = (rows / 16) * (cols / 8);
        rht_axis0_kernel<<<grid_for(n, 256, sm_count, 4), 256, 0, st>>>(x, y, rows, cols, sign_mask);
    }
    return cudaGetLastError();
}

}  // namespace nvfp4

// ============================================================================
// Mixture-of-experts routing (data movement around the expert GEMMs).
// gather: dst[i] = src[idx[i]] (a row of bf16), or zeros where idx[i] < 0 (the
//         padding rows that round each expert's segment up).
// combine: out[t] = bf16( sum_j src[slot[t][j]] ) in fp32, j = 0 .. topk-1 in order.
// ============================================================================
namespace nvfp4 {

__global__ void __launch_bounds__(256) moe_gather_kernel(const uint16_t* __restrict__ src,
                                                         const int32_t* __restrict__ idx,
                                                         uint16_t* __restrict__ dst, int64_t rows,
                                                         int64_t cols) {
    const int64_t vpr = cols / 8;  // 16-byte vectors per row
    const int64_t total = rows * vpr;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / vpr, c = i % vpr;
        const int32_t s = idx[r];
        const uint4 v = s >= 0 ? ld_stream_v4(src + (int64_t)s * cols + c * 8) : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(dst + r * cols + c * 8) = v;
    }
}

__global__ void __launch_bounds__(256) moe_combine_kernel(const uint16_t* __restrict__ src,
                                                          const int32_t* __restrict__ slot,
                                                          uint16_t* __restrict__ dst, int64_t tokens,
                                                          int64_t cols, int topk) {
    const int64_t vpr = cols / 8;
    const int64_t total = tokens * vpr;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / vpr, c = i % vpr;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < topk; ++j) {
            const int32_t s = slot[t * topk + j];
            if (s < 0) continue;
            const uint4 v = ld_stream_v4(src + (int64_t)s * cols + c * 8);
            float f[8];
            f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
            f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z); f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[k] = __fadd_rn(acc[k], f[k]);
        }
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * k], acc[2 * k + 1]);
            w[k] = *reinterpret_cast<const uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(dst + t * cols + c * 8) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

cudaError_t launch_moe_gather(const uint16_t* src, const int32_t* idx, uint16_t* dst, int64_t rows,
                              int64_t cols, int sm_count, cudaStream_t st) {
    const int64_t total = rows * (cols / 8);
    moe_gather_kernel<<<grid_for(total, 256, sm_count, 8), 256, 0, st>>>(src, idx, dst, rows, cols);
    return cudaGetLastError();
}

cudaError_t launch_moe_combine(const uint16_t* src, const int32_t* slot, uint16_t* dst,
                               int64_t tokens, int64_t cols, int topk, int sm_count, cudaStream_t st) {
    const int64_t total = tokens * (cols / 8);
    moe_combine_kernel<<<grid_for(total, 256, sm_count, 8), 256, 0, st>>>(src, slot, dst, tokens, cols,
                                                                         topk);
    return cudaGetLastError();
}

}  // namespace nvfp4
