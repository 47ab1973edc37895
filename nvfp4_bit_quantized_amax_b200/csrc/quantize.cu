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
// Packed fp32 pairs (sm_100 f32x2 arithmetic): element 0 in the low word.  Every
// operation rounds to nearest even and keeps subnormals, like its scalar form.
// ============================================================================
typedef unsigned long long f32x2;

__device__ __forceinline__ f32x2 pk(float lo, float hi) {
    f32x2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ f32x2 pk_bits(uint32_t lo, uint32_t hi) {
    f32x2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}
__device__ __forceinline__ void unpk(f32x2 v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b) {
    f32x2 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f32x2 sub2(f32x2 a, f32x2 b) {
    f32x2 d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
    f32x2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// a + b rounded upward (toward +inf)
__device__ __forceinline__ f32x2 add2_ru(f32x2 a, f32x2 b) {
    f32x2 d;
    asm("add.rp.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// Two 16-bit lanes: signed minimum, unsigned maximum.
__device__ __forceinline__ uint32_t vmin_s16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("min.s16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t vmax_s16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.s16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t vmin_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("min.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Largest and smallest magnitude of bf16 values, per 16-bit lane of packed words,
// from four full-rate packed min/max (no masking per word).  A sign-magnitude
// pattern compares as unsigned by (sign, magnitude) and as signed with the negative
// magnitudes reversed, so the unsigned maximum holds the largest negative magnitude
// (or, with no negative value, the largest positive one) and the signed maximum the
// largest positive magnitude (or, with no nonnegative value, the largest negative
// one): their magnitudes' maximum is the largest magnitude.  Likewise the minima.
template <int N>
__device__ __forceinline__ void chunk_mag_stats(const uint32_t (&w)[N], uint32_t& mx, uint32_t& mn) {
    uint32_t umax = 0u, smax = 0x80008000u, umin = 0xFFFFFFFFu, smin = 0x7FFF7FFFu;
#pragma unroll
    for (int i = 0; i < N; ++i) {
        umax = vmax_u16x2(umax, w[i]);
        smax = vmax_s16x2(smax, w[i]);
        umin = vmin_u16x2(umin, w[i]);
        smin = vmin_s16x2(smin, w[i]);
    }
    mx = vmax_u16x2(umax & 0x7FFF7FFFu, smax & 0x7FFF7FFFu);
    mn = vmin_u16x2(umin & 0x7FFF7FFFu, smin & 0x7FFF7FFFu);
}

// 32-byte streaming load (16 bf16) of data read once; `p` 32-byte aligned.
__device__ __forceinline__ void ld_stream_v8(const void* p, uint32_t (&r)[8]) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "l"(p));
}
// Sixteen bf16 at p (16-byte aligned): one 32-byte load when p is 32-byte aligned,
// else two 16-byte loads.
__device__ __forceinline__ void ld_block16(const uint16_t* p, bool al32, uint32_t (&r)[8]) {
    if (al32) {
        ld_stream_v8(p, r);
    } else {
        const uint4 a = ld_stream_v4(p), b = ld_stream_v4(p + 8);
        r[0] = a.x; r[1] = a.y; r[2] = a.z; r[3] = a.w;
        r[4] = b.x; r[5] = b.y; r[6] = b.z; r[7] = b.w;
    }
}

// ============================================================================
// 16-point random Hadamard transform of bf16 inputs, exactly rounded.
//
// The quantizer sees y_j = RN32(sum_i s_i x_i H16[i][j]): the fp32 rounding of the
// exact sum (Sylvester H16, unnormalised; x . diag(s) . H16 == H16 . (s * x) since
// H16 is symmetric).  Four radix-2 butterfly stages compute it; after three stages
// every value is a signed sum of at most 8 inputs, the fourth adds two of those.
// A bf16 input with biased exponent E has 8 significant bits, so it is a multiple
// of 2^(max(E,1) - 134) below 2^(E - 126).  When the chunk's nonzero inputs satisfy
// E_max - max(E_min, 1) <= 13 (and E_max <= 251, no overflow), a sum of up to 8 of
// them is a multiple of 2^(max(E_min,1) - 134) below 8 * 2^(E_max - 126), i.e. below
// 2^24 such units: exactly representable in fp32.  The first three fp32 stages are
// then exact and the last is one correctly rounded addition of two exact values,
// which is RN32 of the exact sum.  Other chunks (rare: a tiny value beside a large
// one, or Inf / NaN) take an fp64 butterfly, exact while the span is at most 41
// binades; its fp32 rounding is the same RN32 of the exact sum.
// ============================================================================
// An exact zero sum is +0 (the real number 0): adding +0 to the first operand of the
// last stage turns a -0 partial sum into +0, and then a +- b is -0 for no inputs.
__device__ __forceinline__ void fwht16(double (&y)[16]) {
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {
        if (h == 8) {
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = __dadd_rn(y[i], 0.0);
        }
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

// bf16 bit pattern with its sign flipped where the rotation sign is -1.
__device__ __forceinline__ double bf16_signed_to_f64(uint32_t bits16, uint32_t flip) {
    return (double)__uint_as_float((bits16 ^ (flip << 15)) << 16);
}

// The exponent-span test above on one lane of chunk_mag_stats: mx and mn are the
// largest and smallest magnitude (bf16 patterns without sign).  A chunk holding a
// zero beside nonzero values (mn == 0) takes the fp64 path, which needs no span.
__device__ __forceinline__ bool span_ok_mag(uint32_t mx, uint32_t mn) {
    if (mx == 0u) return true;  // all inputs zero
    if (mn == 0u) return false;
    const int emax = (int)(mx >> 7), emin = (int)(mn >> 7);
    return emax <= 251 && emax - max(emin, 1) <= 13;
}

// Outside the fp64 butterfly's exact domain (span above 41 binades, or Inf / NaN):
// the transform is then the fp64 rounding, not the exact sum's.  Recorded in the
// status word (nullable) when a chunk of the quantizer's input lies there.
__device__ __forceinline__ void note_f64_domain(uint32_t vmx, uint32_t vmn, int* status) {
    if (status == nullptr || vmx == 0x7FFFu) return;
    const int emax = (int)((vmx - 0x7FFFu) >> 7);
    const int emin = (int)((vmn - 0x7FFFu) >> 7);
    if (emax <= 254 && emax - max(emin, 1) > 41) set_status(status, kStatusRhtRange);
}

// Chunk statistics of packed bf16 words (two independent lanes): per 16-bit lane,
// the unsigned maximum and signed minimum of v = |x| + 0x7FFF (no carry between the
// lanes: |x| <= 0x7FFF).
template <int N>
__device__ __forceinline__ void chunk_stats(const uint32_t (&w)[N], uint32_t& vmx, uint32_t& vmn) {
    vmx = 0u;
    vmn = 0x7FFF7FFFu;
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const uint32_t v = (w[i] & 0x7FFF7FFFu) + 0x7FFF7FFFu;
        vmx = vmax_u16x2(vmx, v);
        vmn = vmin_s16x2(vmn, v);
    }
}

// fp64 transform of one column of a column pair (half 0: low values, 1: high).
__device__ __forceinline__ void rht16_col_f64(const uint32_t (&w)[16], int half, uint32_t sign_mask,
                                              float (&y)[16]) {
    double d[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        d[i] = bf16_signed_to_f64(half ? (w[i] >> 16) : (w[i] & 0xFFFFu), (sign_mask >> i) & 1u);
    fwht16(d);
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = __double2float_rn(d[i]);
}

// Rotation of a column pair: w[i] holds row i of two adjacent columns (the first in
// the low half).  y0 / y1 receive the transforms of the two columns.
__device__ __forceinline__ void rht16_pair(const uint32_t (&w)[16], const RhtFlips& f, uint32_t sign_mask,
                                           float (&y0)[16], float (&y1)[16], int* status = nullptr) {
    uint32_t mx, mn;
    chunk_mag_stats<16>(w, mx, mn);
    if (span_ok_mag(mx & 0xFFFFu, mn & 0xFFFFu) && span_ok_mag(mx >> 16, mn >> 16)) {
        f32x2 x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = pk_bits(w[i] * 65536u + f.lo[i], (w[i] ^ f.pair[i]) & 0xFFFF0000u);
        const f32x2 zero2 = pk_bits(0u, 0u);
#pragma unroll
        for (int h = 1; h < 16; h <<= 1) {
            if (h == 8) {  // exact zero sums are +0 (see fwht16)
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] = add2(x[i], zero2);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                if ((i & h) == 0) {
                    const f32x2 a = x[i], b = x[i + h];
                    x[i] = add2(a, b);
                    x[i + h] = sub2(a, b);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) unpk(x[i], y0[i], y1[i]);
    } else {
        uint32_t vmx, vmn;
        chunk_stats<16>(w, vmx, vmn);
        note_f64_domain(vmx & 0xFFFFu, vmn & 0xFFFFu, status);
        note_f64_domain(vmx >> 16, vmn >> 16, status);
        rht16_col_f64(w, 0, sign_mask, y0);
        rht16_col_f64(w, 1, sign_mask, y1);
    }
}

// max_j |y_j| over both columns of a column pair.  On the fp32 path the last stage
// is not formed: max(|RN(a+b)|, |RN(a-b)|) = RN(|a| + |b|) exactly (RN is monotone
// and odd, and max(|a+b|, |a-b|) = |a| + |b|).
__device__ __forceinline__ float rht16_pair_absmax(const uint32_t (&w)[16], const RhtFlips& f,
                                                   uint32_t sign_mask, uint32_t mx, uint32_t mn,
                                                   int* status) {
    float m = 0.0f;
    if (span_ok_mag(mx & 0xFFFFu, mn & 0xFFFFu) && span_ok_mag(mx >> 16, mn >> 16)) {
        f32x2 x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = pk_bits(w[i] * 65536u + f.lo[i], (w[i] ^ f.pair[i]) & 0xFFFF0000u);
#pragma unroll
        for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                if ((i & h) == 0) {
                    const f32x2 a = x[i], b = x[i + h];
                    x[i] = add2(a, b);
                    x[i + h] = sub2(a, b);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float a0, a1, b0, b1;
            unpk(x[j], a0, a1);
            unpk(x[j + 8], b0, b1);
            m = fmaxf(m, fmaxf(fabsf(a0) + fabsf(b0), fabsf(a1) + fabsf(b1)));
        }
    } else {
        uint32_t vmx, vmn;
        chunk_stats<16>(w, vmx, vmn);
        note_f64_domain(vmx & 0xFFFFu, vmn & 0xFFFFu, status);
        note_f64_domain(vmx >> 16, vmn >> 16, status);
        float y[16];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            rht16_col_f64(w, half, sign_mask, y);
#pragma unroll
            for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(y[i]));
        }
    }
    return m;
}

// Upper bounds of max_j |y_j| for the two columns of a column pair (w as in
// rht16_pair), and the pair's magnitudes folded into m_row (two packed 16-bit
// maxima, the same as chunk_mag_stats' largest magnitude).  Every entry of H16 is
// +-1, so |y_j| <= sum_i |x_i|.  The sums round upward, so each bound is a float at
// or above the exact sum, hence at or above RN32(|y_j|) for every j.  The high value
// of a word is read as fp32 with the low value's magnitude bits below its mantissa,
// which can only raise it.  An Inf or NaN input makes the bound Inf or NaN.
__device__ __forceinline__ f32x2 pair_l1_up(const uint32_t (&w)[16], uint32_t& m_row) {
    f32x2 s[4];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint32_t t = w[i] & 0x7FFF7FFFu;
        m_row = vmax_u16x2(m_row, t);
        const f32x2 v = pk_bits(t << 16, t);
        s[i & 3] = i < 4 ? v : add2_ru(s[i & 3], v);
    }
    return add2_ru(add2_ru(s[0], s[1]), add2_ru(s[2], s[3]));
}

// Rotation of one row block held by one thread: w[k] holds elements 2k, 2k+1 of the
// block (16 values).  Scalar fp32 butterfly under the same span test, else fp64.
__device__ __forceinline__ void rht16_row(const uint32_t (&w)[8], uint32_t sign_mask, float (&y)[16],
                                          int* status = nullptr) {
    uint32_t mx2, mn2;
    chunk_mag_stats<8>(w, mx2, mn2);
    if (span_ok_mag(max(mx2 & 0xFFFFu, mx2 >> 16), min(mn2 & 0xFFFFu, mn2 >> 16))) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t b = (i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xFFFFu);
            y[i] = __uint_as_float((b ^ (((sign_mask >> i) & 1u) << 15)) << 16);
        }
#pragma unroll
        for (int h = 1; h < 16; h <<= 1) {
            if (h == 8) {  // exact zero sums are +0 (see fwht16)
#pragma unroll
                for (int i = 0; i < 8; ++i) y[i] = __fadd_rn(y[i], 0.0f);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                if ((i & h) == 0) {
                    const float a = y[i], b = y[i + h];
                    y[i] = __fadd_rn(a, b);
                    y[i + h] = __fsub_rn(a, b);
                }
            }
        }
    } else {
        uint32_t vmx, vmn;
        chunk_stats<8>(w, vmx, vmn);
        note_f64_domain(max(vmx & 0xFFFFu, vmx >> 16),
                        (uint32_t)(uint16_t)min((int16_t)(vmn & 0xFFFFu), (int16_t)(vmn >> 16)), status);
        double d[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            d[i] = bf16_signed_to_f64((i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xFFFFu), (sign_mask >> i) & 1u);
        fwht16(d);
#pragma unroll
        for (int i = 0; i < 16; ++i) y[i] = __double2float_rn(d[i]);
    }
}

// 16-point rotation of a row chunk held by a lane pair (even lane: elements 0-7,
// odd lane: 8-15; both lanes of every pair call this together): three butterfly
// stages inside the lane, the last across the pair, in fp64 (exact like fwht16).
// Used by the amax pass of the rotated row orientation.
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

// ============================================================================
// amax prepass.  One warp handles a 16-row x 256-column unit, each lane 16 rows
// x 8 columns (sixteen 16-byte loads).  Word 0 receives max |x| (fp32 bits of a
// bf16 magnitude; NaN patterns sort above Inf), word 1 max |RHT16 down the
// rows| (column orientation), as fp32 bits.  Both are combined with atomicMax.
// Launched for the plain max |x| and for the rotated row orientation; the rotated
// column orientation alone goes through amax_stream_kernel.
// ============================================================================
// Grouped (kGrouped): the rows of a unit lie in one group, whose words are
// words[2g] and words[2g+1]; each unit is folded into them by the warp.
// kRowRht: word 0 (or 2g) is max |RHT16 along the rows| instead of max |x| (the
// row orientation is rotated); a non-finite input still makes it non-finite.
template <bool kColRht, bool kRowRht>
constexpr int amax_min_blocks() {
    return (kColRht && kRowRht) ? 1 : 2;  // both rotations: registers for one CTA per SM
}
template <bool kColRht, bool kGrouped, bool kRowRht>
__global__ void __launch_bounds__(256, (amax_min_blocks<kColRht, kRowRht>())) amax_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                   int64_t cols, uint32_t sign_mask, const RhtFlips flips,
                                                   uint32_t* __restrict__ words,
                                                   const int32_t* __restrict__ row_group,
                                                   int64_t group_rows_uniform, int* status) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t col_units = (cols + 255) >> 8;
    const int64_t units = ((rows + 15) >> 4) * col_units;
    uint32_t m_row = 0;   // two packed 16-bit magnitudes
    float m_col = 0.0f;
    double m_rrht = 0.0;  // kRowRht: max |rotated row|
    for (int64_t u = (int64_t)blockIdx.x * 8 + warp; u < units; u += (int64_t)gridDim.x * 8) {
        const int64_t r0 = (u / col_units) * 16;
        const int64_t c0 = (u % col_units) * 256 + lane * 8;
        if (kGrouped) {
            m_row = 0;
            m_col = 0.0f;
        }
        if (kRowRht || c0 < cols) {
        uint4 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const bool in = c0 < cols && r0 + i < rows;
            v[i] = in ? ld_stream_v4(x + (r0 + i) * cols + c0) : make_uint4(0, 0, 0, 0);
        }
        if (kRowRht) {  // every lane takes part (zeros past the columns)
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                double y[8];
                rht16_lane_pair(v[i], sign_mask, lane, y);
#pragma unroll
                for (int k = 0; k < 8; ++k) m_rrht = fmax(m_rrht, fabs(y[k]));
            }
        }
        if (kColRht) {
            // column pairs (2c, 2c+1) of the lane's 8 columns: the chunk statistics
            // give max |x| too
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) w[i] = c == 0 ? v[i].x : c == 1 ? v[i].y : c == 2 ? v[i].z : v[i].w;
                uint32_t mx, mn;
                chunk_mag_stats<16>(w, mx, mn);
                m_row = vmax_u16x2(m_row, mx);
                m_col = fmaxf(m_col, rht16_pair_absmax(w, flips, sign_mask, mx, mn, status));
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                m_row = __vmaxu2(m_row, v[i].x & 0x7FFF7FFFu);
                m_row = __vmaxu2(m_row, v[i].y & 0x7FFF7FFFu);
                m_row = __vmaxu2(m_row, v[i].z & 0x7FFF7FFFu);
                m_row = __vmaxu2(m_row, v[i].w & 0x7FFF7FFFu);
            }
        }
        }
        if (kGrouped) {
            const int64_t g = row_group ? (int64_t)row_group[r0 >> 7] : r0 / group_rows_uniform;
            uint32_t ur = max(m_row & 0xFFFFu, m_row >> 16) << 16;
            uint32_t uc = kColRht ? __float_as_uint(m_col) : 0u;
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
    uint32_t a_col = kColRht ? __float_as_uint(m_col) : 0u;
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
// amax prepass of the rotated column orientation, streamed through shared
// memory.  Each warp walks a contiguous range of 16-row x 128-column units.  The
// whole warp copies a unit into one of its kAmaxSlots slots with 16-byte cp.async
// (eight per lane; rows past the tensor, padding rows, gathered rows with an index
// past the source and columns past the tensor are zero-filled, so they count as
// zeros); the copies of the next kAmaxSlots - 1 units are in flight while it works
// on one, so the DRAM latency hides behind the arithmetic and no register holds
// data in flight.  Lane l then takes columns 4l .. 4l+3 of the 16 rows (two column
// pairs): max |x|, and max |RHT16 down the rows| (rht16_pair_absmax) for the column
// pairs that can still raise it.  Results, word layout and grouping are those of
// amax_kernel.
//
// The rotation is skipped where it cannot change the result.  The warp keeps a
// threshold: the largest rotated magnitude that it, or any warp that has published to
// the output word (or the group's word), computed.  A column whose rounded-up sum of
// |x| (pair_l1_up) is at most the threshold has no rotated value above it.  The word
// ends at least at the threshold, so skipping such a column leaves the word unchanged.
// A warp publishes its maximum to the word (atomicMax) when the maximum passes the
// threshold.  It reads the word back when it starts the unit after one in which it
// rotated (and on a new group), after that unit's data has landed, so that the read
// sees what the other warps published meanwhile.  Only a rotated chunk records the
// fp64-domain status; the quantizer's tile pass rotates every chunk, so it records
// that status for the same input.
// ============================================================================
__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// 16-byte copy global -> shared, `src_bytes` of it read (the rest zero-filled).
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src), "r"(src_bytes)
                 : "memory");
}
constexpr int kAmaxWarps = 8;
constexpr int kAmaxUnitCols = 128;
constexpr int kAmaxSlotBytes = 16 * kAmaxUnitCols * 2;                  // 4 KB
constexpr int kAmaxSlots = 2;                                           // units in flight + 1
constexpr int kAmaxSmemBytes = kAmaxWarps * kAmaxSlots * kAmaxSlotBytes;  // 64 KB
constexpr int kAmaxCtasPerSm = 2;

template <bool kGrouped, bool kGather>
__global__ void __launch_bounds__(kAmaxWarps * 32, kAmaxCtasPerSm)
    amax_stream_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols, uint32_t sign_mask,
                       const RhtFlips flips, uint32_t* __restrict__ words, const int32_t* __restrict__ row_group,
                       int64_t group_rows_uniform, const int32_t* __restrict__ row_src, int64_t src_rows,
                       int* status) {
    extern __shared__ __align__(128) uint8_t amax_smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t full_mask = 0xFFFFFFFFu;
    uint8_t* const slots = amax_smem + warp * kAmaxSlots * kAmaxSlotBytes;

    const int64_t col_units = (cols + kAmaxUnitCols - 1) / kAmaxUnitCols;
    const int64_t units = ((rows + 15) >> 4) * col_units;
    const int64_t nw = (int64_t)gridDim.x * kAmaxWarps;
    const int64_t per = (units + nw - 1) / nw;
    const int64_t u_begin = ((int64_t)blockIdx.x * kAmaxWarps + warp) * per;
    const int64_t u_end = u_begin + per < units ? u_begin + per : units;

    // Unit u is 16-row block u / col_units, 128-column block u % col_units; the warp's
    // units are consecutive, so both indices advance by counting (one division).
    // Copies of the unit at (ru, cu) into slot `slot`: 16 rows x 16 chunks of 16
    // bytes, chunk lane + 32k of the unit being row 2k + lane / 16, chunk lane % 16.
    // One commit group per unit and lane.
    auto issue = [&](int64_t ru, int64_t cu, int slot) {
        const int64_t r0 = ru * 16;
        const int64_t col = cu * kAmaxUnitCols + (lane & 15) * 8;
        int64_t sr = -1;  // kGather: the source row of unit row `lane` (lanes 0-15)
        if (kGather && lane < 16 && r0 + lane < rows) {
            sr = __ldg(row_src + r0 + lane);
            if (sr >= src_rows) {
                set_status(status, kStatusIndex);
                sr = -1;
            }
        }
        uint8_t* const dst = slots + slot * kAmaxSlotBytes + (lane & 15) * 16;
        if (!kGather && r0 + 16 <= rows && cu * kAmaxUnitCols + kAmaxUnitCols <= cols) {  // a whole unit
            const uint16_t* src = x + (r0 + (lane >> 4)) * cols + col;
#pragma unroll
            for (int k = 0; k < 8; ++k)
                cp_async16(dst + (2 * k + (lane >> 4)) * (kAmaxUnitCols * 2), src + 2 * k * cols, 16u);
            asm volatile("cp.async.commit_group;" ::: "memory");
            return;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int row = 2 * k + (lane >> 4);
            int64_t src_row = r0 + row;
            bool in = col < cols && src_row < rows;
            if (kGather) {
                src_row = __shfl_sync(full_mask, sr, row);
                in = col < cols && src_row >= 0;
            }
            cp_async16(dst + row * (kAmaxUnitCols * 2), in ? (const void*)(x + src_row * cols + col) : (const void*)x,
                       in ? 16u : 0u);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    uint32_t m_row = 0;  // two packed 16-bit magnitudes (the row orientation's max |x|)
    float m_col = 0.0f;
    float thr = 0.0f;     // warp-uniform skip threshold (a rotated magnitude computed for this word)
    bool reread = false;  // read the word again for this unit (the last one rotated, or a new group)
    int64_t g_cur = -1;   // kGrouped: the group the running maxima belong to
    auto row_max = [&]() -> uint32_t {  // fp32 bits of the largest magnitude seen
        return max(m_row & 0xFFFFu, m_row >> 16) << 16;
    };
    auto flush_group = [&]() {
        uint32_t ur = row_max();
        uint32_t uc = __float_as_uint(m_col);
        ur = __reduce_max_sync(full_mask, ur);
        uc = __reduce_max_sync(full_mask, uc);
        if (lane == 0 && g_cur >= 0) {
            if (ur) atomicMax(words + 2 * g_cur, ur);
            if (uc) atomicMax(words + 2 * g_cur + 1, uc);
        }
        m_row = 0;
        m_col = 0.0f;
    };

    int64_t ru = u_begin / col_units, cu = u_begin % col_units;  // the unit being computed
    int64_t ru_n = ru, cu_n = cu;                                // the next unit to copy
    auto advance = [&](int64_t& r, int64_t& c) {
        if (++c == col_units) {
            c = 0;
            ++r;
        }
    };
    // kAmaxSlots - 1 units in flight ahead of the one being computed (one commit group
    // per unit, empty past the warp's range, so that the group count stays fixed)
#pragma unroll
    for (int k = 0; k < kAmaxSlots - 1; ++k) {
        if (u_begin + k < u_end) {
            issue(ru_n, cu_n, k);
            advance(ru_n, cu_n);
        } else {
            asm volatile("cp.async.commit_group;" ::: "memory");
        }
    }
    int slot = 0;
    for (int64_t u = u_begin; u < u_end; ++u) {
        if (u + kAmaxSlots - 1 < u_end) {
            // the slot computed last; every lane's reads of it are done
            issue(ru_n, cu_n, slot == 0 ? kAmaxSlots - 1 : slot - 1);
            advance(ru_n, cu_n);
        } else {
            asm volatile("cp.async.commit_group;" ::: "memory");
        }
        // this lane's copies of the unit landed, then every other lane's
        asm volatile("cp.async.wait_group %0;" ::"n"(kAmaxSlots - 1) : "memory");
        __syncwarp();
        const int64_t r0 = ru * 16;
        if (kGrouped) {
            const int64_t g = row_group ? (int64_t)row_group[r0 >> 7] : r0 / group_rows_uniform;
            if (g != g_cur) {
                flush_group();
                g_cur = g;
                thr = 0.0f;  // the threshold belonged to the last group
                reread = true;
            }
        }
        uint32_t* const col_word = kGrouped ? words + 2 * g_cur + 1 : words + 1;
        const bool lane_in = cu * kAmaxUnitCols + 4 * lane < cols;
        const uint8_t* base = slots + slot * kAmaxSlotBytes + lane * 8;
        uint32_t wa[16], wb[16];  // rows of column pairs (4l, 4l+1) and (4l+2, 4l+3)
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint2 q = *reinterpret_cast<const uint2*>(base + i * (kAmaxUnitCols * 2));
            wa[i] = q.x;
            wb[i] = q.y;
        }
        __syncwarp();  // every lane's reads of the slot are done before its refill
        // the word as other warps have left it (read after the wait, used after the
        // first bound, so that the read has time to return)
        const uint32_t seen = reread ? ld_relaxed_u32(col_word) : 0u;
        float a0, a1, b0, b1;
        unpk(pair_l1_up(wa, m_row), a0, a1);
        thr = fmaxf(thr, __uint_as_float(seen));
        const float t_lane = fmaxf(thr, m_col);
        const bool need_a = !(a0 <= t_lane && a1 <= t_lane);  // a NaN bound is rotated
        if (need_a) {
            uint32_t mx, mn;
            chunk_mag_stats<16>(wa, mx, mn);
            m_col = fmaxf(m_col, rht16_pair_absmax(wa, flips, sign_mask, mx, mn, lane_in ? status : nullptr));
        }
        unpk(pair_l1_up(wb, m_row), b0, b1);
        const bool need_b = !(b0 <= t_lane && b1 <= t_lane);
        if (need_b) {
            uint32_t mx, mn;
            chunk_mag_stats<16>(wb, mx, mn);
            m_col = fmaxf(m_col, rht16_pair_absmax(wb, flips, sign_mask, mx, mn, lane_in ? status : nullptr));
        }
        reread = __any_sync(full_mask, need_a || need_b);
        if (reread) {
            const float wmax = __uint_as_float(__reduce_max_sync(full_mask, __float_as_uint(m_col)));
            if (wmax > thr) {
                thr = wmax;
                if (lane == 0) atomicMax(col_word, __float_as_uint(wmax));
            }
        }
        advance(ru, cu);
        slot = slot + 1 == kAmaxSlots ? 0 : slot + 1;
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    if (kGrouped) {
        flush_group();
        return;
    }
    uint32_t a_row = row_max();
    uint32_t a_col = __float_as_uint(m_col);
    a_row = __reduce_max_sync(full_mask, a_row);
    a_col = __reduce_max_sync(full_mask, a_col);
    __shared__ uint32_t red[2][kAmaxWarps];
    if (lane == 0) {
        red[0][warp] = a_row;
        red[1][warp] = a_col;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t r = 0, c = 0;
#pragma unroll
        for (int w = 0; w < kAmaxWarps; ++w) {
            r = max(r, red[0][w]);
            c = max(c, red[1][w]);
        }
        if (r) atomicMax(words + 0, r);
        if (c) atomicMax(words + 1, c);
    }
}

// ============================================================================
// Shared helpers of the quantize kernels.
// ============================================================================
__device__ __forceinline__ bool finite_bits(uint32_t b) { return (b & 0x7FFFFFFFu) < 0x7F800000u; }

// Element multiplier of E4M3 block-scale code s: 1 / (dec(s) * g), 0 when that
// product is 0, clamped to FLT_MAX (the op order of block_scale).  A CTA fills a
// 256-entry table once per tensor scale and looks the multiplier up per block.
__device__ __forceinline__ float block_inv_of_code(uint32_t s, float g) {
    const float d = __fmul_rn(e4m3_to_f32(s), g);
    return (d == 0.0f) ? 0.0f : fminf(__frcp_rn(d), 3.402823466e38f);  // correctly rounded 1 / d
}
// RN(a / 6) for finite a >= 0.  With y = RN(1/6): q = RN(a y) is within an ulp of
// a / 6, the residual a - 6q is exact in one FMA, and RN(q + r y) is the correctly
// rounded quotient -- the correction step for division by a constant (Markstein;
// Brisebarre, Muller and Raina, "Accelerating correctly rounded floating-point
// division when the divisor is known in advance", IEEE TC 2004).  An exhaustive host
// test (tests/test_div6_host.py) shows it equal to IEEE division for every fp32
// a >= 2^-125; smaller a (quotients near the subnormal range) take the division.
__device__ __forceinline__ float div6_rn(float a) {
    if (a < 0x1p-125f) return __fdiv_rn(a, 6.0f);
    const float y = 0x1.555556p-3f;  // RN(1/6)
    const float q = __fmul_rn(a, y);
    return __fmaf_rn(__fmaf_rn(-q, 6.0f, a), y, q);
}
// E4M3 code of a block with amax_b: RNE_satfinite((amax_b / 6) * enc).
__device__ __forceinline__ uint32_t block_code(float amax_b, const TensorScale& ts) {
    return e4m3_rn_satfinite(__fmul_rn(div6_rn(amax_b), ts.enc));
}

// Stochastic rounding of eight values y * inv to packed E2M1 codes (element i in
// bits [4i, 4i+4), the sign bit of y kept, zero included; |y * inv| > 6 gives 6)
// with the B200's stochastic conversion, cvt.rs.satfinite.e2m1x4.f32.  Given
// {0, b, 0, f} it writes f's code to nibble 0 and b's to nibble 2 and rounds each
// up iff R + floor(p * 2^16) >= 2^16, p the position of |v| between its grid
// neighbours, R = bytes 2:0 of the random word for f and bytes 3:1 for b: two
// elements per conversion, 16 draw bits each (the other two lanes hold exact
// zeros, which no draw moves).  Words x, y, z, w of the Philox block serve the
// element pairs (0,2), (1,3), (4,6), (5,7); two shifted sums interleave the nibbles.
__device__ __forceinline__ uint32_t cvt_rs_e2m1_pair(float b, float f, uint32_t rbits) {
    uint16_t d;
    asm("cvt.rs.satfinite.e2m1x4.f32 %0, {%1, %2, %1, %3}, %4;"
        : "=h"(d)
        : "f"(0.0f), "f"(b), "f"(f), "r"(rbits));
    return d;
}
__device__ __forceinline__ uint32_t sr_codes8(const float (&y)[8], float inv, const Philox4& rnd) {
    const f32x2 iv = pk(inv, inv);
    float v[8];
#pragma unroll
    for (int m = 0; m < 4; ++m) unpk(mul2(pk(y[2 * m], y[2 * m + 1]), iv), v[2 * m], v[2 * m + 1]);
    const uint32_t c02 = cvt_rs_e2m1_pair(v[2], v[0], rnd.x), c13 = cvt_rs_e2m1_pair(v[3], v[1], rnd.y);
    const uint32_t c46 = cvt_rs_e2m1_pair(v[6], v[4], rnd.z), c57 = cvt_rs_e2m1_pair(v[7], v[5], rnd.w);
    return (c02 + (c13 << 4)) | ((c46 + (c57 << 4)) << 16);
}

// Round-to-nearest-even codes of y * inv, eight values.
__device__ __forceinline__ uint32_t rn_codes8(const float (&y)[8], float inv) {
    const f32x2 iv = pk(inv, inv);
    float q[8];
#pragma unroll
    for (int m = 0; m < 4; ++m) unpk(mul2(pk(y[2 * m], y[2 * m + 1]), iv), q[2 * m], q[2 * m + 1]);
    return e2m1x8_rn(q);
}

// One 16-element block (element index e0 % 16 == 0 of the quantized tensor) ->
// two words of packed codes, RNE or SR (stream `stream`).
__device__ __forceinline__ uint2 encode16(const float (&y)[16], float inv, bool sr, const uint32_t (&rk)[20],
                                          uint32_t stream, uint64_t e0) {
    float lo[8], hi[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        lo[i] = y[i];
        hi[i] = y[8 + i];
    }
    if (!sr) return make_uint2(rn_codes8(lo, inv), rn_codes8(hi, inv));
    return make_uint2(sr_codes8(lo, inv, sr_draws8(rk, stream, e0 >> 3)),
                      sr_codes8(hi, inv, sr_draws8(rk, stream, (e0 >> 3) + 1)));
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

__device__ __forceinline__ void unpack16(const uint32_t (&w)[8], float (&v)[16]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        v[2 * k] = bf16_lo(w[k]);
        v[2 * k + 1] = bf16_hi(w[k]);
    }
}

// max |x| of a 16-element block (two full-rate packed maxima per word, see
// chunk_mag_stats); NaN patterns sort above Inf.
__device__ __forceinline__ float absmax16(const uint32_t (&w)[8]) {
    uint32_t u = 0u, sg = 0x80008000u;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        u = vmax_u16x2(u, w[k]);
        sg = vmax_s16x2(sg, w[k]);
    }
    const uint32_t m = vmax_u16x2(u & 0x7FFF7FFFu, sg & 0x7FFF7FFFu);
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
// Row orientation only, 1x16 blocks: every thread owns whole 16-element blocks
// (one 32-byte load each).  Grid-stride over blocks.
// ============================================================================
__global__ void __launch_bounds__(256) quant_rows_kernel(QuantParams p) {
    TensorScale tr, tc;
    if (!load_tensor_scales(p, tr, tc)) return;
    __shared__ float inv_tab[256];
    inv_tab[threadIdx.x] = block_inv_of_code(threadIdx.x, tr.g);
    __syncthreads();
    const int64_t bpr = p.cols >> 4;  // 16-blocks per row
    const int64_t nblocks = p.rows * bpr;
    const int64_t katoms = (bpr + 3) >> 2;
    const bool al32 = (reinterpret_cast<uintptr_t>(p.x) & 31u) == 0;
    // grid-stride over blocks; the next block's 32 bytes are loaded while this one is
    // encoded, and its (row, block) position advances by counting
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= nblocks) return;
    const int64_t stride_r = stride / bpr, stride_kb = stride % bpr;
    int64_t r = b / bpr, kb = b % bpr;
    uint32_t w[8];
    ld_block16(p.x + b * 16, al32, w);
    for (;;) {
        const int64_t bn = b + stride;
        uint32_t wn[8];
        if (bn < nblocks) ld_block16(p.x + bn * 16, al32, wn);
        const uint32_t s = block_code(absmax16(w), tr);
        const float inv = inv_tab[s];
        float v[16];
        unpack16(w, v);
        const uint2 codes = encode16(v, inv, p.row_sr, p.rk, 0u, (uint64_t)b * 16);
        reinterpret_cast<uint2*>(p.row_data)[b] = codes;
        p.row_sf[sf_offset(r, kb, katoms)] = (uint8_t)s;
        if (bn >= nblocks) break;
        b = bn;
        r += stride_r;
        kb += stride_kb;
        if (kb >= bpr) {
            kb -= bpr;
            ++r;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) w[k] = wn[k];
    }
}

// ============================================================================
// Tile kernel: a CTA quantizes one 128 x 128 bf16 tile (a grouped tensor's group
// boundaries are multiples of 128 rows, so a tile lies in one group).  The tile goes
// straight from global to shared memory (cp.async, 16 bytes per copy, eight per
// thread; rows and columns past the tensor and gathered padding rows are zero-filled
// by the copy itself), so no register holds it in flight.  Then one thread per
// 16-element row block writes the row orientation, and one thread per column pair
// and 16-row chunk writes the column orientation.  k2D: 16x16 blocks, the tile scale is found by the
// column pass and shared by both orientations.  kRht: the 16-point RHT down each
// column chunk before the column orientation is quantized.  kRowRht: the row
// orientation is rotated along each row block (the Mosaic recipe's dgrad operands).
// kGrouped: the tile's rows lie in one group g (see QuantParams), which supplies the
// tensor scales, the Philox key seed + g and the origin of the element indices.
// Tiles run bottom-up (the grid's y extent reversed), so the first tiles re-read the
// rows the amax pass read last (still in L2).
// ============================================================================
constexpr int kTR = 128, kTC = 128, kPitch = kTC + 8;  // +16 bytes per row: conflict-free column reads

// The work on one tile whose bf16 values are in `tile` (rows r0.., columns c0..)
// with the multiplier tables filled: row orientation, column orientation and the
// scale atoms.  Every thread of the CTA calls it (it meets the CTA's barriers).
template <bool k2D, bool kRht, bool kGrouped, bool kRowRht>
__device__ __forceinline__ void tile_passes(const QuantParams& p, int64_t r0, int64_t c0,
                                            const uint16_t (*tile)[kPitch], const float (*inv_tab)[256],
                                            uint32_t (*tile_s)[kTC / 16], float (*tile_inv)[kTC / 16],
                                            uint8_t* col_atom, uint8_t (*row_atoms)[32][16],
                                            const TensorScale& tr, const TensorScale& tc,
                                            const uint32_t (&rk)[20], int64_t g_row0, int64_t g_rows) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    (void)lane;  // not every variant reads both
    (void)warp;
    const bool want_row = p.row_data != nullptr;
    const bool want_col = p.col_data != nullptr;
    // ---- row pass: row block b = k * 256 + tid is row b / 8, columns (b % 8) * 16 .. + 15
    auto row_pass = [&]() {
#pragma unroll
        for (int k = 0; k < kTR / 32; ++k) {
            const int lr = (k * 256 + tid) >> 3, bc = tid & 7, lc = bc * 16;
            const int64_t r = r0 + lr, c = c0 + lc;
            // two 16-byte reads, the lane quads of a row taking the halves in opposite
            // order so that eight lanes cover all 32 banks
            const int h = (lane >> 2) & 1;
            const uint4* src = reinterpret_cast<const uint4*>(&tile[lr][lc]);
            const uint4 q0 = src[h], q1 = src[h ^ 1];
            const uint4 lo = h ? q1 : q0, hi = h ? q0 : q1;
            const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
            const bool inside = r < p.rows && c < p.cols;
            uint32_t sc;
            float inv;
            float v[16];
            if (kRowRht) {
                rht16_row(w, p.sign_mask, v, inside ? p.status : nullptr);
                float amax = 0.0f;
#pragma unroll
                for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(v[e]));
                sc = block_code(amax, tr);
                inv = inv_tab[0][sc];
            } else if (k2D) {
                sc = tile_s[lr >> 4][bc];
                inv = tile_inv[lr >> 4][bc];
                unpack16(w, v);
            } else {
                sc = block_code(absmax16(w), tr);
                inv = inv_tab[0][sc];
                unpack16(w, v);
            }
            const uint2 codes =
                encode16(v, inv, p.row_sr, rk, 0u, (uint64_t)(r - g_row0) * (uint64_t)p.cols + (uint64_t)c);
            if (inside) *reinterpret_cast<uint2*>(p.row_data + r * (p.cols >> 1) + (c >> 1)) = codes;
            // (row lr, block bc): atom bc / 4, line lr % 32, byte 4 * (lr / 32) + bc % 4
            row_atoms[bc >> 2][lr & 31][(lr >> 5) * 4 + (bc & 3)] = inside ? (uint8_t)sc : (uint8_t)0;
        }
    };
    if (want_row && !k2D) row_pass();

    // ---- column pass: thread -> column pair cp (columns 2cp, 2cp+1), 16-row chunks
    // j = tid / 64 + 4 i
    if (want_col || k2D) {
#pragma unroll 1
    for (int jj = 0; jj < kTR / 64; ++jj) {
        const int cp = tid & 63, j = (tid >> 6) + 4 * jj;
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) w[e] = *reinterpret_cast<const uint32_t*>(&tile[16 * j + e][2 * cp]);
        const bool rin = r0 + 16 * j < p.rows;
        const bool chunk_in = c0 + 2 * cp < p.cols && rin;
        float a0 = 0.0f, a1 = 0.0f;
        float y0[16], y1[16];
        if (kRht) {
            rht16_pair(w, p.flips, p.sign_mask, y0, y1, chunk_in ? p.status : nullptr);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                a0 = fmaxf(a0, fabsf(y0[e]));
                a1 = fmaxf(a1, fabsf(y1[e]));
            }
        } else {
            uint32_t u = 0u, sg = 0x80008000u;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                u = vmax_u16x2(u, w[e]);
                sg = vmax_s16x2(sg, w[e]);
            }
            const uint32_t m = vmax_u16x2(u & 0x7FFF7FFFu, sg & 0x7FFF7FFFu);
            a0 = __uint_as_float(m << 16);
            a1 = __uint_as_float(m & 0xFFFF0000u);
        }
        uint32_t s0, s1;
        float inv0, inv1;
        if (k2D) {
            // the 16x16 tile: 8 consecutive lanes hold its 16 columns
            float a = fmaxf(a0, a1);
#pragma unroll
            for (int o = 4; o >= 1; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
            s0 = s1 = block_code(a, tc);
            inv0 = inv1 = inv_tab[1][s0];
            if ((cp & 7) == 0) {
                tile_s[j][cp >> 3] = s0;
                tile_inv[j][cp >> 3] = inv0;
            }
        } else {
            s0 = block_code(a0, tc);
            s1 = block_code(a1, tc);
            inv0 = inv_tab[1][s0];
            inv1 = inv_tab[1][s1];
        }
        if (want_col) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int lc = 2 * cp + h;
                const int64_t c = c0 + lc;
                const uint64_t e0 = (uint64_t)c * (uint64_t)g_rows + (uint64_t)(r0 - g_row0 + 16 * j);
                uint2 codes;
                if (kRht) {
                    codes = encode16(h ? y1 : y0, h ? inv1 : inv0, p.col_sr, rk, 1u, e0);
                } else {
                    float y[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) y[e] = h ? bf16_hi(w[e]) : bf16_lo(w[e]);
                    codes = encode16(y, h ? inv1 : inv0, p.col_sr, rk, 1u, e0);
                }
                const bool inside = c < p.cols && rin;
                if (inside)
                    *reinterpret_cast<uint2*>(p.col_data + c * (p.rows >> 1) + ((r0 + 16 * j) >> 1)) = codes;
                // staged block-major (byte j * 128 + lc: a warp's stores are consecutive
                // bytes); the atom store below reorders them into the atom's lines
                col_atom[j * 128 + lc] = inside ? (uint8_t)(h ? s1 : s0) : (uint8_t)0;
            }
        }
    }
    }
    if (want_row && k2D) {
        __syncthreads();  // tile scales written
        row_pass();
    }

    // ---- scale stores.  Every entry written lies inside the scale buffer: a
    // column atom is (128-column group c0 / 128, blocks 4a .. 4a+3 of rows) for the
    // tile's 64-row groups a that start below the padded block count; the row atoms
    // cover the tile's 128 rows below pad128(rows), and the second is skipped when its
    // blocks start past the padded block count.
    __syncthreads();
    if (want_col && warp < kTR / 64) {
        const int64_t katoms_c = (p.rows / 16 + 3) >> 2;
        if ((r0 >> 6) + warp < katoms_c) {
            const int64_t atom = (c0 >> 7) * katoms_c + (r0 >> 6) + warp;
            const uint8_t* ca = col_atom + warp * 512;
            // line l of the atom: byte 4w + j holds (column l + 32w, block j)
            uint32_t line[4];
#pragma unroll
            for (int w = 0; w < 4; ++w)
                line[w] = (uint32_t)ca[lane + 32 * w] | ((uint32_t)ca[128 + lane + 32 * w] << 8) |
                          ((uint32_t)ca[256 + lane + 32 * w] << 16) | ((uint32_t)ca[384 + lane + 32 * w] << 24);
            *reinterpret_cast<uint4*>(p.col_sf + atom * 512 + lane * 16) = make_uint4(line[0], line[1], line[2], line[3]);
        }
    }
    if (want_row && (warp == 2 || warp == 3)) {
        const int64_t katoms_r = (p.cols / 16 + 3) >> 2;
        const int a = warp - 2;
        if ((c0 >> 6) + a < katoms_r) {
            const int64_t atom = (r0 >> 7) * katoms_r + (c0 >> 6) + a;
            *reinterpret_cast<uint4*>(p.row_sf + atom * 512 + lane * 16) =
                *reinterpret_cast<const uint4*>(row_atoms[a][lane]);
        }
    }
}

// Resident CTAs per SM the register budget is sized for (each CTA quantizes one tile,
// so more resident CTAs keep more copies and more independent arithmetic in flight).
// Three (80 registers) for the dense rotated passes, which spill 20 B there and run
// 3% faster than at four; four (64 registers) for the others, the grouped rotated
// variant included (three measured the same).
template <bool k2D, bool kRht, bool kGrouped>
constexpr int quant_tile_min_blocks() {
    return (kRht && !kGrouped) ? 3 : 4;
}

template <bool k2D, bool kRht, bool kGrouped, bool kRowRht>
__global__ void __launch_bounds__(256, (quant_tile_min_blocks<k2D, kRht, kGrouped>()))
    quant_tile_kernel(const QuantParams p) {
    __shared__ __align__(16) uint16_t tile[kTR][kPitch];
    __shared__ float inv_tab[2][256];  // element multipliers of every scale code: rows, columns
    __shared__ uint32_t tile_s[kTR / 16][kTC / 16];
    __shared__ float tile_inv[kTR / 16][kTC / 16];
    // The tile's scales, staged so that they leave in wide stores instead of one
    // byte each: each 64-row half of the column orientation's 128 columns x 8 blocks
    // is exactly one 512-byte atom (staged block-major, reordered into lines when
    // stored); the row orientation's 128 rows x 8 blocks are exactly two atoms.
    // Entries past the tensor hold 0 (the padding).
    __shared__ __align__(16) uint8_t col_atom[kTR / 16 * 128];
    __shared__ __align__(16) uint8_t row_atoms[2][32][16];

    const int tid = threadIdx.x;
    const int64_t r0 = (int64_t)(gridDim.y - 1 - blockIdx.y) * kTR, c0 = (int64_t)blockIdx.x * kTC;

    // ---- copies first (they do not depend on the scales): 2048 x 16 bytes, eight per
    // thread; copy q covers row q / 16, columns (q % 16) * 8 .. + 7.  Gathered rows:
    // the source-row indices of a thread are all loaded before any is checked, so
    // their latencies overlap.
    constexpr int kCopies = kTR / 16;
    int64_t sr[kCopies];
    bool in[kCopies];
#pragma unroll
    for (int k = 0; k < kCopies; ++k) {
        const int64_t r = r0 + ((k * 256 + tid) >> 4), c = c0 + ((k * 256 + tid) & 15) * 8;
        sr[k] = r;
        in[k] = r < p.rows && c < p.cols;
    }
    if (p.row_src != nullptr) {
        int32_t idx[kCopies];
#pragma unroll
        for (int k = 0; k < kCopies; ++k) idx[k] = in[k] ? __ldg(p.row_src + sr[k]) : -1;
#pragma unroll
        for (int k = 0; k < kCopies; ++k) {
            if (in[k] && idx[k] >= p.src_rows) {
                set_status(p.status, kStatusIndex);
                in[k] = false;
            }
            in[k] = in[k] && idx[k] >= 0;
            sr[k] = idx[k];
        }
    }
#pragma unroll
    for (int k = 0; k < kCopies; ++k) {
        const int q = k * 256 + tid;
        const int lr = q >> 4, lc = (q & 15) * 8;
        cp_async16(&tile[lr][lc], in[k] ? (const void*)(p.x + sr[k] * p.cols + c0 + lc) : (const void*)p.x,
                   in[k] ? 16u : 0u);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");

    // ---- the tensor scales (one thread computes them, the CTA shares them)
    __shared__ float sh_scales[4];  // row g, row enc, column g, column enc
    int64_t g = 0, g_row0 = 0, g_rows = p.rows;  // the group; the rows the element indices count in
    uint32_t wr, wc;
    if (kGrouped) {
        g = p.row_group ? (int64_t)p.row_group[r0 >> 7] : r0 / p.group_rows_uniform;
        g_row0 = p.row_group ? p.group_row0[g] : g * p.group_rows_uniform;
        g_rows = p.row_group ? p.group_nrows[g] : p.group_rows_uniform;
        wr = p.amax_words[2 * g];
        wc = p.col_rht ? p.amax_words[2 * g + 1] : wr;
    } else {
        wr = p.amax_words[0];
        wc = p.col_rht ? p.amax_words[1] : wr;
    }
    const bool first = tid == 0 && (kGrouped ? (r0 == g_row0 && c0 == 0) : (blockIdx.x == 0 && blockIdx.y == 0));
    if (!finite_bits(wr) || !finite_bits(wc)) {  // the same for the whole CTA
        if (first) {
            set_status(p.status, kStatusNonFinite);
            if (p.row_g) p.row_g[g] = __uint_as_float(0x7FC00000u);
            if (p.col_g) p.col_g[g] = __uint_as_float(0x7FC00000u);
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");  // let the copies land before leaving
        return;
    }
    if (tid == 0) {
        const TensorScale a = tensor_scale_from_amax(__uint_as_float(wr));
        const TensorScale b = tensor_scale_from_amax(__uint_as_float(wc));
        sh_scales[0] = a.g;
        sh_scales[1] = a.enc;
        sh_scales[2] = b.g;
        sh_scales[3] = b.enc;
        if (first) {
            if (p.row_g) p.row_g[g] = a.g;
            if (p.col_g) p.col_g[g] = b.g;
        }
    }
    uint32_t rkg[20];  // the group's Philox round keys
    if (kGrouped) {
        uint32_t k0 = (uint32_t)(p.seed + (uint64_t)g), k1 = (uint32_t)((p.seed + (uint64_t)g) >> 32);
#pragma unroll
        for (int r = 0; r < 10; ++r) {
            rkg[2 * r] = k0;
            rkg[2 * r + 1] = k1;
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
    }
    __syncthreads();
    const TensorScale tr{sh_scales[0], sh_scales[1]}, tc{sh_scales[2], sh_scales[3]};
    const uint32_t (&rkc)[20] = rkg;
    const uint32_t (&rk)[20] = kGrouped ? rkc : p.rk;
    {
        const float dec = e4m3_to_f32((uint32_t)tid);
        const float gr = __fmul_rn(dec, tr.g), gc = __fmul_rn(dec, tc.g);
        inv_tab[0][tid] = (gr == 0.0f) ? 0.0f : fminf(__frcp_rn(gr), 3.402823466e38f);
        inv_tab[1][tid] = (gc == 0.0f) ? 0.0f : fminf(__frcp_rn(gc), 3.402823466e38f);
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();  // tile and tables in shared memory

    tile_passes<k2D, kRht, kGrouped, kRowRht>(p, r0, c0, tile, inv_tab, tile_s, tile_inv, col_atom, row_atoms,
                                              tr, tc, rk, g_row0, g_rows);
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
// Standalone RHT, through the same exactly rounded transforms as the quantizer.
// axis 1: a thread transforms one 16-element chunk of a row (rht16_row).
// axis 0: a thread transforms a column pair x 16 rows (rht16_pair); consecutive
// lanes take consecutive column pairs, so loads and stores are coalesced.
// ============================================================================
__global__ void __launch_bounds__(256) rht_axis1_kernel(const uint16_t* __restrict__ x, float* __restrict__ y,
                                                       int64_t nchunks, uint32_t sign_mask) {
    const bool al32 = (reinterpret_cast<uintptr_t>(x) & 31u) == 0;
    for (int64_t ch = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; ch < nchunks;
         ch += (int64_t)gridDim.x * blockDim.x) {
        uint32_t w[8];
        ld_block16(x + ch * 16, al32, w);
        float v[16];
        rht16_row(w, sign_mask, v);
        float4* out = reinterpret_cast<float4*>(y + ch * 16);
#pragma unroll
        for (int i = 0; i < 4; ++i) out[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
}

__global__ void __launch_bounds__(256) rht_axis0_kernel(const uint16_t* __restrict__ x, float* __restrict__ y,
                                                       int64_t rows, int64_t cols, uint32_t sign_mask,
                                                       const RhtFlips flips) {
    const int64_t cpairs = cols / 2;
    const int64_t units = (rows / 16) * cpairs;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < units;
         u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r0 = (u / cpairs) * 16, c = (u % cpairs) * 2;
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t*>(x + (r0 + i) * cols + c));
        float y0[16], y1[16];
        rht16_pair(w, flips, sign_mask, y0, y1);
#pragma unroll
        for (int i = 0; i < 16; ++i) *reinterpret_cast<float2*>(y + (r0 + i) * cols + c) = make_float2(y0[i], y1[i]);
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

// The streamed kernel: whole-SM residency (two CTAs of eight warps per SM) up to
// the number of units.  The shared-memory size is set on every launch: it belongs
// to the current context, which a device reset replaces.
template <bool kGrouped, bool kGather>
static cudaError_t launch_amax_stream(const uint16_t* x, int64_t rows, int64_t cols, uint32_t sign_mask,
                                      const RhtFlips& f, uint32_t* words, const int32_t* row_group,
                                      int64_t group_rows_uniform, const int32_t* row_src, int64_t src_rows,
                                      int* status, int sm_count, cudaStream_t st) {
    const cudaError_t e = cudaFuncSetAttribute(amax_stream_kernel<kGrouped, kGather>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, kAmaxSmemBytes);
    if (e != cudaSuccess) return e;
    const int64_t units = ((rows + 15) / 16) * ((cols + kAmaxUnitCols - 1) / kAmaxUnitCols);
    const int grid = grid_for(units, kAmaxWarps, sm_count, kAmaxCtasPerSm);
    amax_stream_kernel<kGrouped, kGather><<<grid, kAmaxWarps * 32, kAmaxSmemBytes, st>>>(
        x, rows, cols, sign_mask, f, words, row_group, group_rows_uniform, row_src, src_rows, status);
    return cudaGetLastError();
}
// Bulk copies need 16-byte aligned rows.
static bool stream_ok(const uint16_t* x, int64_t cols) {
    return (reinterpret_cast<uintptr_t>(x) & 15u) == 0 && cols % 8 == 0;
}

cudaError_t launch_amax(const uint16_t* x, int64_t rows, int64_t cols, bool col_rht,
                        uint32_t sign_mask, uint32_t* words, int sm_count, cudaStream_t st,
                        bool row_rht, int* status) {
    const int64_t units = ((rows + 15) / 16) * ((cols + 255) / 256);
    const int grid = grid_for(units, 8, sm_count, 8);
    RhtFlips f;
    rht_flips(sign_mask, f);
    // The column rotation's arithmetic hides the copies best when streamed; the plain
    // max |x| is pure load throughput, where sixteen 16-byte loads per lane in flight
    // (amax_kernel) beat the two-slot stream (W 20480 x 5120: 0.148 vs 0.158 ms).  The
    // C ABI refuses rows that are not 16-byte aligned before any launch.
    if (col_rht && !row_rht) {
        if (!stream_ok(x, cols)) return cudaErrorInvalidValue;
        return launch_amax_stream<false, false>(x, rows, cols, sign_mask, f, words, nullptr, 0, nullptr, 0,
                                                status, sm_count, st);
    }
    if (row_rht && col_rht)
        amax_kernel<true, false, true><<<grid, 256, 0, st>>>(x, rows, cols, sign_mask, f, words, nullptr, 0, status);
    else if (row_rht)
        amax_kernel<false, false, true><<<grid, 256, 0, st>>>(x, rows, cols, sign_mask, f, words, nullptr, 0, status);
    else
        amax_kernel<false, false, false><<<grid, 256, 0, st>>>(x, rows, cols, sign_mask, f, words, nullptr, 0, status);
    return cudaGetLastError();
}

cudaError_t launch_amax_grouped(const QuantParams& p, int sm_count, cudaStream_t st) {
    const int64_t units = ((p.rows + 15) >> 4) * ((p.cols + 255) >> 8);
    const int grid = grid_for(units, 8, sm_count, 8);
    uint32_t* words = const_cast<uint32_t*>(p.amax_words);
    RhtFlips f;
    rht_flips(p.sign_mask, f);
    if (p.col_rht) {
        if (!stream_ok(p.x, p.cols)) return cudaErrorInvalidValue;
        if (p.row_src)
            return launch_amax_stream<true, true>(p.x, p.rows, p.cols, p.sign_mask, f, words, p.row_group,
                                                  p.group_rows_uniform, p.row_src, p.src_rows, p.status,
                                                  sm_count, st);
        return launch_amax_stream<true, false>(p.x, p.rows, p.cols, p.sign_mask, f, words, p.row_group,
                                               p.group_rows_uniform, nullptr, 0, p.status, sm_count, st);
    }
    if (p.row_src) return cudaErrorInvalidValue;  // gathered rows come with the column rotation only
    amax_kernel<false, true, false><<<grid, 256, 0, st>>>(p.x, p.rows, p.cols, p.sign_mask, f, words, p.row_group,
                                                          p.group_rows_uniform, p.status);
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
constexpr int kGroupTableThreads = 1024;  // one thread per group in the scan
static_assert(kMaxGroups <= kGroupTableThreads, "one scan thread per group");

// Largest e < n with v[e] <= x (v nondecreasing, v[0] <= x).  A group with no rows
// shares its start with the next group, so the largest index found is never an
// empty group while x lies below the total.
template <typename T>
__device__ __forceinline__ int last_at_or_below(const T* v, int n, int64_t x) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((int64_t)v[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(kGroupTableThreads)
    group_tables_kernel(GroupSizes gs, int E, int32_t* __restrict__ block_group, int64_t* __restrict__ row0,
                        int64_t* __restrict__ nrows, int64_t* __restrict__ pair_row0,
                        int32_t* __restrict__ pair_group, int32_t* __restrict__ pair_rows) {
    __shared__ int64_t start[kMaxGroups + 1];  // first row of every group; start[E] = all rows
    __shared__ int32_t tstart[kMaxGroups + 1]; // first 256-row tile of every group
    __shared__ int64_t warp_rows[32];
    __shared__ int32_t warp_tiles[32];
    const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
    // exclusive scans of the row counts and of the 256-row tile counts
    const int64_t r = e < E ? gs.rows[e] : 0;
    const int32_t t = (int32_t)((r + 255) / 256);
    int64_t ir = r;
    int32_t it = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t ur = __shfl_up_sync(0xFFFFFFFFu, ir, o);
        const int32_t ut = __shfl_up_sync(0xFFFFFFFFu, it, o);
        if (lane >= o) {
            ir += ur;
            it += ut;
        }
    }
    if (lane == 31) {
        warp_rows[warp] = ir;
        warp_tiles[warp] = it;
    }
    __syncthreads();
    if (warp == 0) {
        int64_t wr = warp_rows[lane];
        int32_t wt = warp_tiles[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t ur = __shfl_up_sync(0xFFFFFFFFu, wr, o);
            const int32_t ut = __shfl_up_sync(0xFFFFFFFFu, wt, o);
            if (lane >= o) {
                wr += ur;
                wt += ut;
            }
        }
        warp_rows[lane] = wr - warp_rows[lane];  // rows / tiles of the warps before
        warp_tiles[lane] = wt - warp_tiles[lane];
    }
    __syncthreads();
    if (e < E) {
        start[e] = warp_rows[warp] + ir - r;
        tstart[e] = warp_tiles[warp] + it - t;
        if (e == E - 1) {  // the totals
            start[E] = warp_rows[warp] + ir;
            tstart[E] = warp_tiles[warp] + it;
        }
    }
    __syncthreads();
    if (blockIdx.x == 0 && e < E) {
        row0[e] = start[e];
        nrows[e] = gs.rows[e];
    }
    // the 256-row tiles of every group: a group of 128 * odd rows ends with a tile
    // whose second half lies past the group
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    if (pair_row0) {
        for (int64_t q = (int64_t)blockIdx.x * blockDim.x + e; q < tstart[E]; q += stride) {
            const int g = last_at_or_below(tstart, E, q);
            const int64_t first = start[g] + 256 * (q - tstart[g]);
            const int64_t left = start[g + 1] - first;
            pair_row0[q] = first;
            pair_group[q] = g;
            pair_rows[q] = (int32_t)(left < 256 ? left : 256);
        }
    }
    const int64_t blocks = start[E] / 128;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + e; b < blocks; b += stride)
        block_group[b] = last_at_or_below(start, E, b * 128);
}

cudaError_t launch_group_tables(const int64_t* group_rows, int E, int32_t* block_group, int64_t* row0,
                                int64_t* nrows, cudaStream_t st, int64_t* pair_row0, int32_t* pair_group,
                                int32_t* pair_rows) {
    if (E < 1 || E > kMaxGroups) return cudaErrorInvalidValue;
    GroupSizes gs;
    memset(&gs, 0, sizeof gs);
    int64_t total = 0;
    for (int e = 0; e < E; ++e) {
        gs.rows[e] = group_rows[e];
        total += group_rows[e];
    }
    const int64_t blocks = total / 128;
    const int64_t grid = (blocks + kGroupTableThreads - 1) / kGroupTableThreads;
    group_tables_kernel<<<grid < 1 ? 1 : (grid > 16 ? 16 : (int)grid), kGroupTableThreads, 0, st>>>(
        gs, E, block_group, row0, nrows, pair_row0, pair_group, pair_rows);
    return cudaGetLastError();
}

cudaError_t launch_quant_rows(const QuantParams& params, int sm_count, cudaStream_t st) {
    QuantParams p = params;
    philox_round_keys(p.seed, p.rk);
    const int64_t nblocks = p.rows * (p.cols / 16);
    const int grid = grid_for(nblocks, 256, sm_count, 4);  // the CTAs resident at 62 registers
    quant_rows_kernel<<<grid, 256, 0, st>>>(p);
    return cudaGetLastError();
}

template <bool k2D, bool kRht, bool kGrouped, bool kRowRht>
static cudaError_t launch_tile(const QuantParams& p, int sm_count, cudaStream_t st) {
    (void)sm_count;
    if (!kGrouped && p.row_src != nullptr) return cudaErrorInvalidValue;  // gathered rows come grouped only
    const dim3 grid((unsigned)((p.cols + kTC - 1) / kTC), (unsigned)((p.rows + kTR - 1) / kTR));
    quant_tile_kernel<k2D, kRht, kGrouped, kRowRht><<<grid, 256, 0, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_quant_tile(const QuantParams& params, bool two_d, int sm_count, cudaStream_t st) {
    QuantParams p = params;
    philox_round_keys(p.seed, p.rk);
    rht_flips(p.sign_mask, p.flips);
    const bool grouped = p.row_group != nullptr || p.group_rows_uniform > 0;
    if (p.row_rht && (grouped || two_d)) return cudaErrorInvalidValue;
    const bool col_rht = p.col_rht && p.col_data;
    if (grouped) {
        if (two_d) return launch_tile<true, false, true, false>(p, sm_count, st);
        if (col_rht) return launch_tile<false, true, true, false>(p, sm_count, st);
        return launch_tile<false, false, true, false>(p, sm_count, st);
    }
    if (two_d) return launch_tile<true, false, false, false>(p, sm_count, st);
    if (p.row_rht && col_rht) return launch_tile<false, true, false, true>(p, sm_count, st);
    if (p.row_rht) return launch_tile<false, false, false, true>(p, sm_count, st);
    if (col_rht) return launch_tile<false, true, false, false>(p, sm_count, st);
    return launch_tile<false, false, false, false>(p, sm_count, st);
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
        const int64_t n = (rows / 16) * (cols / 2);
        RhtFlips f;
        rht_flips(sign_mask, f);
        rht_axis0_kernel<<<grid_for(n, 256, sm_count, 4), 256, 0, st>>>(x, y, rows, cols, sign_mask, f);
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
