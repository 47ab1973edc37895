/*
 * nvfp4_oracle.c -- plain, slow CPU oracle of the NVFP4 linear-layer training path.
 *
 * TEST INFRASTRUCTURE ONLY (see nvfp4_oracle.h).  Written for clarity, not speed:
 * scalar loops, brute-force nearest-value searches, an explicit 16x16 Hadamard
 * matrix product, and an fp64 dot product per GEMM output.  OpenMP only splits
 * independent rows / output elements across host threads; it never changes an
 * operation or its order within one result.
 *
 * Build: gcc -std=c11 -O2 -fno-fast-math -ffp-contract=off -fopenmp -shared -fPIC
 * so that every `float` operation below is one IEEE-754 binary32 operation with
 * round-to-nearest-even and gradual underflow (no FMA contraction, no FTZ).
 *
 * Readings of points the pages leave open (each one is the oracle's frozen spec):
 *  R1  E2M1 code = sign(bit 3) | exponent(bits 2:1, bias 1) | mantissa(bit 0);
 *      magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}.  ([NVX] "What NVFP4 actually is"
 *      fixes the 1-2-1 bit split; the value set follows from it.)
 *  R2  E4M3 = bias 7, subnormals m*2^-9, S.1111.111 = NaN, max finite 448.
 *  R3  decode scale g = amax / (6*448) in fp32; encode factor
 *      enc = 2688 / amax (fp32, clamped to FLT_MAX; 0 when amax == 0).
 *  R4  block scale (FP32 op order is a convention, "parity unpinned"):
 *        t = (amax_b / 6) * enc ; s = E4M3_rne_satfinite(t) ; d = dec(s) * g ;
 *        inv = d == 0 ? 0 : min(1 / d, FLT_MAX) ; v = x * inv
 *  R5  E2M1 round-to-nearest-even, |v| > 6 saturates to 6.
 *  R6  the code's sign bit is the sign bit of v, also when |v| rounds to zero
 *      ("parity unpinned" convention: -0 keeps its sign).
 *  R7  RHT: y = x . diag(s) . H16 with the unnormalised Sylvester H16 (H H^T = 16 I);
 *      the quantizer sees the fp32 rounding of the exact sum.
 *  R8  stochastic rounding: lo <= |v| < hi adjacent E2M1 magnitudes,
 *      p = (|v| - lo) / (hi - lo); round up iff R + floor(p * 2^16) >= 2^16, with R
 *      the element's 16-bit Philox draw (see ora_sr_draw16).  The round-up
 *      probability floor(p * 2^16) / 2^16 is within 2^-16 of p and never above it.
 *      (The B200's stochastic E2M1 conversion applies this rule to the draws it is
 *      given, which the draw layout of ora_sr_draw16 follows.)
 *  R9  amax == 0 gives g = 0, enc = 0, all scales 0 and all codes +-0.
 *  R14 RHT on both backward GEMMs ([LTD] "Main findings", the Mosaic recipe): the
 *      dgrad operands dY and W^T are rotated along N, their shared reduction axis,
 *      i.e. along the rows of the quantized view (orient 0 with rht); the dgrad
 *      alpha takes the 1/16.
 *  R15 MXFP4 ([NVX] "What NVFP4 actually is" names it: E2M1 elements, a power-of-two
 *      E8M0 scale per 32 elements, no tensor scale): the block scale is the smallest
 *      power of two 2^k with amax_b <= 6 * 2^k (nothing clipped), E8M0 code
 *      k + 127; elements round to nearest even.
 */
#include "nvfp4_oracle.h"

#include <float.h>
#include <limits.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static int ora_threads(int n) {
#ifdef _OPENMP
    return n > 0 ? n : omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* element codecs                                                            */
/* ------------------------------------------------------------------------ */

float ora_bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* R1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit; exponent 0 is
 * subnormal (m * 0.5).                                                        */
double ora_e2m1_decode(unsigned code) {
    unsigned s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
    double mag = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
    return s ? -mag : mag;
}

/* R5 + R6: brute-force nearest magnitude among the 8 codes; on an exact tie the
 * code with mantissa bit 0 (an even code) wins, which is round-half-to-even.
 * Magnitudes of 6 and above saturate to 6 (checked first: for huge |v| every
 * fp64 distance below would round to the same value).                         */
unsigned ora_e2m1_encode_rne(float v) {
    unsigned sign = signbit(v) ? 8u : 0u;
    double a = fabs((double)v);
    if (a >= 6.0) return sign | 7u; /* satfinite: everything above 6 is 6 */
    unsigned best = 0;
    double bestd = a;
    for (unsigned c = 1; c < 8; ++c) {
        double d = fabs(a - ora_e2m1_decode(c));
        if (d < bestd || (d == bestd && (c & 1u) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return sign | best;
}

/* R2: E4M3 with bias 7.  (1 + m/8) * 2^(e-7) == (8 + m) * 2^(e-10).            */
double ora_e4m3_decode(unsigned code) {
    unsigned s = (code >> 7) & 1u, e = (code >> 3) & 15u, m = code & 7u;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ldexp((double)m, -9) : ldexp(8.0 + (double)m, (int)e - 10);
    return s ? -mag : mag;
}

/* R2 + R4: round-to-nearest-even onto the non-negative finite E4M3 codes,
 * saturating (satfinite) at 448 = code 0x7E.  Brute force over all 127 codes.  */
unsigned ora_e4m3_encode_rne_sat(float t) {
    double a = (double)t;
    if (!(a >= 0.0)) return 0; /* negative or NaN never reach here (amax >= 0) */
    if (a >= 448.0) return 0x7E;
    unsigned best = 0;
    double bestd = a;
    for (unsigned c = 1; c <= 0x7E; ++c) {
        double d = fabs(a - ora_e4m3_decode(c));
        if (d < bestd || (d == bestd && (c & 1u) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return best;
}

/* ------------------------------------------------------------------------ */
/* Philox4x32-10, Salmon et al. SC'11 section 4                              */
/* ------------------------------------------------------------------------ */

/* One Philox round: two 32x32->64 multiplications, the high halves xor-ed with
 * the other two counter words and the round key; words are permuted.          */
static void ora_philox_round(uint32_t c[4], const uint32_t k[2]) {
    const uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)c[0];
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)c[2];
    const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c[1] ^ k[0];
    uint32_t n2 = hi0 ^ c[3] ^ k[1];
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
}

void ora_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
    uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
    uint32_t k[2] = {key[0], key[1]};
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { /* Weyl key schedule: golden ratio and sqrt(3)-1 */
            k[0] += 0x9E3779B9u;
            k[1] += 0xBB67AE85u;
        }
        ora_philox_round(c, k);
    }
    out[0] = c[0];
    out[1] = c[1];
    out[2] = c[2];
    out[3] = c[3];
}

/* R8: element `idx` (row-major index in the quantized tensor V) takes 16 bits of
 * the Philox block with counter (idx>>3 low, idx>>3 high, stream, 0) and key
 * (seed low, seed high).  With j = idx & 7, the block's words pair the elements
 * (0,2), (1,3), (4,6), (5,7): element j reads word (j & 1) + 2 * (j >> 2); the
 * first element of a pair (bit 1 of j clear) takes bytes 2 (high) and 0 (low) of
 * that word, the second bytes 3 (high) and 1 (low).  Every bit of the block serves
 * exactly one element.                                                          */
unsigned ora_sr_draw16(uint64_t seed, uint32_t stream, uint64_t idx) {
    uint64_t g = idx >> 3;
    uint32_t ctr[4] = {(uint32_t)g, (uint32_t)(g >> 32), stream, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t w[4];
    ora_philox4x32_10(ctr, key, w);
    unsigned j = (unsigned)(idx & 7u);
    uint32_t word = w[(j & 1u) + 2u * (j >> 2)];
    unsigned h = (j >> 1) & 1u;
    unsigned byte_lo = (word >> (8u * h)) & 0xFFu;
    unsigned byte_hi = (word >> (8u * (2u + h))) & 0xFFu;
    return (byte_hi << 8) | byte_lo;
}

/* R8: stochastic rounding onto the E2M1 grid.  p = (|v| - lo) / (hi - lo) is exact
 * in fp64 (|v| is a float, lo and hi are grid points); the element rounds up iff
 * its draw R (uniform in [0, 65536)) satisfies R + floor(p * 65536) >= 65536, so
 * floor(p * 65536) of the 65536 draws round up.                                */
unsigned ora_e2m1_encode_sr(float v, unsigned r16) {
    unsigned sign = signbit(v) ? 8u : 0u;
    double a = fabs((double)v);
    if (a >= 6.0) return sign | 7u;
    unsigned c = 0;
    while (c < 7 && ora_e2m1_decode(c + 1) <= a) ++c;
    double lo = ora_e2m1_decode(c), hi = ora_e2m1_decode(c + 1);
    double p = (a - lo) / (hi - lo);
    double t = floor(p * 65536.0);
    unsigned up = ((double)r16 + t >= 65536.0) ? 1u : 0u;
    return sign | (c + up);
}

void ora_e2m1_sr_array(const float* v, int64_t n, uint64_t seed, uint32_t stream,
                       uint64_t idx0, uint8_t* codes) {
    for (int64_t i = 0; i < n; ++i)
        codes[i] = (uint8_t)ora_e2m1_encode_sr(v[i], ora_sr_draw16(seed, stream, idx0 + (uint64_t)i));
}

/* ------------------------------------------------------------------------ */
/* Random Hadamard transform ([NVX] "the three fixes"; [ART])                */
/* ------------------------------------------------------------------------ */

/* Sylvester construction H_{2n} = [[H, H], [H, -H]]: entry (i, j) is -1 exactly
 * when i and j share an odd number of set bits.                               */
int ora_hadamard16(int i, int j) {
    return (__builtin_popcount((unsigned)(i & j)) & 1) ? -1 : 1;
}

/* R7: explicit matrix product in fp64.  The 16 inputs are bf16 values (8
 * significant bits); every partial sum is exact in fp64 while the nonzero
 * inputs' exponents span at most 41 binades (8 + 4 + 41 <= 53 bits), which the
 * function reports; then the caller's (float) cast is the correctly rounded
 * fp32 value of the exact sum.                                                */
int ora_rht16(const double x[16], const int8_t s[16], double y[16]) {
    int emin = INT_MAX, emax = INT_MIN;
    for (int i = 0; i < 16; ++i) {
        if (x[i] != 0.0 && isfinite(x[i])) {
            int e = ilogb(x[i]);
            if (e < emin) emin = e;
            if (e > emax) emax = e;
        }
    }
    for (int j = 0; j < 16; ++j) {
        double acc = 0.0;
        for (int i = 0; i < 16; ++i) acc += x[i] * (double)s[i] * (double)ora_hadamard16(i, j);
        y[j] = acc;
    }
    return (emax != INT_MIN && emax - emin > 41) ? -1 : 0;
}

int ora_rht(const uint16_t* x, int64_t rows, int64_t cols, int axis,
            const int8_t signs[16], float* y) {
    int64_t len = axis == 1 ? cols : rows;
    if (len % 16 != 0) return -2;
    int bad = 0;
    int64_t nchunks = (axis == 1) ? rows * (cols / 16) : (rows / 16) * cols;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t ch = 0; ch < nchunks; ++ch) {
        double in[16], out[16];
        int64_t base_r, base_c, step_r, step_c;
        if (axis == 1) {
            base_r = ch / (cols / 16);
            base_c = (ch % (cols / 16)) * 16;
            step_r = 0;
            step_c = 1;
        } else {
            base_r = (ch / cols) * 16;
            base_c = ch % cols;
            step_r = 1;
            step_c = 0;
        }
        for (int i = 0; i < 16; ++i)
            in[i] = ora_bf16_to_f32(x[(base_r + i * step_r) * cols + base_c + i * step_c]);
        if (ora_rht16(in, signs, out) != 0) bad = 1;
        for (int j = 0; j < 16; ++j)
            y[(base_r + j * step_r) * cols + base_c + j * step_c] = (float)out[j];
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------ */
/* the tensor that gets quantized                                            */
/* ------------------------------------------------------------------------ */

/* Materialise row `vr` of V (length vcols, fp32).  Returns -1 if an RHT chunk
 * falls outside the exact domain of ora_rht16.                                */
static int ora_v_row(const uint16_t* x, int64_t rows, int64_t cols, int orient, int rht,
                     const int8_t signs[16], int64_t vr, float* out) {
    if (orient == 0 && !rht) {
        for (int64_t c = 0; c < cols; ++c) out[c] = ora_bf16_to_f32(x[vr * cols + c]);
        return 0;
    }
    if (orient == 0) {
        /* R14: the rotation along the row (dgrad operands rotated along N) */
        int bad = 0;
        for (int64_t j = 0; j < cols / 16; ++j) {
            double in[16], y[16];
            for (int i = 0; i < 16; ++i) in[i] = ora_bf16_to_f32(x[vr * cols + 16 * j + i]);
            if (ora_rht16(in, signs, y) != 0) bad = 1;
            for (int t = 0; t < 16; ++t) out[16 * j + t] = (float)y[t];
        }
        return bad ? -1 : 0;
    }
    /* orient 1: V row vr is column vr of x, blocks along the rows of x */
    if (!rht) {
        for (int64_t r = 0; r < rows; ++r) out[r] = ora_bf16_to_f32(x[r * cols + vr]);
        return 0;
    }
    int bad = 0;
    for (int64_t j = 0; j < rows / 16; ++j) {
        double in[16], y[16];
        for (int i = 0; i < 16; ++i) in[i] = ora_bf16_to_f32(x[(16 * j + i) * cols + vr]);
        if (ora_rht16(in, signs, y) != 0) bad = 1;
        for (int t = 0; t < 16; ++t) out[16 * j + t] = (float)y[t];
    }
    return bad ? -1 : 0;
}

int ora_tensor_amax(const uint16_t* x, int64_t rows, int64_t cols, int orient, int rht,
                    const int8_t signs[16], float* amax, int nthreads) {
    if (rht && (orient ? rows : cols) % 16 != 0) return -2;
    int64_t vrows = orient ? cols : rows, vcols = orient ? rows : cols;
    float m = 0.0f;
    int bad = 0;
    if (!rht) {
        /* the same set of elements either way */
#pragma omp parallel for num_threads(ora_threads(nthreads)) reduction(max : m)
        for (int64_t i = 0; i < rows * cols; ++i) {
            float a = fabsf(ora_bf16_to_f32(x[i]));
            if (isnan(a)) a = INFINITY;
            if (a > m) m = a;
        }
    } else {
#pragma omp parallel num_threads(ora_threads(nthreads)) reduction(max : m) reduction(| : bad)
        {
            float* row = (float*)malloc(sizeof(float) * (size_t)vcols);
#pragma omp for schedule(static)
            for (int64_t vr = 0; vr < vrows; ++vr) {
                if (ora_v_row(x, rows, cols, orient, rht, signs, vr, row) != 0) bad = 1;
                for (int64_t c = 0; c < vcols; ++c) {
                    float a = fabsf(row[c]);
                    if (isnan(a)) a = INFINITY;
                    if (a > m) m = a;
                }
            }
            free(row);
        }
    }
    *amax = m;
    return bad ? -1 : 0;
}

/* R3 */
float ora_tensor_scale(float amax) { return amax / 2688.0f; }

static float ora_encode_factor(float amax) {
    if (amax == 0.0f) return 0.0f;
    float e = 2688.0f / amax;
    return (e > FLT_MAX) ? FLT_MAX : e;
}

/* R4: scale code and per-element multiplier of one block */
static void ora_block_scale(float amax_b, float enc, float g, unsigned* s_out, float* inv_out) {
    float t = (amax_b / 6.0f) * enc;
    unsigned s = ora_e4m3_encode_rne_sat(t);
    float d = (float)ora_e4m3_decode(s) * g;
    float inv = 0.0f;
    if (d != 0.0f) {
        inv = 1.0f / d;
        if (inv > FLT_MAX) inv = FLT_MAX;
    }
    *s_out = s;
    *inv_out = inv;
}

int ora_quantize_rows(const uint16_t* x, int64_t rows, int64_t cols, int orient, int rht,
                      const int8_t signs[16], int block_mode, int rounding, uint64_t seed,
                      float amax, int64_t r0, int64_t r1, uint8_t* packed, uint8_t* sf,
                      int nthreads) {
    const int64_t vrows = orient ? cols : rows, vcols = orient ? rows : cols;
    if (vcols % 16 != 0) return -2;
    if (block_mode == 1 && (vrows % 16 != 0 || r0 % 16 != 0 || r1 % 16 != 0)) return -2;
    if (r0 < 0 || r1 > vrows || r0 > r1) return -2;
    if (!isfinite(amax)) return -3;
    const float g = ora_tensor_scale(amax);
    const float enc = ora_encode_factor(amax);
    const int64_t nkb = vcols / 16;
    const int64_t group = block_mode == 1 ? 16 : 1;
    const uint32_t stream = (uint32_t)orient;
    int bad = 0;
#pragma omp parallel num_threads(ora_threads(nthreads)) reduction(| : bad)
    {
        float* v = (float*)malloc(sizeof(float) * (size_t)(vcols * group));
#pragma omp for schedule(dynamic, 1)
        for (int64_t gr = r0; gr < r1; gr += group) {
            int64_t nr = (gr + group <= r1) ? group : (r1 - gr);
            for (int64_t i = 0; i < nr; ++i)
                if (ora_v_row(x, rows, cols, orient, rht, signs, gr + i, v + i * vcols) != 0)
                    bad = 1;
            for (int64_t b = 0; b < nkb; ++b) {
                unsigned s = 0;
                float inv = 0.0f;
                if (block_mode == 1) {
                    /* one scale for the 16x16 tile ([ART]: 16x16 weight blocks) */
                    float amax_b = 0.0f;
                    for (int64_t i = 0; i < 16; ++i)
                        for (int64_t c = 0; c < 16; ++c) {
                            float a = fabsf(v[i * vcols + 16 * b + c]);
                            if (a > amax_b) amax_b = a;
                        }
                    ora_block_scale(amax_b, enc, g, &s, &inv);
                }
                for (int64_t i = 0; i < nr; ++i) {
                    const float* vb = v + i * vcols + 16 * b;
                    if (block_mode == 0) {
                        /* 1x16 strip along the reduction axis ([NVX]) */
                        float amax_b = 0.0f;
                        for (int c = 0; c < 16; ++c) {
                            float a = fabsf(vb[c]);
                            if (a > amax_b) amax_b = a;
                        }
                        ora_block_scale(amax_b, enc, g, &s, &inv);
                    }
                    const int64_t vr = gr + i;
                    for (int c = 0; c < 16; ++c) {
                        float q = vb[c] * inv;
                        unsigned code;
                        if (rounding == 1) {
                            uint64_t idx = (uint64_t)vr * (uint64_t)vcols + (uint64_t)(16 * b + c);
                            code = ora_e2m1_encode_sr(q, ora_sr_draw16(seed, stream, idx));
                        } else {
                            code = ora_e2m1_encode_rne(q);
                        }
                        int64_t byte = (vr - r0) * (vcols / 2) + (16 * b + c) / 2;
                        if ((c & 1) == 0)
                            packed[byte] = (uint8_t)code;
                        else
                            packed[byte] = (uint8_t)(packed[byte] | (code << 4));
                    }
                    sf[(vr - r0) * nkb + b] = (uint8_t)s;
                }
            }
        }
        free(v);
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------ */
/* scale-factor layout                                                        */
/* ------------------------------------------------------------------------ */
/* The block-scaled MMA reads scale factors in 512-byte atoms covering 128 rows x
 * 4 consecutive 16-element blocks: inside an atom, row r and block kb sit at
 * (r % 32) * 16 + (r / 32) * 4 + kb; atoms advance along the reduction axis
 * first, then by 128-row groups.  Rows pad to 128 and blocks to 4 with zeros.  */
static int64_t ora_pad(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

int64_t ora_sf_bytes(int64_t vrows, int64_t vcols) {
    return ora_pad(vrows, 128) * ora_pad(vcols / 16, 4);
}

int64_t ora_sf_offset(int64_t r, int64_t kb, int64_t vcols) {
    int64_t katoms = ora_pad(vcols / 16, 4) / 4;
    int64_t atom = (r / 128) * katoms + kb / 4;
    int64_t rr = r % 128;
    return atom * 512 + (rr % 32) * 16 + (rr / 32) * 4 + (kb % 4);
}

void ora_sf_swizzle(const uint8_t* sf_logical, int64_t vrows, int64_t vcols,
                    uint8_t* sf_swizzled) {
    int64_t nkb = vcols / 16;
    memset(sf_swizzled, 0, (size_t)ora_sf_bytes(vrows, vcols));
    for (int64_t r = 0; r < vrows; ++r)
        for (int64_t kb = 0; kb < nkb; ++kb)
            sf_swizzled[ora_sf_offset(r, kb, vcols)] = sf_logical[r * nkb + kb];
}

/* ------------------------------------------------------------------------ */
/* block-scaled GEMM over dequantized operands ([ART]: fprop/dgrad/wgrad)    */
/* ------------------------------------------------------------------------ */

static double ora_deq(const uint8_t* P, const uint8_t* sf, int64_t row, int64_t k, int64_t K) {
    uint8_t byte = P[row * (K / 2) + k / 2];
    unsigned code = (k & 1) ? (byte >> 4) : (byte & 15u);
    return ora_e2m1_decode(code) * ora_e4m3_decode(sf[row * (K / 16) + k / 16]);
}

static void ora_dot(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB,
                    int64_t K, double alpha, int64_t m, int64_t n, double* out, double* bound) {
    double acc = 0.0, mag = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        double p = ora_deq(A, sfA, m, k, K) * ora_deq(B, sfB, n, k, K);
        acc += p;
        mag += fabs(p);
    }
    *out = alpha * acc;
    *bound = fabs(alpha) * mag;
}

void ora_gemm_pairs(const uint8_t* A, const uint8_t* sfA, const uint8_t* B,
                    const uint8_t* sfB, int64_t K, double alpha, int64_t npairs,
                    const int64_t* m_idx, const int64_t* n_idx, double* out,
                    double* bound, int nthreads) {
#pragma omp parallel for num_threads(ora_threads(nthreads)) schedule(dynamic, 16)
    for (int64_t i = 0; i < npairs; ++i)
        ora_dot(A, sfA, B, sfB, K, alpha, m_idx[i], n_idx[i], &out[i], &bound[i]);
}

void ora_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB,
              int64_t M, int64_t N, int64_t K, double alpha, double* D, double* bound,
              int nthreads) {
#pragma omp parallel for num_threads(ora_threads(nthreads)) schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            ora_dot(A, sfA, B, sfB, K, alpha, m, n, &D[m * N + n], &bound[m * N + n]);
}

/* ------------------------------------------------------------------------ */
/* MXFP4, the comparison format ([NVX] "What NVFP4 actually is": E2M1 elements,  */
/* one power-of-two E8M0 scale per 32-element block, 4.25 bits per element)     */
/* ------------------------------------------------------------------------ */

/* E8M0: value 2^(e - 127) for e in 0..254; 255 is NaN. */
double ora_e8m0_decode(unsigned code) {
    code &= 0xFFu;
    if (code == 255u) return NAN;
    return ldexp(1.0, (int)code - 127);
}

/* R15: the block scale is the smallest power of two 2^k with amax_b <= 6 * 2^k,
 * so no element is clipped; e = k + 127 clamped to [0, 254] (an all-zero block
 * takes e = 0).  Found by brute force over k.                                  */
unsigned ora_mx_scale_code(double amax_b) {
    if (!(amax_b > 0.0)) return 0u;
    for (int k = -127; k <= 127; ++k)
        if (amax_b <= 6.0 * ldexp(1.0, k)) {
            int e = k + 127;
            return (unsigned)(e < 0 ? 0 : (e > 254 ? 254 : e));
        }
    return 254u;
}

/* Row orientation, 1x32 blocks along the columns, round-to-nearest-even: each
 * element is x / 2^(e - 127) (exact in fp64) encoded to E2M1.  packed: rows x
 * cols/2 bytes (low nibble = even element); sf: rows x cols/32 logical codes.   */
int ora_mx_quantize_rows(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* packed,
                         uint8_t* sf) {
    if (cols % 32 != 0) return -2;
    const int64_t nkb = cols / 32;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t kb = 0; kb < nkb; ++kb) {
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) {
                double a = fabs((double)ora_bf16_to_f32(x[r * cols + kb * 32 + i]));
                if (isnan(a)) return -3;
                if (a > amax) amax = a;
            }
            if (isinf(amax)) return -3;
            const unsigned e = ora_mx_scale_code(amax);
            sf[r * nkb + kb] = (uint8_t)e;
            const double scale = ora_e8m0_decode(e);
            for (int i = 0; i < 32; ++i) {
                const int64_t c = kb * 32 + i;
                const double v = (double)ora_bf16_to_f32(x[r * cols + c]) / scale;
                const unsigned code = ora_e2m1_encode_rne(v);
                uint8_t* byte = &packed[r * (cols / 2) + c / 2];
                if (c & 1)
                    *byte = (uint8_t)((*byte & 0x0Fu) | (code << 4));
                else
                    *byte = (uint8_t)((*byte & 0xF0u) | code);
            }
        }
    }
    return 0;
}

/* D[m][n] = alpha * sum_k a(m,k) * b(n,k), a = e2m1 * 2^(e - 127) per 32-block,
 * in fp64 (every product exact); bound = |alpha| * sum |a * b|.                */
static double ora_mx_deq(const uint8_t* P, const uint8_t* sf, int64_t row, int64_t k, int64_t K) {
    uint8_t byte = P[row * (K / 2) + k / 2];
    unsigned code = (k & 1) ? (byte >> 4) : (byte & 15u);
    return ora_e2m1_decode(code) * ora_e8m0_decode(sf[row * (K / 32) + k / 32]);
}

void ora_mx_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB,
                 int64_t M, int64_t N, int64_t K, double alpha, double* D, double* bound,
                 int nthreads) {
#pragma omp parallel for num_threads(ora_threads(nthreads)) schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = ora_mx_deq(A, sfA, m, k, K) * ora_mx_deq(B, sfB, n, k, K);
                acc += p;
                mag += fabs(p);
            }
            D[m * N + n] = alpha * acc;
            bound[m * N + n] = fabs(alpha) * mag;
        }
}
