/*
 * nvfp4_oracle.h -- plain, slow CPU oracle for the NVFP4 linear-layer training path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference legs may load or call this library.  It shares no code,
 * header, table or constant generator with the CUDA library, and neither includes
 * the other.
 *
 * Sources (web pages on NVFP4 training):
 *   [NVX]  "Nemotron NVFP4" explainer, ai.thesatyajit.com/articles/nemotron-nvfp4:
 *          sections "What NVFP4 actually is" (E2M1 element, FP8 E4M3 scale per 16
 *          elements, FP32 per-tensor scale, 4.5 bits/element) and "Why 4-bit training
 *          normally falls apart -- and the three fixes" (2D weight blocks, random
 *          Hadamard transform on the wgrad inputs, stochastic rounding of gradients).
 *   [ART]  "NVIDIA's 4-bit floating point pushes AI training limits", artiverse.ca:
 *          fprop/dgrad/wgrad GEMMs in NVFP4; 16x16 weight blocks vs 1x16; RHT on
 *          weight gradients; stochastic rounding on gradients only.
 *   [LTD]  "Paper of the day: What matters for NVFP4 training?", thelatentdaily.com,
 *          "Main findings" / "A methodological warning" (random sign vectors).
 *   Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as
 *          1, 2, 3", SC'11, section 4 (Philox S-box, multipliers and Weyl key schedule).
 *
 * Readings of points the pages leave open are documented at each function.
 *
 * Parity status: every function below is pinned by tests/test_oracle_*.py against
 * closed forms, exhaustive enumeration, brute force or published known-answer
 * vectors, except the two conventions listed as "parity unpinned" in
 * nvfp4_oracle.c (the FP32 op order of the block-scale computation and the sign
 * of a zero code), which the pages cannot arbitrate.
 */
#ifndef NVFP4_ORACLE_H
#define NVFP4_ORACLE_H
#include <stdint.h>
#ifdef __cplusplus
extern "C" {
#endif

/* ---- element codecs ---------------------------------------------------- */
double   ora_e2m1_decode(unsigned code);            /* 4-bit code -> value            */
unsigned ora_e2m1_encode_rne(float v);              /* nearest, ties to even, sat +-6 */
double   ora_e4m3_decode(unsigned code);            /* 8-bit code -> value (NaN 0x7F) */
unsigned ora_e4m3_encode_rne_sat(float t);          /* t >= 0 -> code in [0, 0x7E]    */
float    ora_bf16_to_f32(uint16_t b);

/* ---- Philox4x32-10 (SC'11) ---------------------------------------------- */
void ora_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);
/* 16-bit uniform draw of output element `idx` of random stream `stream`.      */
unsigned ora_sr_draw16(uint64_t seed, uint32_t stream, uint64_t idx);
/* one stochastic rounding of |v| (v finite), returns the 4-bit code          */
unsigned ora_e2m1_encode_sr(float v, unsigned r16);
/* codes[i] = SR of v[i] with the draw of element idx0 + i                      */
void ora_e2m1_sr_array(const float* v, int64_t n, uint64_t seed, uint32_t stream,
                       uint64_t idx0, uint8_t* codes);

/* ---- Hadamard ----------------------------------------------------------- */
int  ora_hadamard16(int i, int j);                  /* Sylvester H16 entry, +-1        */
/* y_j = sum_i x_i * s_i * H16[i][j] over fp64; returns 0 when exact, -1 when the
 * 16 inputs span more binades than fp64 can sum exactly (see .c)               */
int  ora_rht16(const double x[16], const int8_t s[16], double y[16]);
/* standalone transform of a bf16 matrix: 16-chunks along `axis` (1 = contiguous
 * columns, 0 = rows).  y has the same [rows][cols] layout, fp32.               */
int  ora_rht(const uint16_t* x, int64_t rows, int64_t cols, int axis,
             const int8_t signs[16], float* y);

/* ---- quantizer ----------------------------------------------------------- */
/* The tensor V that is quantized:
 *   orient 0: V = x                      ([rows][cols], blocks along cols)
 *   orient 1: V = x^T                    ([cols][rows], blocks along rows of x)
 *   orient 1 with rht: V[c][16j+t] = RHT16(x[16j..16j+15][c], signs)[t]
 *   orient 0 with rht: V[r][16j+t] = RHT16(x[r][16j..16j+15], signs)[t]    (R14)
 * amax of V as fp32 (max |V|).  Returns 0, or -1 if the RHT domain check fails. */
int   ora_tensor_amax(const uint16_t* x, int64_t rows, int64_t cols, int orient,
                      int rht, const int8_t signs[16], float* amax, int nthreads);
float ora_tensor_scale(float amax);                 /* decode scale g = amax / 2688  */
/* quantize output rows [r0, r1) of V with the given tensor amax.
 * packed: (r1-r0) x (vcols/2) bytes, low nibble = even element.
 * sf:     (r1-r0) x (vcols/16) logical E4M3 codes (16x16 mode: the tile's code in
 *         every one of its 16 rows).  For block_mode 1, r0 and r1 must be multiples
 *         of 16 (or r1 == vrows).                                                  */
int ora_quantize_rows(const uint16_t* x, int64_t rows, int64_t cols, int orient,
                      int rht, const int8_t signs[16], int block_mode, int rounding,
                      uint64_t seed, float amax, int64_t r0, int64_t r1,
                      uint8_t* packed, uint8_t* sf, int nthreads);

/* ---- scale-factor layout of the block-scaled MMA ------------------------- */
int64_t ora_sf_bytes(int64_t vrows, int64_t vcols);
int64_t ora_sf_offset(int64_t r, int64_t kb, int64_t vcols);
void    ora_sf_swizzle(const uint8_t* sf_logical, int64_t vrows, int64_t vcols,
                       uint8_t* sf_swizzled);

/* ---- GEMM over dequantized operands --------------------------------------- */
/* D[m][n] = alpha * sum_k a(m,k) * b(n,k) with a = e2m1 * e4m3(sf) decoded in fp64.
 * A: [M][K/2] packed + sfA logical [M][K/16]; B likewise with N rows.
 * Computes only the listed (m,n) pairs; bound[i] = |alpha| * sum_k |a*b|.        */
void ora_gemm_pairs(const uint8_t* A, const uint8_t* sfA, const uint8_t* B,
                    const uint8_t* sfB, int64_t K, double alpha, int64_t npairs,
                    const int64_t* m_idx, const int64_t* n_idx, double* out,
                    double* bound, int nthreads);
/* dense version: D is [M][N] */
void ora_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B,
              const uint8_t* sfB, int64_t M, int64_t N, int64_t K, double alpha,
              double* D, double* bound, int nthreads);

#ifdef __cplusplus
}
#endif
/* ---- MXFP4, the comparison format --------------------------------------- */
/* E8M0 scale 2^(e-127) (255 NaN); R15: block scale = smallest 2^k with
 * amax_b <= 6 * 2^k (e clamped to [0, 254]; all-zero block: e = 0).  Row
 * orientation, 1x32 blocks, RNE.  Scale layout: the atoms of ora_sf_swizzle over
 * 32-element blocks (call it with vcols / 2).                                   */
double   ora_e8m0_decode(unsigned code);
unsigned ora_mx_scale_code(double amax_b);
int  ora_mx_quantize_rows(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* packed,
                          uint8_t* sf);
void ora_mx_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB,
                 int64_t M, int64_t N, int64_t K, double alpha, double* D, double* bound,
                 int nthreads);

#endif
