/*
 * nvfp4.h -- C ABI of libnvfp4.so, the B200 (sm_100a) NVFP4 linear-layer training path.
 *
 * What the library computes (web pages on NVFP4 training):
 *  - NVFP4: E2M1 4-bit elements, one E4M3 scale per 16 elements and one FP32 scale
 *    per tensor, 4.5 bits per element ("Nemotron NVFP4" explainer,
 *    ai.thesatyajit.com, "What NVFP4 actually is").
 *  - 1x16 blocks for activations and gradients, 16x16 blocks for weights;
 *    round-to-nearest-even, stochastic rounding for gradients only; a random
 *    Hadamard transform on the weight-gradient GEMM inputs; fprop, dgrad and
 *    wgrad GEMMs in NVFP4 ("NVIDIA's 4-bit floating point pushes AI training
 *    limits", artiverse.ca; explainer, "Why 4-bit training normally falls apart --
 *    and the three fixes").
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library never
 *    allocates device memory.  Host pointers are marked "host".
 *  - bf16 tensors are row-major [rows][cols] (cols contiguous), 16-byte aligned.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default).
 *    Argument errors are detected on the host before anything is launched and
 *    returned as a negative nvfp4_status; nothing is written in that case.
 *  - Errors found on the device (non-finite input, a bounded wait that ran out)
 *    are recorded in a status word in the caller's workspace; read it with
 *    nvfp4_read_status() (which synchronizes the stream).
 *  - No entry point traps, asserts on the device or throws across the ABI.
 *  - A tensor quantized in both orientations or in 16x16 blocks (nvfp4_quantize_2d,
 *    16x16 nvfp4_quantize, the linear and expert-layer calls) has at most
 *    4,194,240 rows (65535 tiles of 64); larger ones return NVFP4_ERR_SHAPE.
 *
 * Numerics (fixed readings of points the pages leave open):
 *  - decode scale g = amax / (6 * 448) (fp32), encode factor 2688 / amax.
 *  - block scale s = E4M3_rne_satfinite((amax_b / 6) * enc); element
 *    v = x * (1 / (dec(s) * g)) rounded to E2M1 (RNE, or stochastic: with p the
 *    position of |v| between its two grid neighbours, v rounds up iff
 *    R + floor(p * 2^16) >= 2^16, R the element's 16-bit draw from the
 *    Philox4x32-10 block of counter (e/8 low, e/8 high, stream, 0) and key seed,
 *    e the element's row-major index; the block's words serve the element pairs
 *    (0,2), (1,3), (4,6), (5,7) of its 8 elements, the first of a pair taking
 *    bytes 2:0 of its word and the second bytes 3:1).
 *  - scales are stored in the block-scaled MMA layout: 512-byte atoms of
 *    128 rows x 4 blocks, rows padded to 128 and blocks to 4 with zeros.
 *  - packed codes: [rows][cols/2] bytes, element 2j in the low nibble.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* nvfp4_stream_t; /* identical to cudaStream_t */

typedef enum nvfp4_status {
    NVFP4_OK = 0,
    NVFP4_ERR_ARG = -1,       /* null pointer, bad enum value, bad sign vector      */
    NVFP4_ERR_SHAPE = -2,     /* a size is not a multiple the operation needs       */
    NVFP4_ERR_ALIGN = -3,     /* a pointer is not 16-byte aligned                   */
    NVFP4_ERR_CUDA = -4,      /* a CUDA runtime call or launch failed               */
    NVFP4_ERR_NONFINITE = -5, /* device status: the input held Inf or NaN           */
    NVFP4_ERR_TIMEOUT = -6,   /* device status: a bounded wait in a kernel ran out  */
    NVFP4_ERR_WORKSPACE = -7, /* workspace pointer null or smaller than required    */
    NVFP4_ERR_DEVICE = -8,    /* the current device is not sm_100 (B200 class)      */
    NVFP4_ERR_INDEX = -9,     /* a row index lies outside its source tensor (device) */
    NVFP4_ERR_RHT_RANGE = -10 /* a rotated 16-chunk's inputs span more than 41 binades
                                 (device): the outputs were still written, but that
                                 chunk's transform is the fp64 rounding of its sum,
                                 not the correctly rounded exact sum                  */
} nvfp4_status;

enum { NVFP4_BLOCK_1X16 = 0, NVFP4_BLOCK_16X16 = 1 };
enum { NVFP4_ROUND_RNE = 0, NVFP4_ROUND_SR = 1 };

/* One quantized operand as the GEMM reads it (reduction axis = cols). */
typedef struct nvfp4_tensor {
    uint8_t* data;        /* E2M1 codes, nvfp4_packed_bytes(rows, cols) bytes        */
    uint8_t* scales;      /* E4M3 block scales, nvfp4_scale_bytes(rows, cols) bytes   */
    float* tensor_scale;  /* one fp32: the decode scale g                            */
    int64_t rows;
    int64_t cols;
} nvfp4_tensor;

/* Sizes (bytes).  packed = rows*cols/2; scales = pad128(rows) * pad4(cols/16). */
size_t nvfp4_packed_bytes(int64_t rows, int64_t cols);
size_t nvfp4_scale_bytes(int64_t rows, int64_t cols);
/* Scratch of nvfp4_quantize / nvfp4_quantize_2d (tensor amax words + status). */
size_t nvfp4_quantize_workspace_bytes(void);

/*
 * nvfp4_quantize -- quantize a bf16 tensor along its rows (blocks run along cols).
 * Defines: the two-level NVFP4 encoding of the explainer's "What NVFP4 actually
 * is"; 1x16 strips ("activations and gradients") or 16x16 tiles ("weights",
 * artiverse.ca).
 *   x            [rows][cols] bf16.  cols % 16 == 0; 16x16 also needs rows % 16 == 0.
 *   block_mode   NVFP4_BLOCK_1X16 or NVFP4_BLOCK_16X16.
 *   rounding     NVFP4_ROUND_RNE or NVFP4_ROUND_SR (Philox stream 0, key = seed).
 *   packed       out, nvfp4_packed_bytes(rows, cols) bytes.
 *   scales       out, nvfp4_scale_bytes(rows, cols) bytes (padding written as 0).
 *   tensor_scale out, one float: g = amax / 2688 (NaN if x held Inf/NaN).
 *   workspace    nvfp4_quantize_workspace_bytes() bytes of device scratch; its status
 *                word reports NVFP4_ERR_NONFINITE (see nvfp4_read_status).
 * Launches: one amax pass and one quantize pass (two reads of x).
 */
int nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int block_mode, int rounding,
                   uint64_t seed, uint8_t* packed, uint8_t* scales, float* tensor_scale,
                   void* workspace, nvfp4_stream_t stream);

/*
 * nvfp4_quantize_2d -- one read of x, up to two quantized orientations.
 * Defines: the row orientation as nvfp4_quantize; the column orientation quantizes
 * x^T (blocks run down the rows of x), optionally after the 16-point random
 * Hadamard transform along the rows ("Random Hadamard transform on the wgrad
 * inputs", explainer).  With 16x16 blocks both orientations share the tile scales,
 * so their codes are exact transposes ("consistency between forward and backward",
 * artiverse.ca).
 *   row_out  nullable; rows x cols operand (data, scales, tensor_scale filled).
 *   col_out  nullable; cols x rows operand.  Needs rows % 16 == 0.
 *   opts     host struct below; rht_signs is a HOST array of 16 entries, each +1/-1.
 * The column orientation draws from Philox stream 1, the row orientation stream 0.
 */
typedef struct nvfp4_quantize_opts {
    int block_mode;          /* NVFP4_BLOCK_1X16 / NVFP4_BLOCK_16X16                 */
    int row_rounding;        /* NVFP4_ROUND_RNE / NVFP4_ROUND_SR                      */
    int col_rounding;        /* NVFP4_ROUND_RNE / NVFP4_ROUND_SR                      */
    uint64_t seed;           /* Philox key for stochastic rounding                    */
    int col_rht;             /* 1: transform the column orientation (1x16 only)       */
    const int8_t* rht_signs; /* host, 16 x (+1|-1); required when col_rht == 1         */
} nvfp4_quantize_opts;
int nvfp4_quantize_2d(const void* x, int64_t rows, int64_t cols, const nvfp4_quantize_opts* opts,
                      nvfp4_tensor* row_out, nvfp4_tensor* col_out, void* workspace,
                      nvfp4_stream_t stream);

/*
 * nvfp4_rht -- standalone 16-point random Hadamard transform, fp32 output.
 * Defines: y = x . diag(signs) . H16 on every 16-element chunk along `axis`, with
 * the unnormalised Sylvester H16 (H16 H16^T = 16 I), so the transform is undone
 * analytically by dividing the wgrad product by 16 (explainer, "the three fixes").
 *   x      [rows][cols] bf16;  y  [rows][cols] fp32 (same layout).
 *   axis   1: chunks along cols (cols % 16 == 0);  0: chunks along rows (rows % 16 == 0).
 *   signs  HOST array of n entries, each +1 or -1;  n must be 16.
 * Each output is the fp32 rounding of the exact sum (exact when the 16 inputs'
 * exponents span at most 41 binades).
 */
int nvfp4_rht(const void* x, int64_t rows, int64_t cols, int axis, const int8_t* signs, int n,
              float* y, nvfp4_stream_t stream);

/*
 * nvfp4_gemm -- block-scaled FP4 GEMM with fp32 accumulation.
 * Defines: D[m][n] = alpha * gA * gB * sum_k a[m][k] * b[n][k], a and b the decoded
 * E2M1 x E4M3 values (fprop, dgrad and wgrad all have this form; artiverse.ca).
 *   A, sfA     M x K operand (codes, swizzled scales).   B, sfB   N x K operand.
 *   scale_a/b  device pointers to the tensor scales gA, gB (nullable: 1.0).
 *   alpha      host multiplier (1/16 for the RHT-rotated wgrad).
 *   D_bf16     nullable; [M][N] bf16, rounded to nearest even from the fp32 value.
 *   D_f32      nullable; [M][N] fp32 (the value before the bf16 rounding).
 *   status     nullable device int; set to NVFP4_ERR_TIMEOUT if a pipeline wait ran
 *              out (the output is then incomplete).
 * Needs K % 64 == 0, N % 8 == 0, at least one of D_bf16 / D_f32, 16-byte alignment.
 */
int nvfp4_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB,
               const float* scale_a, const float* scale_b, float alpha, int64_t M, int64_t N,
               int64_t K, void* D_bf16, float* D_f32, int* status, nvfp4_stream_t stream);

/*
 * nvfp4_gemm_wait_limit -- nvfp4_gemm with the pipeline waits' bound set by the
 * caller instead of the default 2^31 clock cycles (about a second): a testing hook
 * for the failure path, not a computation of the pages.  With a bound of a few
 * cycles the waits run out in normal operation; the kernel then records
 * NVFP4_ERR_TIMEOUT in *status, stops issuing work, waits (with the default bound)
 * for the copies and MMAs it already issued, frees its tensor memory and returns,
 * and D is incomplete.  wait_cycles >= 0 (0 selects the default); other arguments
 * as nvfp4_gemm.
 */
int nvfp4_gemm_wait_limit(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB,
                          const float* scale_a, const float* scale_b, float alpha, int64_t M,
                          int64_t N, int64_t K, void* D_bf16, float* D_f32, int* status,
                          long long wait_cycles, nvfp4_stream_t stream);

/*
 * Linear layer Y = X W^T in NVFP4 (artiverse.ca: forward, backward and weight-gradient
 * GEMMs in 4 bits; 16x16 weight blocks; RHT on the weight-gradient inputs; stochastic
 * rounding on gradients only).
 *   X [M][K], W [N][K], Y [M][N], dY [M][N], dX [M][K], dW [N][K]; all bf16.
 *   M, K and N multiples of 64 (each is the reduction axis of one of the GEMMs).
 *   ws / ws_bytes  device workspace of nvfp4_linear_workspace_bytes(M, K, N) bytes.
 *                  It holds the quantized operands between the three calls.
 *   rht_signs      HOST array of 16 x (+1|-1); the same vector must be passed to
 *                  fprop, dgrad and wgrad of one step.
 * fprop: quantizes X (rows RNE + columns RHT RNE, one read) and W (16x16, both
 *        orientations, one read); Y = X W^T.
 * dgrad: quantizes dY (rows SR stream 0 + columns RHT SR stream 1, one read);
 *        dX = dY W.
 * wgrad: dW = (dY^T D H)(X^T D H)^T / 16.  dY nullable: NULL reuses the quantized dY
 *        that dgrad left in ws; non-NULL quantizes dY's columns here.
 */
size_t nvfp4_linear_workspace_bytes(int64_t M, int64_t K, int64_t N);
int nvfp4_linear_fprop(const void* X, const void* W, void* Y, int64_t M, int64_t K, int64_t N,
                       const int8_t* rht_signs, void* ws, size_t ws_bytes, nvfp4_stream_t stream);
int nvfp4_linear_dgrad(const void* dY, void* dX, int64_t M, int64_t K, int64_t N, uint64_t seed,
                       const int8_t* rht_signs, void* ws, size_t ws_bytes, nvfp4_stream_t stream);
int nvfp4_linear_wgrad(const void* dY, void* dW, int64_t M, int64_t K, int64_t N, uint64_t seed,
                       const int8_t* rht_signs, void* ws, size_t ws_bytes, nvfp4_stream_t stream);

/*
 * Mixture-of-experts expert layer in NVFP4.  Only the expert weight-GEMMs run in FP4
 * in the models the pages describe ("Nemotron NVFP4" explainer, "The model underneath"
 * and "The honest part"); each expert is a linear layer with its own tensor scales and
 * the same recipe as above.
 *   Token rows are permuted into expert-contiguous segments: expert e owns rows
 *   [off_e, off_e + group_rows[e]) of the permuted buffers (off_e = prefix sum), with
 *   group_rows[e] a multiple of 64 (the routed tokens followed by zero rows).
 *   group_rows: HOST array of E entries (0 allowed: the expert is skipped).
 *   W [E][N][K] and dW [E][N][K] bf16; X_perm [sum][K], Y_perm / dY_perm [sum][N],
 *   dX_perm [sum][K].  Expert e draws stochastic rounding with seed + e.
 *   ws: nvfp4_moe_workspace_bytes() bytes; it holds one linear workspace per expert
 *   (nvfp4_moe_expert_workspace gives expert e's, for nvfp4_linear_operand and
 *   nvfp4_read_status).
 */
size_t nvfp4_moe_workspace_bytes(const int64_t* group_rows, int E, int64_t K, int64_t N);
int nvfp4_moe_expert_workspace(void* ws, const int64_t* group_rows, int E, int64_t K, int64_t N,
                               int expert, void** expert_ws, size_t* expert_ws_bytes);
int nvfp4_moe_linear_fprop(const void* X_perm, const void* W, void* Y_perm,
                           const int64_t* group_rows, int E, int64_t K, int64_t N,
                           const int8_t* rht_signs, void* ws, size_t ws_bytes,
                           nvfp4_stream_t stream);
int nvfp4_moe_linear_dgrad(const void* dY_perm, void* dX_perm, const int64_t* group_rows, int E,
                           int64_t K, int64_t N, uint64_t seed, const int8_t* rht_signs, void* ws,
                           size_t ws_bytes, nvfp4_stream_t stream);
int nvfp4_moe_linear_wgrad(void* dW, const int64_t* group_rows, int E, int64_t K, int64_t N,
                           uint64_t seed, const int8_t* rht_signs, void* ws, size_t ws_bytes,
                           nvfp4_stream_t stream);
/*
 * Grouped expert layer: the computation of nvfp4_moe_linear_* (each expert a linear
 * layer with its own tensor scales; expert e draws stochastic rounding with seed + e
 * and counts element indices inside its own tensors, so the codes, scales and
 * outputs equal the per-expert calls'), with every step one launch over all experts:
 * the permuted tensors are quantized whole, in both orientations, with per-expert
 * tensor scales, and one persistent GEMM walks the tiles of all experts.  (The
 * explainer's "The model underneath": most of the FP4 FLOPs are expert GEMMs.)
 *   group_rows: HOST array of E <= 1024 entries, each a multiple of 128 (0 allowed),
 *   their sum R >= 128; K, N multiples of 128.  X_perm [R][K], Y_perm / dY_perm [R][N],
 *   dX_perm [R][K] bf16 in expert order; W, dW [E][N][K] bf16.
 *   ws: nvfp4_moe_grouped_workspace_bytes() bytes, 256-byte aligned; its status word
 *   is read with nvfp4_read_status.  fprop fills the X and W operands, dgrad the dY
 *   operands and wgrad reads both (call them in that order on one workspace).  The
 *   dW of an expert with no rows is written as zero.
 *   nvfp4_moe_grouped_operand: views (NVFP4_LIN_*) of the whole quantized tensors,
 *   X [R][K], X^T [K][R], W [E*N][K], W^T [K][E*N], dY [R][N], dY^T [N][R]; a view's
 *   tensor_scale points at E floats, one per expert.  No device access.
 */
size_t nvfp4_moe_grouped_workspace_bytes(const int64_t* group_rows, int E, int64_t K, int64_t N);
int nvfp4_moe_grouped_operand(void* ws, const int64_t* group_rows, int E, int64_t K, int64_t N,
                              int which, nvfp4_tensor* out);
int nvfp4_moe_grouped_fprop(const void* X_perm, const void* W, void* Y_perm, const int64_t* group_rows,
                            int E, int64_t K, int64_t N, const int8_t* rht_signs, void* ws,
                            size_t ws_bytes, nvfp4_stream_t stream);
/* nvfp4_moe_grouped_fprop with the routing gather fused into the quantization of X:
 * row r of the permuted X is row row_src[r] of X_tok [tokens][K] (row_src: device
 * int32 [R]; -1 reads as a zero row, the padding).  The permuted bf16 copy is never
 * written.  Results equal nvfp4_moe_gather followed by nvfp4_moe_grouped_fprop.  An
 * entry >= tokens is read as a zero row and recorded as NVFP4_ERR_INDEX in the status
 * word.                                                                              */
int nvfp4_moe_grouped_fprop_gather(const void* X_tok, const int32_t* row_src, int64_t tokens, const void* W,
                                   void* Y_perm, const int64_t* group_rows, int E, int64_t K, int64_t N,
                                   const int8_t* rht_signs, void* ws, size_t ws_bytes, nvfp4_stream_t stream);
int nvfp4_moe_grouped_dgrad(const void* dY_perm, void* dX_perm, const int64_t* group_rows, int E,
                            int64_t K, int64_t N, uint64_t seed, const int8_t* rht_signs, void* ws,
                            size_t ws_bytes, nvfp4_stream_t stream);
int nvfp4_moe_grouped_wgrad(void* dW, const int64_t* group_rows, int E, int64_t K, int64_t N,
                            void* ws, size_t ws_bytes, nvfp4_stream_t stream);
/*
 * nvfp4_moe_gather: dst[i] = src[row_src[i]] for rows of `cols` bf16 (row_src device
 * int32 [rows]; -1 writes a zero row).  cols % 8 == 0.
 * nvfp4_moe_combine: dst[t] = bf16(sum over j < topk of src[slots[t*topk + j]]) with an
 * fp32 sum in j order (slots device int32 [tokens][topk]; -1 entries are skipped).
 */
int nvfp4_moe_gather(const void* src, const int32_t* row_src, int64_t rows, int64_t cols,
                     void* dst, nvfp4_stream_t stream);
int nvfp4_moe_combine(const void* src, const int32_t* slots, int64_t tokens, int topk,
                      int64_t cols, void* dst, nvfp4_stream_t stream);

/*
 * Recipe options of the linear layer (NULL = the defaults above).
 *   weight_block_mode  NVFP4_BLOCK_16X16 (default): one quantization of W shared by
 *                      fprop and dgrad; NVFP4_BLOCK_1X16: the 1D-weight recipe, W
 *                      quantized 1x16 along K for fprop and, separately, 1x16 along N
 *                      for dgrad (the 1D-versus-2D weight comparison of "Paper of the
 *                      day: What matters for NVFP4 training?", "The problem").
 *   dgrad_rht          1: rotate both dgrad operands (dY and W^T) along N with the same
 *                      16-point RHT, dgrad alpha 1/16 (RHT on both backward GEMMs, the
 *                      Mosaic recipe of "Paper of the day: What matters for NVFP4
 *                      training?", "Main findings"); needs weight_block_mode 1X16.
 * The options change fprop's quantization of W and dgrad's of dY; pass the same
 * options to both calls on one workspace (wgrad is unaffected).  Invalid options:
 * NVFP4_ERR_ARG.
 */
typedef struct {
    int weight_block_mode;
    int dgrad_rht;
} nvfp4_linear_opts;
int nvfp4_linear_fprop_ex(const void* X, const void* W, void* Y, int64_t M, int64_t K, int64_t N,
                          const int8_t* rht_signs, const nvfp4_linear_opts* opts, void* ws,
                          size_t ws_bytes, nvfp4_stream_t stream);
int nvfp4_linear_dgrad_ex(const void* dY, void* dX, int64_t M, int64_t K, int64_t N, uint64_t seed,
                          const int8_t* rht_signs, const nvfp4_linear_opts* opts, void* ws,
                          size_t ws_bytes, nvfp4_stream_t stream);

/*
 * MXFP4, the comparison format ("Nemotron NVFP4" explainer, "What NVFP4 actually
 * is": E2M1 elements with one power-of-two E8M0 scale per 32 elements, 4.25 bits
 * per element, no tensor scale).  The pages fix no scale rule; the block scale is
 * the smallest power of two 2^k with amax_b <= 6 * 2^k, so no element clips (E8M0
 * code k + 127; 0 for an all-zero block; 255 when the block holds Inf or NaN), and
 * elements round to nearest even.
 * nvfp4_mx_quantize: row orientation, blocks along cols (cols % 32 == 0); one read.
 *   packed  out, rows * cols / 2 bytes; scales out, nvfp4_mx_scale_bytes(rows, cols)
 *   bytes in the layout of nvfp4_scale_bytes' scales over 32-element blocks (512-byte
 *   atoms of 128 rows x 4 blocks; padding written as 0).
 * nvfp4_mx_gemm: D = alpha * A B^T over MXFP4 operands (tcgen05 block-scaled MMA,
 *   scale_vec::2X with UE8M0 scales); K % 128 == 0, N % 8 == 0; D_bf16 and / or
 *   D_f32 as in nvfp4_gemm; status (nullable) as in nvfp4_gemm.
 */
size_t nvfp4_mx_scale_bytes(int64_t rows, int64_t cols);
int nvfp4_mx_quantize(const void* x, int64_t rows, int64_t cols, uint8_t* packed, uint8_t* scales,
                      nvfp4_stream_t stream);
int nvfp4_mx_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB, float alpha,
                  int64_t M, int64_t N, int64_t K, void* D_bf16, float* D_f32, int* status,
                  nvfp4_stream_t stream);

/* Views of the quantized operands a linear workspace holds (no device access). */
enum {
    NVFP4_LIN_X_ROW = 0,  /* X,   M x K, 1x16 RNE                 */
    NVFP4_LIN_X_COL = 1,  /* X^T, K x M, RHT + 1x16 RNE           */
    NVFP4_LIN_W_ROW = 2,  /* W,   N x K, 16x16 RNE                */
    NVFP4_LIN_W_COL = 3,  /* W^T, K x N, 16x16 RNE                */
    NVFP4_LIN_DY_ROW = 4, /* dY,  M x N, 1x16 SR                  */
    NVFP4_LIN_DY_COL = 5  /* dY^T, N x M, RHT + 1x16 SR           */
};
int nvfp4_linear_operand(void* ws, int64_t M, int64_t K, int64_t N, int which,
                         nvfp4_tensor* out);

/*
 * nvfp4_quantize_noalloc -- nvfp4_quantize without the workspace argument, for
 * callers that cannot allocate device memory (for example a plugin that is handed
 * only its input and output buffers by a host framework owning every device
 * allocation, or a real-time loop that must not allocate after start-up).
 * The pages have no counterpart; this is a library convenience.
 * Arguments, layouts, results and errors are those of nvfp4_quantize.  Its 64
 * bytes of scratch (tensor amax words, status word) live in a static device array
 * of NVFP4_NOALLOC_SCRATCH_BYTES bytes that every GPU loading the library holds
 * until exit; a call needing more than that would be refused with
 * NVFP4_ERR_WORKSPACE.  The first call on a device looks the array's address up
 * (cudaGetSymbolAddress) with that device current and caches it for that device;
 * make that first call before any stream capture.  The cached address belongs to
 * the device's current context: after cudaDeviceReset the next call sees a new
 * context and looks the address up again (make that call outside a capture too).  All calls share the array and each clears it on its stream
 * before use: calls that overlap on the GPU (other streams, other threads) race.
 * There is no status word to read back: an Inf/NaN input shows as a NaN
 * tensor_scale.  It calls no allocator.
 */
#define NVFP4_NOALLOC_SCRATCH_BYTES 256
int nvfp4_quantize_noalloc(const void* x, int64_t rows, int64_t cols, int block_mode,
                           int rounding, uint64_t seed, uint8_t* packed, uint8_t* scales,
                           float* tensor_scale, nvfp4_stream_t stream);

/* Status word of a quantize or linear workspace: synchronizes `stream`, then
 * copies the word to *status (host): NVFP4_OK or the first device error recorded
 * since the word was last cleared.  Every call that takes the workspace clears
 * the word on its stream before its first kernel, so the word describes the
 * latest such call; reading it does not change it.                            */
int nvfp4_read_status(void* workspace, int* status, nvfp4_stream_t stream);

const char* nvfp4_status_string(int status);
int nvfp4_version(void); /* major * 10000 + minor * 100 + patch */

#ifdef __cplusplus
}
#endif
#endif /* NVFP4_H */
