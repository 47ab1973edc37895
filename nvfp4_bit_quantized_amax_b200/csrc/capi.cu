// capi.cu -- the extern "C" boundary of libnvfp4 (declared in include/nvfp4.h).
//
// Host-side only: argument validation (before any launch), workspace layout,
// and the order of kernel launches for each entry point.  Every step of the
// computation runs in the kernels of quantize.cu and gemm.cu.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>
#include <string.h>

#include "../../include/nvfp4.h"
#include "internal.h"

using namespace nvfp4;

// NVTX range over one C-ABI call (a no-op unless a profiler is attached), so that
// timelines show each entry point around its kernels.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};
#define NVFP4_RANGE(name) NvtxRange nvfp4_range_(name)

namespace {

constexpr int64_t kCtrlBytes = 256;   // control block at the start of a workspace
constexpr int kWordStatus = 8;        // int status at byte 32 of every workspace
constexpr int64_t kClearBytes = 64;   // amax words + status, cleared by every call
// linear workspace: amax words and tensor-scale slots inside the control block
constexpr int kWX = 0, kWW = 2, kWDY = 4;                   // word pairs [row, col]
constexpr int kGxr = 16, kGxc = 17, kGw = 18, kGwc = 19, kGdyr = 20, kGdyc = 21;  // float slots

int64_t pad(int64_t v, int64_t m) { return (v + m - 1) / m * m; }
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

struct DevInfo {
    int sm_count = 0;
    int status = 0;  // 0 unknown, 1 ok, -1 not sm_100
};

int device_check(int* sm_count) {
    static DevInfo info[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NVFP4_ERR_CUDA;
    DevInfo& d = info[dev];
    if (d.status == 0) {
        int major = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        d.sm_count = sms;
        d.status = (major == 10) ? 1 : -1;
    }
    if (d.status < 0) return NVFP4_ERR_DEVICE;
    *sm_count = d.sm_count;
    return NVFP4_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

// Sign vector (+1/-1 x 16, host) -> bit mask of the -1 entries.
int sign_mask_of(const int8_t* signs, uint32_t* mask) {
    if (!signs) return NVFP4_ERR_ARG;
    uint32_t m = 0;
    for (int i = 0; i < 16; ++i) {
        if (signs[i] == -1)
            m |= 1u << i;
        else if (signs[i] != 1)
            return NVFP4_ERR_ARG;
    }
    *mask = m;
    return NVFP4_OK;
}

struct LinLayout {
    int64_t x_row, x_row_sf, x_col, x_col_sf, w_row, w_row_sf, w_col, w_col_sf;
    int64_t dy_row, dy_row_sf, dy_col, dy_col_sf, total;
};
LinLayout lin_layout(int64_t M, int64_t K, int64_t N) {
    LinLayout L;
    int64_t off = kCtrlBytes;
    auto take = [&](int64_t bytes) {
        const int64_t o = off;
        off = pad(off + bytes, 256);
        return o;
    };
    L.x_row = take(M * K / 2);
    L.x_row_sf = take((int64_t)nvfp4_scale_bytes(M, K));
    L.x_col = take(K * M / 2);
    L.x_col_sf = take((int64_t)nvfp4_scale_bytes(K, M));
    L.w_row = take(N * K / 2);
    L.w_row_sf = take((int64_t)nvfp4_scale_bytes(N, K));
    L.w_col = take(K * N / 2);
    L.w_col_sf = take((int64_t)nvfp4_scale_bytes(K, N));
    L.dy_row = take(M * N / 2);
    L.dy_row_sf = take((int64_t)nvfp4_scale_bytes(M, N));
    L.dy_col = take(N * M / 2);
    L.dy_col_sf = take((int64_t)nvfp4_scale_bytes(N, M));
    L.total = off;
    return L;
}

int run_quantize(const void* x, int64_t rows, int64_t cols, bool two_d, int row_sr, int col_sr,
                 uint64_t seed, int col_rht, uint32_t mask, uint8_t* rd, uint8_t* rsf, float* rg,
                 uint8_t* cd, uint8_t* csf, float* cg, uint32_t* words, int* status, int sms,
                 cudaStream_t st, bool rows_only_kernel, int row_rht = 0) {
    cudaError_t e = launch_amax(static_cast<const uint16_t*>(x), rows, cols, col_rht && cd, mask,
                                words, sms, st, row_rht != 0, status);
    if (e != cudaSuccess) return NVFP4_ERR_CUDA;
    QuantParams p;
    memset(&p, 0, sizeof p);
    p.x = static_cast<const uint16_t*>(x);
    p.rows = rows;
    p.cols = cols;
    p.row_data = rd;
    p.row_sf = rsf;
    p.row_g = rg;
    p.col_data = cd;
    p.col_sf = csf;
    p.col_g = cg;
    p.amax_words = words;
    p.status = status;
    p.seed = seed;
    p.row_sr = row_sr;
    p.col_sr = col_sr;
    p.col_rht = (col_rht && cd) ? 1 : 0;
    p.row_rht = row_rht;
    p.sign_mask = mask;
    e = rows_only_kernel && !row_rht ? launch_quant_rows(p, sms, st) : launch_quant_tile(p, two_d, sms, st);
    if (e != cudaSuccess) return NVFP4_ERR_CUDA;
    if (rsf && (e = launch_sf_pad(rsf, rows, cols / 16, sms, st)) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (csf && (e = launch_sf_pad(csf, cols, rows / 16, sms, st)) != cudaSuccess) return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}

int gemm_call(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB,
              const float* sa, const float* sb, float alpha, int64_t M, int64_t N, int64_t K,
              void* Dbf, float* Df, int* status, int sms, cudaStream_t st, long long wait_cycles = 0) {
    GemmParams g{};
    g.wait_cycles = wait_cycles;
    g.A = A;
    g.sfA = sfA;
    g.B = B;
    g.sfB = sfB;
    g.scale_a = sa;
    g.scale_b = sb;
    g.alpha = alpha;
    g.M = M;
    g.N = N;
    g.K = K;
    g.D_bf16 = Dbf;
    g.D_f32 = Df;
    g.status = status;
    return cuda_status(launch_gemm(g, sms, st));
}

// ---------------------------------------------------------------- mixture of experts
int moe_check(const int64_t* group_rows, int E, int64_t K, int64_t N) {
    if (!group_rows || E < 1) return NVFP4_ERR_ARG;
    if (K < 64 || N < 64 || K % 64 || N % 64 || N > kMaxTileRows) return NVFP4_ERR_SHAPE;
    for (int e = 0; e < E; ++e)
        if (group_rows[e] < 0 || group_rows[e] % 64 || group_rows[e] > kMaxTileRows) return NVFP4_ERR_SHAPE;
    return NVFP4_OK;
}

}  // namespace

extern "C" size_t nvfp4_moe_workspace_bytes(const int64_t* group_rows, int E, int64_t K, int64_t N);

namespace {
// Calls fn(e, row offset, expert workspace, bytes) for every non-empty expert.
template <class F>
int moe_for_each(const int64_t* group_rows, int E, int64_t K, int64_t N, void* ws,
                        size_t ws_bytes, F&& fn) {
    int rc = moe_check(group_rows, E, K, N);
    if (rc) return rc;
    if (!ws) return NVFP4_ERR_WORKSPACE;
    if (ws_bytes < nvfp4_moe_workspace_bytes(group_rows, E, K, N)) return NVFP4_ERR_WORKSPACE;
    int64_t row = 0;
    size_t off = 0;
    for (int e = 0; e < E; ++e) {
        const int64_t m = group_rows[e];
        if (m == 0) continue;
        const size_t bytes = nvfp4_linear_workspace_bytes(m, K, N);
        rc = fn(e, row, static_cast<uint8_t*>(ws) + off, bytes);
        if (rc) return rc;
        row += m;
        off += (size_t)pad((int64_t)bytes, 256);
    }
    return NVFP4_OK;
}

}  // namespace

extern "C" {

int nvfp4_version(void) { return 100; }

const char* nvfp4_status_string(int s) {
    switch (s) {
        case NVFP4_OK: return "ok";
        case NVFP4_ERR_ARG: return "invalid argument";
        case NVFP4_ERR_SHAPE: return "unsupported shape";
        case NVFP4_ERR_ALIGN: return "pointer not 16-byte aligned";
        case NVFP4_ERR_CUDA: return "CUDA error";
        case NVFP4_ERR_NONFINITE: return "input holds Inf or NaN";
        case NVFP4_ERR_TIMEOUT: return "a bounded wait in a kernel ran out";
        case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
        case NVFP4_ERR_DEVICE: return "device is not sm_100";
        case NVFP4_ERR_INDEX: return "a row index lies outside its source tensor";
        case NVFP4_ERR_RHT_RANGE: return "a rotated 16-chunk spans more than 41 binades";
        default: return "unknown status";
    }
}

size_t nvfp4_packed_bytes(int64_t rows, int64_t cols) {
    return (rows <= 0 || cols <= 0) ? 0 : (size_t)(rows * cols / 2);
}

size_t nvfp4_scale_bytes(int64_t rows, int64_t cols) {
    return (rows <= 0 || cols <= 0) ? 0 : (size_t)(pad(rows, 128) * pad(cols / 16, 4));
}

size_t nvfp4_quantize_workspace_bytes(void) { return (size_t)kCtrlBytes; }

int nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int block_mode, int rounding,
                   uint64_t seed, uint8_t* packed, uint8_t* scales, float* tensor_scale,
                   void* workspace, nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_quantize");
    if (!x || !packed || !scales || !tensor_scale) return NVFP4_ERR_ARG;
    if (!workspace) return NVFP4_ERR_WORKSPACE;
    if (block_mode != NVFP4_BLOCK_1X16 && block_mode != NVFP4_BLOCK_16X16) return NVFP4_ERR_ARG;
    if (rounding != NVFP4_ROUND_RNE && rounding != NVFP4_ROUND_SR) return NVFP4_ERR_ARG;
    if (rows < 1 || cols < 16 || cols % 16 != 0) return NVFP4_ERR_SHAPE;
    if (block_mode == NVFP4_BLOCK_16X16 && (rows % 16 != 0 || rows > kMaxTileRows)) return NVFP4_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(scales, 16) || !aligned(workspace, 16) ||
        !aligned(tensor_scale, 4))
        return NVFP4_ERR_ALIGN;
    int sms = 0;
    int rc = device_check(&sms);
    if (rc) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint32_t* words = static_cast<uint32_t*>(workspace);
    if (cudaMemsetAsync(words, 0, kClearBytes, st) != cudaSuccess) return NVFP4_ERR_CUDA;
    return run_quantize(x, rows, cols, block_mode == NVFP4_BLOCK_16X16, rounding, 0, seed, 0, 0,
                        packed, scales, tensor_scale, nullptr, nullptr, nullptr, words,
                        reinterpret_cast<int*>(words + kWordStatus), sms, st,
                        block_mode == NVFP4_BLOCK_1X16);
}

int nvfp4_quantize_2d(const void* x, int64_t rows, int64_t cols, const nvfp4_quantize_opts* o,
                      nvfp4_tensor* row_out, nvfp4_tensor* col_out, void* workspace,
                      nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_quantize_2d");
    if (!x || !o || (!row_out && !col_out)) return NVFP4_ERR_ARG;
    if (!workspace) return NVFP4_ERR_WORKSPACE;
    if (o->block_mode != NVFP4_BLOCK_1X16 && o->block_mode != NVFP4_BLOCK_16X16) return NVFP4_ERR_ARG;
    if ((o->row_rounding != 0 && o->row_rounding != 1) || (o->col_rounding != 0 && o->col_rounding != 1))
        return NVFP4_ERR_ARG;
    uint32_t mask = 0;
    if (o->col_rht) {
        if (o->block_mode != NVFP4_BLOCK_1X16) return NVFP4_ERR_ARG;
        if (sign_mask_of(o->rht_signs, &mask)) return NVFP4_ERR_ARG;
    }
    if (rows < 1 || cols < 16 || cols % 16 != 0 || rows > kMaxTileRows) return NVFP4_ERR_SHAPE;
    if ((col_out || o->block_mode == NVFP4_BLOCK_16X16) && rows % 16 != 0) return NVFP4_ERR_SHAPE;
    for (nvfp4_tensor* t : {row_out, col_out}) {
        if (!t) continue;
        if (!t->data || !t->scales || !t->tensor_scale) return NVFP4_ERR_ARG;
        if (!aligned(t->data, 16) || !aligned(t->scales, 16) || !aligned(t->tensor_scale, 4))
            return NVFP4_ERR_ALIGN;
    }
    if (!aligned(x, 16) || !aligned(workspace, 16)) return NVFP4_ERR_ALIGN;
    int sms = 0;
    int rc = device_check(&sms);
    if (rc) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint32_t* words = static_cast<uint32_t*>(workspace);
    if (cudaMemsetAsync(words, 0, kClearBytes, st) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (row_out) {
        row_out->rows = rows;
        row_out->cols = cols;
    }
    if (col_out) {
        col_out->rows = cols;
        col_out->cols = rows;
    }
    return run_quantize(x, rows, cols, o->block_mode == NVFP4_BLOCK_16X16, o->row_rounding,
                        o->col_rounding, o->seed, o->col_rht, mask,
                        row_out ? row_out->data : nullptr, row_out ? row_out->scales : nullptr,
                        row_out ? row_out->tensor_scale : nullptr, col_out ? col_out->data : nullptr,
                        col_out ? col_out->scales : nullptr,
                        col_out ? col_out->tensor_scale : nullptr, words,
                        reinterpret_cast<int*>(words + kWordStatus), sms, st, false);
}

int nvfp4_rht(const void* x, int64_t rows, int64_t cols, int axis, const int8_t* signs, int n,
              float* y, nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_rht");
    if (!x || !y) return NVFP4_ERR_ARG;
    if (n != 16 || (axis != 0 && axis != 1)) return NVFP4_ERR_ARG;
    uint32_t mask = 0;
    if (sign_mask_of(signs, &mask)) return NVFP4_ERR_ARG;
    if (rows < 1 || cols < 1) return NVFP4_ERR_SHAPE;
    if (axis == 1 && cols % 16 != 0) return NVFP4_ERR_SHAPE;
    if (axis == 0 && (rows % 16 != 0 || cols % 8 != 0)) return NVFP4_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(y, 16)) return NVFP4_ERR_ALIGN;
    int sms = 0;
    int rc = device_check(&sms);
    if (rc) return rc;
    return cuda_status(launch_rht(static_cast<const uint16_t*>(x), y, rows, cols, axis, mask, sms,
                                  reinterpret_cast<cudaStream_t>(stream)));
}

int nvfp4_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB,
               const float* scale_a, const float* scale_b, float alpha, int64_t M, int64_t N,
               int64_t K, void* D_bf16, float* D_f32, int* status, nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_gemm");
    return nvfp4_gemm_wait_limit(A, sfA, B, sfB, scale_a, scale_b, alpha, M, N, K, D_bf16, D_f32,
                                 status, 0, stream);
}

int nvfp4_gemm_wait_limit(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB,
                          const float* scale_a, const float* scale_b, float alpha, int64_t M,
                          int64_t N, int64_t K, void* D_bf16, float* D_f32, int* status,
                          long long wait_cycles, nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_gemm_wait_limit");
    if (!A || !sfA || !B || !sfB || (!D_bf16 && !D_f32)) return NVFP4_ERR_ARG;
    if (wait_cycles < 0) return NVFP4_ERR_ARG;
    if (M < 1 || N < 8 || K < 64 || K % 64 != 0 || N % 8 != 0) return NVFP4_ERR_SHAPE;
    if (M > (1ll << 31) - 256 || N > (1ll << 31) - 256 || K / 2 > (1ll << 31)) return NVFP4_ERR_SHAPE;
    if (!aligned(A, 16) || !aligned(B, 16) || !aligned(sfA, 16) || !aligned(sfB, 16) ||
        (D_bf16 && !aligned(D_bf16, 16)) || (D_f32 && !aligned(D_f32, 16)))
        return NVFP4_ERR_ALIGN;
    int sms = 0;
    int rc = device_check(&sms);
    if (rc) return rc;
    return gemm_call(A, sfA, B, sfB, scale_a, scale_b, alpha, M, N, K, D_bf16, D_f32, status, sms,
                     reinterpret_cast<cudaStream_t>(stream), wait_cycles);
}

size_t nvfp4_linear_workspace_bytes(int64_t M, int64_t K, int64_t N) {
    if (M <= 0 || K <= 0 || N <= 0) return 0;
    return (size_t)lin_layout(M, K, N).total;
}

int nvfp4_linear_operand(void* ws, int64_t M, int64_t K, int64_t N, int which, nvfp4_tensor* out) {
    if (!ws || !out) return NVFP4_ERR_ARG;
    if (M <= 0 || K <= 0 || N <= 0) return NVFP4_ERR_SHAPE;
    const LinLayout L = lin_layout(M, K, N);
    uint8_t* b = static_cast<uint8_t*>(ws);
    float* g = reinterpret_cast<float*>(b);
    switch (which) {
        case NVFP4_LIN_X_ROW: *out = {b + L.x_row, b + L.x_row_sf, g + kGxr, M, K}; break;
        case NVFP4_LIN_X_COL: *out = {b + L.x_col, b + L.x_col_sf, g + kGxc, K, M}; break;
        case NVFP4_LIN_W_ROW: *out = {b + L.w_row, b + L.w_row_sf, g + kGw, N, K}; break;
        case NVFP4_LIN_W_COL: *out = {b + L.w_col, b + L.w_col_sf, g + kGwc, K, N}; break;
        case NVFP4_LIN_DY_ROW: *out = {b + L.dy_row, b + L.dy_row_sf, g + kGdyr, M, N}; break;
        case NVFP4_LIN_DY_COL: *out = {b + L.dy_col, b + L.dy_col_sf, g + kGdyc, N, M}; break;
        default: return NVFP4_ERR_ARG;
    }
    return NVFP4_OK;
}

static int lin_check(int64_t M, int64_t K, int64_t N, void* ws, size_t ws_bytes) {
    if (!ws) return NVFP4_ERR_WORKSPACE;
    if (M < 64 || K < 64 || N < 64 || M % 64 || K % 64 || N % 64) return NVFP4_ERR_SHAPE;
    if (M > kMaxTileRows || N > kMaxTileRows) return NVFP4_ERR_SHAPE;
    if (ws_bytes < nvfp4_linear_workspace_bytes(M, K, N)) return NVFP4_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return NVFP4_ERR_ALIGN;
    return NVFP4_OK;
}

static int opts_check(const nvfp4_linear_opts* o) {
    if (!o) return NVFP4_OK;
    if (o->weight_block_mode != NVFP4_BLOCK_16X16 && o->weight_block_mode != NVFP4_BLOCK_1X16)
        return NVFP4_ERR_ARG;
    if (o->dgrad_rht != 0 && o->dgrad_rht != 1) return NVFP4_ERR_ARG;
    if (o->dgrad_rht && o->weight_block_mode != NVFP4_BLOCK_1X16) return NVFP4_ERR_ARG;
    return NVFP4_OK;
}

int nvfp4_linear_fprop_ex(const void* X, const void* W, void* Y, int64_t M, int64_t K, int64_t N,
                          const int8_t* rht_signs, const nvfp4_linear_opts* opts, void* ws,
                          size_t ws_bytes, nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_linear_fprop_ex");
    if (!X || !W || !Y) return NVFP4_ERR_ARG;
    uint32_t mask = 0;
    if (sign_mask_of(rht_signs, &mask)) return NVFP4_ERR_ARG;
    int rc = opts_check(opts);
    if (rc) return rc;
    const bool w1d = opts && opts->weight_block_mode == NVFP4_BLOCK_1X16;
    const int dgrad_rht = opts ? opts->dgrad_rht : 0;
    if ((rc = lin_check(M, K, N, ws, ws_bytes))) return rc;
    if (!aligned(X, 16) || !aligned(W, 16) || !aligned(Y, 16)) return NVFP4_ERR_ALIGN;
    int sms = 0;
    if ((rc = device_check(&sms))) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    nvfp4_tensor xr{}, xc{}, wr{}, wc{};
    nvfp4_linear_operand(ws, M, K, N, NVFP4_LIN_X_ROW, &xr);
    nvfp4_linear_operand(ws, M, K, N, NVFP4_LIN_X_COL, &xc);
    nvfp4_linear_operand(ws, M, K, N, NVFP4_LIN_W_ROW, &wr);
    nvfp4_linear_operand(ws, M, K, N, NVFP4_LIN_W_COL, &wc);
    uint32_t* words = static_cast<uint32_t*>(ws);
    int* status = reinterpret_cast<int*>(words + kWordStatus);
    if (cudaMemsetAsync(words, 0, kClearBytes, st) != cudaSuccess) return NVFP4_ERR_CUDA;
    // X: rows (1x16 RNE) for fprop, RHT columns (1x16 RNE) for wgrad -- one read
    rc = run_quantize(X, M, K, false, 0, 0, 0, 1, mask, xr.data, xr.scales, xr.tensor_scale, xc.data,
                      xc.scales, xc.tensor_scale, words + kWX, status, sms, st, false);
    if (rc) return rc;
    // W -- one read: 16x16 RNE shared by both orientations, or (1D-weight recipe) 1x16
    // RNE along K for fprop and, separately, 1x16 RNE along N for dgrad, rotated
    // along N under the Mosaic recipe
    rc = run_quantize(W, N, K, !w1d, 0, 0, 0, w1d ? dgrad_rht : 0, mask, wr.data, wr.scales,
                      wr.tensor_scale, wc.data, wc.scales, wc.tensor_scale, words + kWW, status, sms, st,
                      false);
    if (rc) return rc;
    return gemm_call(xr.data, xr.scales, wr.data, wr.scales, xr.tensor_scale, wr.tensor_scale, 1.0f,
                     M, N, K, Y, nullptr, status, sms, st);
}

int nvfp4_linear_fprop(const void* X, const void* W, void* Y, int64_t M, int64_t K, int64_t N,
                       const int8_t* rht_signs, void* ws, size_t ws_bytes, nvfp4_stream_t stream) {
    return nvfp4_linear_fprop_ex(X, W, Y, M, K, N, rht_signs, nullptr, ws, ws_bytes, stream);
}

int nvfp4_linear_dgrad_ex(const void* dY, void* dX, int64_t M, int64_t K, int64_t N, uint64_t seed,
                          const int8_t* rht_signs, const nvfp4_linear_opts* opts, void* ws,
                          size_t ws_bytes, nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_linear_dgrad_ex");
    if (!dY || !dX) return NVFP4_ERR_ARG;
    uint32_t mask = 0;
    if (sign_mask_of(rht_signs, &mask)) return NVFP4_ERR_ARG;
    int rc = opts_check(opts);
    if (rc) return rc;
    const int dgrad_rht = opts ? opts->dgrad_rht : 0;
    if ((rc = lin_check(M, K, N, ws, ws_bytes))) return rc;
    if (!aligned(dY, 16) || !aligned(dX, 16)) return NVFP4_ERR_ALIGN;
    int sms = 0;
    if ((rc = device_check(&sms))) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    nvfp4_tensor dr{}, dc{}, wc{};
    nvfp4_linear_operand(ws, M, K, N, NVFP4_LIN_DY_ROW, &dr);
    nvfp4_linear_operand(ws, M, K, N, NVFP4_LIN_DY_COL, &dc);
    nvfp4_linear_operand(ws, M, K, N, NVFP4_LIN_W_COL, &wc);
    uint32_t* words = static_cast<uint32_t*>(ws);
    int* status = reinterpret_cast<int*>(words + kWordStatus);
    if (cudaMemsetAsync(words, 0, kClearBytes, st) != cudaSuccess) return NVFP4_ERR_CUDA;
    // dY: rows (1x16 SR, stream 0; rotated along N under the Mosaic recipe) for dgrad,
    // RHT columns (1x16 SR, stream 1) for wgrad
    rc = run_quantize(dY, M, N, false, 1, 1, seed, 1, mask, dr.data, dr.scales, dr.tensor_scale,
                      dc.data, dc.scales, dc.tensor_scale, words + kWDY, status, sms, st, false, dgrad_rht);
    if (rc) return rc;
    // with both operands rotated along N the rotation cancels: H H^T = 16 I
    return gemm_call(dr.data, dr.scales, wc.data, wc.scales, dr.tensor_scale, wc.tensor_scale,
                     dgrad_rht ? 1.0f / 16.0f : 1.0f, M, K, N, dX, nullptr, status, sms, st);
}

int nvfp4_linear_dgrad(const void* dY, void* dX, int64_t M, int64_t K, int64_t N, uint64_t seed,
                       const int8_t* rht_signs, void* ws, size_t ws_bytes, nvfp4_stream_t stream) {
    return nvfp4_linear_dgrad_ex(dY, dX, M, K, N, seed, rht_signs, nullptr, ws, ws_bytes, stream);
}

int nvfp4_linear_wgrad(const void* dY, void* dW, int64_t M, int64_t K, int64_t N, uint64_t seed,
                       const int8_t* rht_signs, void* ws, size_t ws_bytes, nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_linear_wgrad");
    if (!dW) return NVFP4_ERR_ARG;
    uint32_t mask = 0;
    if (dY && sign_mask_of(rht_signs, &mask)) return NVFP4_ERR_ARG;
    int rc = lin_check(M, K, N, ws, ws_bytes);
    if (rc) return rc;
    if ((dY && !aligned(dY, 16)) || !aligned(dW, 16)) return NVFP4_ERR_ALIGN;
    int sms = 0;
    if ((rc = device_check(&sms))) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    nvfp4_tensor dc{}, xc{};
    nvfp4_linear_operand(ws, M, K, N, NVFP4_LIN_DY_COL, &dc);
    nvfp4_linear_operand(ws, M, K, N, NVFP4_LIN_X_COL, &xc);
    uint32_t* words = static_cast<uint32_t*>(ws);
    int* status = reinterpret_cast<int*>(words + kWordStatus);
    if (cudaMemsetAsync(words, 0, kClearBytes, st) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (dY) {
        rc = run_quantize(dY, M, N, false, 0, 1, seed, 1, mask, nullptr, nullptr, nullptr, dc.data,
                          dc.scales, dc.tensor_scale, words + kWDY, status, sms, st, false);
        if (rc) return rc;
    }
    // dW = (dY^T D H)(X^T D H)^T / 16: the rotation cancels, H H^T = 16 I
    return gemm_call(dc.data, dc.scales, xc.data, xc.scales, dc.tensor_scale, xc.tensor_scale,
                     1.0f / 16.0f, N, K, M, dW, nullptr, status, sms, st);
}

size_t nvfp4_moe_workspace_bytes(const int64_t* group_rows, int E, int64_t K, int64_t N) {
    if (moe_check(group_rows, E, K, N)) return 0;
    size_t total = 0;
    for (int e = 0; e < E; ++e)
        if (group_rows[e] > 0) total += (size_t)pad((int64_t)nvfp4_linear_workspace_bytes(group_rows[e], K, N), 256);
    return total;
}

int nvfp4_moe_expert_workspace(void* ws, const int64_t* group_rows, int E, int64_t K, int64_t N,
                               int expert, void** expert_ws, size_t* expert_ws_bytes) {
    int rc = moe_check(group_rows, E, K, N);
    if (rc) return rc;
    if (!ws || !expert_ws || !expert_ws_bytes || expert < 0 || expert >= E) return NVFP4_ERR_ARG;
    size_t off = 0;
    for (int e = 0; e < expert; ++e)
        if (group_rows[e] > 0) off += (size_t)pad((int64_t)nvfp4_linear_workspace_bytes(group_rows[e], K, N), 256);
    *expert_ws = static_cast<uint8_t*>(ws) + off;
    *expert_ws_bytes = group_rows[expert] > 0 ? nvfp4_linear_workspace_bytes(group_rows[expert], K, N) : 0;
    return NVFP4_OK;
}

int nvfp4_moe_linear_fprop(const void* X_perm, const void* W, void* Y_perm,
                           const int64_t* group_rows, int E, int64_t K, int64_t N,
                           const int8_t* rht_signs, void* ws, size_t ws_bytes,
                           nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_moe_linear_fprop");
    if (!X_perm || !W || !Y_perm) return NVFP4_ERR_ARG;
    return moe_for_each(group_rows, E, K, N, ws, ws_bytes, [&](int e, int64_t row, void* w, size_t b) {
        return nvfp4_linear_fprop(static_cast<const uint16_t*>(X_perm) + row * K,
                                  static_cast<const uint16_t*>(W) + (int64_t)e * N * K,
                                  static_cast<uint16_t*>(Y_perm) + row * N, group_rows[e], K, N,
                                  rht_signs, w, b, stream);
    });
}

int nvfp4_moe_linear_dgrad(const void* dY_perm, void* dX_perm, const int64_t* group_rows, int E,
                           int64_t K, int64_t N, uint64_t seed, const int8_t* rht_signs, void* ws,
                           size_t ws_bytes, nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_moe_linear_dgrad");
    if (!dY_perm || !dX_perm) return NVFP4_ERR_ARG;
    return moe_for_each(group_rows, E, K, N, ws, ws_bytes, [&](int e, int64_t row, void* w, size_t b) {
        return nvfp4_linear_dgrad(static_cast<const uint16_t*>(dY_perm) + row * N,
                                  static_cast<uint16_t*>(dX_perm) + row * K, group_rows[e], K, N,
                                  seed + (uint64_t)e, rht_signs, w, b, stream);
    });
}

int nvfp4_moe_linear_wgrad(void* dW, const int64_t* group_rows, int E, int64_t K, int64_t N,
                           uint64_t seed, const int8_t* rht_signs, void* ws, size_t ws_bytes,
                           nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_moe_linear_wgrad");
    if (!dW) return NVFP4_ERR_ARG;
    return moe_for_each(group_rows, E, K, N, ws, ws_bytes, [&](int e, int64_t row, void* w, size_t b) {
        (void)row;
        return nvfp4_linear_wgrad(nullptr, static_cast<uint16_t*>(dW) + (int64_t)e * N * K,
                                  group_rows[e], K, N, seed + (uint64_t)e, rht_signs, w, b, stream);
    });
}

int nvfp4_moe_gather(const void* src, const int32_t* row_src, int64_t rows, int64_t cols,
                     void* dst, nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_moe_gather");
    if (!src || !row_src || !dst) return NVFP4_ERR_ARG;
    if (rows < 1 || cols < 8 || cols % 8) return NVFP4_ERR_SHAPE;
    if (!aligned(src, 16) || !aligned(dst, 16) || !aligned(row_src, 4)) return NVFP4_ERR_ALIGN;
    int sms = 0;
    int rc = device_check(&sms);
    if (rc) return rc;
    return cuda_status(launch_moe_gather(static_cast<const uint16_t*>(src), row_src,
                                         static_cast<uint16_t*>(dst), rows, cols, sms,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

int nvfp4_moe_combine(const void* src, const int32_t* slots, int64_t tokens, int topk,
                      int64_t cols, void* dst, nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_moe_combine");
    if (!src || !slots || !dst || topk < 1) return NVFP4_ERR_ARG;
    if (tokens < 1 || cols < 8 || cols % 8) return NVFP4_ERR_SHAPE;
    if (!aligned(src, 16) || !aligned(dst, 16) || !aligned(slots, 4)) return NVFP4_ERR_ALIGN;
    int sms = 0;
    int rc = device_check(&sms);
    if (rc) return rc;
    return cuda_status(launch_moe_combine(static_cast<const uint16_t*>(src), slots,
                                          static_cast<uint16_t*>(dst), tokens, cols, topk, sms,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

int nvfp4_read_status(void* workspace, int* status, nvfp4_stream_t stream) {
    if (!workspace || !status) return NVFP4_ERR_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return NVFP4_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, static_cast<uint32_t*>(workspace) + kWordStatus, sizeof v,
                   cudaMemcpyDeviceToHost) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    *status = v;
    return NVFP4_OK;
}


}  // extern "C"

// ---------------------------------------------------------------- grouped mixture of experts
namespace {
// Workspace of the grouped expert layer: a header (status), per-group amax words
// and tensor scales, the group tables, then every quantized operand of the whole
// permuted tensors (rows R = sum of group rows):
//   X row [R][K], X^T col [K][R] (RHT), W row [E*N][K], W^T col [K][E*N],
//   dY row [R][N], dY^T col [N][R] (RHT).
struct MoeLayout {
    int64_t words_x, words_w, words_dy;          // 2E words each
    int64_t gx_row, gx_col, gw_row, gw_col, gdy_row, gdy_col;  // E floats each
    int64_t mtile_group, group_row0, group_nrows;
    int64_t pair_row0, pair_group, pair_rows;  // 256-row tiles of the groups
    int64_t x_row, x_row_sf, x_col, x_col_sf, w_row, w_row_sf, w_col, w_col_sf;
    int64_t dy_row, dy_row_sf, dy_col, dy_col_sf, total;
    int64_t R;
    int64_t pair_tiles;  // sum over groups of ceil(rows / 256)
};
MoeLayout moe_layout(const int64_t* group_rows, int E, int64_t K, int64_t N) {
    MoeLayout L;
    L.R = 0;
    L.pair_tiles = 0;
    for (int e = 0; e < E; ++e) {
        L.R += group_rows[e];
        L.pair_tiles += (group_rows[e] + 255) / 256;
    }
    int64_t off = 256;  // header: status word
    auto take = [&](int64_t bytes) {
        const int64_t o = off;
        off = pad(off + (bytes > 0 ? bytes : 1), 256);
        return o;
    };
    L.words_x = take(8 * E);
    L.words_w = take(8 * E);
    L.words_dy = take(8 * E);
    L.gx_row = take(4 * E);
    L.gx_col = take(4 * E);
    L.gw_row = take(4 * E);
    L.gw_col = take(4 * E);
    L.gdy_row = take(4 * E);
    L.gdy_col = take(4 * E);
    L.mtile_group = take(4 * (L.R / 128));
    L.group_row0 = take(8 * E);
    L.group_nrows = take(8 * E);
    L.pair_row0 = take(8 * L.pair_tiles);
    L.pair_group = take(4 * L.pair_tiles);
    L.pair_rows = take(4 * L.pair_tiles);
    const int64_t R = L.R, EN = (int64_t)E * N;
    L.x_row = take(R * K / 2);
    L.x_row_sf = take((int64_t)nvfp4_scale_bytes(R, K));
    L.x_col = take(K * R / 2);
    L.x_col_sf = take((int64_t)nvfp4_scale_bytes(K, R));
    L.w_row = take(EN * K / 2);
    L.w_row_sf = take((int64_t)nvfp4_scale_bytes(EN, K));
    L.w_col = take(K * EN / 2);
    L.w_col_sf = take((int64_t)nvfp4_scale_bytes(K, EN));
    L.dy_row = take(R * N / 2);
    L.dy_row_sf = take((int64_t)nvfp4_scale_bytes(R, N));
    L.dy_col = take(N * R / 2);
    L.dy_col_sf = take((int64_t)nvfp4_scale_bytes(N, R));
    L.total = off;
    return L;
}

int moe_grouped_check(const int64_t* group_rows, int E, int64_t K, int64_t N) {
    if (!group_rows || E < 1 || E > kMaxGroups) return NVFP4_ERR_ARG;
    if (K < 128 || N < 128 || K % 128 || N % 128) return NVFP4_ERR_SHAPE;
    int64_t R = 0;
    for (int e = 0; e < E; ++e) {
        if (group_rows[e] < 0 || group_rows[e] % 128) return NVFP4_ERR_SHAPE;
        R += group_rows[e];
    }
    if (R < 128 || R > kMaxTileRows || (int64_t)E * N > kMaxTileRows) return NVFP4_ERR_SHAPE;
    return NVFP4_OK;
}

// Common checks; writes the group tables into the workspace (copied from a host
// staging buffer on `st`).
int moe_grouped_begin(const int64_t* group_rows, int E, int64_t K, int64_t N, void* ws,
                      size_t ws_bytes, cudaStream_t st, MoeLayout* L, int* sms) {
    int rc = moe_grouped_check(group_rows, E, K, N);
    if (rc) return rc;
    *L = moe_layout(group_rows, E, K, N);
    if (!ws) return NVFP4_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return NVFP4_ERR_ALIGN;
    if (ws_bytes < (size_t)L->total) return NVFP4_ERR_WORKSPACE;
    if ((rc = device_check(sms))) return rc;
    uint8_t* b = static_cast<uint8_t*>(ws);
    if (launch_group_tables(group_rows, E, reinterpret_cast<int32_t*>(b + L->mtile_group),
                            reinterpret_cast<int64_t*>(b + L->group_row0),
                            reinterpret_cast<int64_t*>(b + L->group_nrows), st,
                            reinterpret_cast<int64_t*>(b + L->pair_row0),
                            reinterpret_cast<int32_t*>(b + L->pair_group),
                            reinterpret_cast<int32_t*>(b + L->pair_rows)) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}

// Grouped quantize of one tensor: amax per group, then both orientations.
int run_quantize_grouped(const void* x, int64_t rows, int64_t cols, bool two_d, int row_sr, int col_sr,
                         uint64_t seed, int col_rht, uint32_t mask, uint8_t* rd, uint8_t* rsf, float* rg,
                         uint8_t* cd, uint8_t* csf, float* cg, uint32_t* words, int* status,
                         const int32_t* row_group, const int64_t* row0, const int64_t* nrows,
                         int64_t uniform, int sms, cudaStream_t st, const int32_t* row_src = nullptr,
                         int64_t src_rows = 0) {
    QuantParams p;
    memset(&p, 0, sizeof p);
    p.x = static_cast<const uint16_t*>(x);
    p.rows = rows;
    p.cols = cols;
    p.row_data = rd;
    p.row_sf = rsf;
    p.row_g = rg;
    p.col_data = cd;
    p.col_sf = csf;
    p.col_g = cg;
    p.amax_words = words;
    p.status = status;
    p.seed = seed;
    p.row_sr = row_sr;
    p.col_sr = col_sr;
    p.col_rht = (col_rht && cd) ? 1 : 0;
    p.sign_mask = mask;
    p.row_group = row_group;
    p.group_row0 = row0;
    p.group_nrows = nrows;
    p.group_rows_uniform = uniform;
    p.row_src = row_src;
    p.src_rows = src_rows;
    cudaError_t e = launch_amax_grouped(p, sms, st);
    if (e != cudaSuccess) return NVFP4_ERR_CUDA;
    e = launch_quant_tile(p, two_d, sms, st);
    return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

int moe_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB, const float* sa,
             const float* sb, float alpha, int64_t M, int64_t N, int64_t K, void* D, int* status, int mode,
             const int32_t* mtile_group, int64_t b_group_rows, int64_t b_group_k, int64_t Kb,
             const int64_t* k_start, const int64_t* k_len, int groups, int sms, cudaStream_t st,
             const MoeLayout* L = nullptr, const uint8_t* ws = nullptr) {
    GemmParams g{};
    if (mode == 1 && L && ws) {  // the 256-row group tiles of the two-SM kernel
        g.pair_row0 = reinterpret_cast<const int64_t*>(ws + L->pair_row0);
        g.pair_group = reinterpret_cast<const int32_t*>(ws + L->pair_group);
        g.pair_rows = reinterpret_cast<const int32_t*>(ws + L->pair_rows);
        g.num_pair_tiles = L->pair_tiles;
    }
    g.A = A;
    g.sfA = sfA;
    g.B = B;
    g.sfB = sfB;
    g.scale_a = sa;
    g.scale_b = sb;
    g.alpha = alpha;
    g.M = M;
    g.N = N;
    g.K = K;
    g.D_bf16 = D;
    g.status = status;
    g.group_mode = mode;
    g.mtile_group = mtile_group;
    g.b_group_rows = b_group_rows;
    g.b_group_k = b_group_k;
    g.Kb = Kb;
    g.k_start = k_start;
    g.k_len = k_len;
    g.num_groups = groups;
    return cuda_status(launch_gemm(g, sms, st));
}
}  // namespace

extern "C" {

size_t nvfp4_mx_scale_bytes(int64_t rows, int64_t cols) {
    if (rows <= 0 || cols <= 0 || cols % 32) return 0;
    return (size_t)(pad(rows, 128) * pad(cols / 32, 4));
}

int nvfp4_mx_quantize(const void* x, int64_t rows, int64_t cols, uint8_t* packed, uint8_t* scales,
                      nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_mx_quantize");
    if (!x || !packed || !scales) return NVFP4_ERR_ARG;
    if (rows < 1 || cols < 32 || cols % 32 || rows > (1ll << 40) / cols) return NVFP4_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(packed, 16)) return NVFP4_ERR_ALIGN;
    int sms = 0;
    int rc = device_check(&sms);
    if (rc) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = launch_mx_quant_rows(static_cast<const uint16_t*>(x), rows, cols, packed, scales, sms, st);
    if (e == cudaSuccess) e = launch_sf_pad(scales, rows, cols / 32, sms, st);
    return cuda_status(e);
}

int nvfp4_mx_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB, float alpha,
                  int64_t M, int64_t N, int64_t K, void* D_bf16, float* D_f32, int* status,
                  nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_mx_gemm");
    if (!A || !sfA || !B || !sfB || (!D_bf16 && !D_f32)) return NVFP4_ERR_ARG;
    if (M < 1 || N < 8 || K < 128 || K % 128 != 0 || N % 8 != 0) return NVFP4_ERR_SHAPE;
    if (M > (1ll << 31) - 256 || N > (1ll << 31) - 256 || K / 2 > (1ll << 31)) return NVFP4_ERR_SHAPE;
    if (!aligned(A, 16) || !aligned(B, 16) || !aligned(sfA, 16) || !aligned(sfB, 16) ||
        (D_bf16 && !aligned(D_bf16, 16)) || (D_f32 && !aligned(D_f32, 16)))
        return NVFP4_ERR_ALIGN;
    int sms = 0;
    int rc = device_check(&sms);
    if (rc) return rc;
    GemmParams g{};
    g.A = A;
    g.sfA = sfA;
    g.B = B;
    g.sfB = sfB;
    g.alpha = alpha;
    g.M = M;
    g.N = N;
    g.K = K;
    g.D_bf16 = D_bf16;
    g.D_f32 = D_f32;
    g.status = status;
    g.mx = 1;
    return cuda_status(launch_gemm(g, sms, reinterpret_cast<cudaStream_t>(stream)));
}

size_t nvfp4_moe_grouped_workspace_bytes(const int64_t* group_rows, int E, int64_t K, int64_t N) {
    if (moe_grouped_check(group_rows, E, K, N)) return 0;
    return (size_t)moe_layout(group_rows, E, K, N).total;
}

int nvfp4_moe_grouped_operand(void* ws, const int64_t* group_rows, int E, int64_t K, int64_t N,
                              int which, nvfp4_tensor* out) {
    int rc = moe_grouped_check(group_rows, E, K, N);
    if (rc) return rc;
    if (!ws || !out || which < 0 || which > 5) return NVFP4_ERR_ARG;
    const MoeLayout L = moe_layout(group_rows, E, K, N);
    uint8_t* b = static_cast<uint8_t*>(ws);
    const int64_t R = L.R, EN = (int64_t)E * N;
    switch (which) {
        case NVFP4_LIN_X_ROW: *out = {b + L.x_row, b + L.x_row_sf, (float*)(b + L.gx_row), R, K}; break;
        case NVFP4_LIN_X_COL: *out = {b + L.x_col, b + L.x_col_sf, (float*)(b + L.gx_col), K, R}; break;
        case NVFP4_LIN_W_ROW: *out = {b + L.w_row, b + L.w_row_sf, (float*)(b + L.gw_row), EN, K}; break;
        case NVFP4_LIN_W_COL: *out = {b + L.w_col, b + L.w_col_sf, (float*)(b + L.gw_col), K, EN}; break;
        case NVFP4_LIN_DY_ROW: *out = {b + L.dy_row, b + L.dy_row_sf, (float*)(b + L.gdy_row), R, N}; break;
        default: *out = {b + L.dy_col, b + L.dy_col_sf, (float*)(b + L.gdy_col), N, R}; break;
    }
    return NVFP4_OK;
}

}  // extern "C"

namespace {
// Grouped fprop; X rows come from X_perm directly (row_src null) or from the token
// rows row_src[r] of X (tokens rows).
int moe_grouped_fprop(const void* X, const int32_t* row_src, int64_t tokens, const void* W, void* Y_perm,
                      const int64_t* group_rows, int E, int64_t K, int64_t N, const int8_t* rht_signs,
                      void* ws, size_t ws_bytes, nvfp4_stream_t stream) {
    if (!X || !W || !Y_perm) return NVFP4_ERR_ARG;
    if (!aligned(X, 16) || !aligned(W, 16) || !aligned(Y_perm, 16)) return NVFP4_ERR_ALIGN;
    const void* X_perm = X;
    uint32_t mask = 0;
    if (sign_mask_of(rht_signs, &mask)) return NVFP4_ERR_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    MoeLayout L;
    int sms = 0;
    int rc = moe_grouped_begin(group_rows, E, K, N, ws, ws_bytes, st, &L, &sms);
    if (rc) return rc;
    uint8_t* b = static_cast<uint8_t*>(ws);
    int* status = reinterpret_cast<int*>(b + 32);  // the word nvfp4_read_status reads
    if (cudaMemsetAsync(b, 0, 256, st) != cudaSuccess ||
        cudaMemsetAsync(b + L.words_x, 0, 8 * (size_t)E, st) != cudaSuccess ||
        cudaMemsetAsync(b + L.words_w, 0, 8 * (size_t)E, st) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    const int32_t* mt = reinterpret_cast<const int32_t*>(b + L.mtile_group);
    const int64_t* r0 = reinterpret_cast<const int64_t*>(b + L.group_row0);
    const int64_t* nr = reinterpret_cast<const int64_t*>(b + L.group_nrows);
    // X: rows (1x16 RNE) for fprop, RHT columns (1x16 RNE) for wgrad, per expert
    rc = run_quantize_grouped(X_perm, L.R, K, false, 0, 0, 0, 1, mask, b + L.x_row, b + L.x_row_sf,
                              (float*)(b + L.gx_row), b + L.x_col, b + L.x_col_sf, (float*)(b + L.gx_col),
                              (uint32_t*)(b + L.words_x), status, mt, r0, nr, 0, sms, st, row_src, tokens);
    if (rc) return rc;
    // W [E][N][K] as [E*N][K]: 16x16 RNE, both orientations, per expert
    rc = run_quantize_grouped(W, (int64_t)E * N, K, true, 0, 0, 0, 0, 0, b + L.w_row, b + L.w_row_sf,
                              (float*)(b + L.gw_row), b + L.w_col, b + L.w_col_sf, (float*)(b + L.gw_col),
                              (uint32_t*)(b + L.words_w), status, nullptr, nullptr, nullptr, N, sms, st);
    if (rc) return rc;
    // Y rows of expert e = X rows of e times W_e^T
    return moe_gemm(b + L.x_row, b + L.x_row_sf, b + L.w_row, b + L.w_row_sf, (float*)(b + L.gx_row),
                    (float*)(b + L.gw_row), 1.0f, L.R, N, K, Y_perm, status, 1, mt, N, 0, 0, nullptr,
                    nullptr, E, sms, st, &L, b);
}
}  // namespace

extern "C" {

int nvfp4_moe_grouped_fprop(const void* X_perm, const void* W, void* Y_perm, const int64_t* group_rows,
                            int E, int64_t K, int64_t N, const int8_t* rht_signs, void* ws,
                            size_t ws_bytes, nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_moe_grouped_fprop");
    return moe_grouped_fprop(X_perm, nullptr, 0, W, Y_perm, group_rows, E, K, N, rht_signs, ws, ws_bytes,
                             stream);
}

int nvfp4_moe_grouped_fprop_gather(const void* X_tok, const int32_t* row_src, int64_t tokens, const void* W,
                                   void* Y_perm, const int64_t* group_rows, int E, int64_t K, int64_t N,
                                   const int8_t* rht_signs, void* ws, size_t ws_bytes, nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_moe_grouped_fprop_gather");
    if (!row_src) return NVFP4_ERR_ARG;
    if (tokens < 1 || tokens > (1ll << 31) - 1) return NVFP4_ERR_SHAPE;
    if (!aligned(row_src, 4)) return NVFP4_ERR_ALIGN;
    return moe_grouped_fprop(X_tok, row_src, tokens, W, Y_perm, group_rows, E, K, N, rht_signs, ws, ws_bytes,
                             stream);
}

int nvfp4_moe_grouped_dgrad(const void* dY_perm, void* dX_perm, const int64_t* group_rows, int E,
                            int64_t K, int64_t N, uint64_t seed, const int8_t* rht_signs, void* ws,
                            size_t ws_bytes, nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_moe_grouped_dgrad");
    if (!dY_perm || !dX_perm) return NVFP4_ERR_ARG;
    if (!aligned(dY_perm, 16) || !aligned(dX_perm, 16)) return NVFP4_ERR_ALIGN;
    uint32_t mask = 0;
    if (sign_mask_of(rht_signs, &mask)) return NVFP4_ERR_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    MoeLayout L;
    int sms = 0;
    int rc = moe_grouped_begin(group_rows, E, K, N, ws, ws_bytes, st, &L, &sms);
    if (rc) return rc;
    uint8_t* b = static_cast<uint8_t*>(ws);
    int* status = reinterpret_cast<int*>(b + 32);  // the word nvfp4_read_status reads
    if (cudaMemsetAsync(b, 0, 256, st) != cudaSuccess ||
        cudaMemsetAsync(b + L.words_dy, 0, 8 * (size_t)E, st) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    const int32_t* mt = reinterpret_cast<const int32_t*>(b + L.mtile_group);
    const int64_t* r0 = reinterpret_cast<const int64_t*>(b + L.group_row0);
    const int64_t* nr = reinterpret_cast<const int64_t*>(b + L.group_nrows);
    // dY: rows (1x16 SR, stream 0) for dgrad, RHT columns (1x16 SR, stream 1) for wgrad;
    // expert e draws with seed + e
    rc = run_quantize_grouped(dY_perm, L.R, N, false, 1, 1, seed, 1, mask, b + L.dy_row, b + L.dy_row_sf,
                              (float*)(b + L.gdy_row), b + L.dy_col, b + L.dy_col_sf, (float*)(b + L.gdy_col),
                              (uint32_t*)(b + L.words_dy), status, mt, r0, nr, 0, sms, st);
    if (rc) return rc;
    // dX rows of expert e = dY rows of e times W_e (B = W^T [K][E*N], columns of e)
    return moe_gemm(b + L.dy_row, b + L.dy_row_sf, b + L.w_col, b + L.w_col_sf, (float*)(b + L.gdy_row),
                    (float*)(b + L.gw_col), 1.0f, L.R, K, N, dX_perm, status, 1, mt, 0, N, (int64_t)E * N,
                    nullptr, nullptr, E, sms, st, &L, b);
}

int nvfp4_moe_grouped_wgrad(void* dW, const int64_t* group_rows, int E, int64_t K, int64_t N,
                            void* ws, size_t ws_bytes, nvfp4_stream_t stream) {
    NVFP4_RANGE("nvfp4_moe_grouped_wgrad");
    if (!dW) return NVFP4_ERR_ARG;
    if (!aligned(dW, 16)) return NVFP4_ERR_ALIGN;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    MoeLayout L;
    int sms = 0;
    int rc = moe_grouped_begin(group_rows, E, K, N, ws, ws_bytes, st, &L, &sms);
    if (rc) return rc;
    uint8_t* b = static_cast<uint8_t*>(ws);
    int* status = reinterpret_cast<int*>(b + 32);  // the word nvfp4_read_status reads
    // dW_e = (dY_e^T D H)(X_e^T D H)^T / 16 over expert e's rows (zero if it has none)
    return moe_gemm(b + L.dy_col, b + L.dy_col_sf, b + L.x_col, b + L.x_col_sf, (float*)(b + L.gdy_col),
                    (float*)(b + L.gx_col), 1.0f / 16.0f, N, K, L.R, dW, status, 2, nullptr, 0, 0, 0,
                    reinterpret_cast<const int64_t*>(b + L.group_row0),
                    reinterpret_cast<const int64_t*>(b + L.group_nrows), E, sms, st);
}

}  // extern "C"
