// noalloc.cu -- nvfp4_quantize_noalloc: the quantizer for callers that cannot
// allocate device memory.
//
// nvfp4_quantize needs 64 bytes of device scratch (the tensor amax words and a
// status word) that the caller passes as `workspace`.  Some callers have no way
// to provide it: a plugin that is handed only its input and output buffers by a
// host framework which owns every device allocation, or a real-time loop that
// must not allocate after start-up.  This entry point takes the same arguments
// minus the workspace and keeps its scratch in a file-scope static device array
// instead, so it allocates nothing.
//
// The array is NVFP4_NOALLOC_SCRATCH_BYTES (256) bytes, held by every GPU that
// loads this library until the process exits.  All calls share it: the call
// clears the words that must start at zero on its stream before using them, and
// calls that overlap on the GPU (other streams, other host threads) race on it.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/nvfp4.h"
#include "internal.h"

using namespace nvfp4;

namespace {

constexpr size_t kScratchBytes = 256;  // NVFP4_NOALLOC_SCRATCH_BYTES
constexpr size_t kNeededBytes = 64;    // amax words [0..1] + status word [8], cleared per call
constexpr int kStatusWord = 8;

// The scratch itself.  In host code this name is only a stand-in for the symbol;
// the device address comes from cudaGetSymbolAddress, per device.
static __device__ __align__(256) uint32_t g_noalloc_scratch[kScratchBytes / 4];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
uint32_t* g_scratch_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};
unsigned long long g_ctx_id[kMaxDevices] = {};  // context the cached address belongs to

// Unique id of the calling thread's current context (0 when it cannot be read).
// A device's primary context gets a new id when it is re-created, e.g. after
// cudaDeviceReset, and a module's symbol address is only valid in the context it
// was resolved in.
unsigned long long current_context_id() {
    typedef CUresult (*GetCurrent)(CUcontext*);
    typedef CUresult (*GetId)(CUcontext, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static bool looked_up = false;
    if (!looked_up) {
        void* a = nullptr;
        void* b = nullptr;
        cudaDriverEntryPointQueryResult qa, qb;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
            qa == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
            qb == cudaDriverEntryPointSuccess) {
            get_current = reinterpret_cast<GetCurrent>(a);
            get_id = reinterpret_cast<GetId>(b);
        }
        looked_up = true;
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Once per device (and again if that device's context was re-created), with the
// device current: resolve the array's device address.
int scratch_for_current_device(uint32_t** ptr, int* sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    // 0 when no context is current on this thread yet (the runtime binds the
    // primary context at its first call that needs one, cudaGetSymbolAddress below)
    const unsigned long long ctx = current_context_id();
    if (!g_scratch_ptr[dev] || ctx == 0 || ctx != g_ctx_id[dev]) {
        int major = 0, count = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        if (major != 10) return NVFP4_ERR_DEVICE;
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return NVFP4_ERR_CUDA;
        g_sm_count[dev] = count;
        g_scratch_ptr[dev] = static_cast<uint32_t*>(p);
        g_ctx_id[dev] = current_context_id();
    }
    *ptr = g_scratch_ptr[dev];
    *sms = g_sm_count[dev];
    return NVFP4_OK;
}

bool is_aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" int nvfp4_quantize_noalloc(const void* x, int64_t rows, int64_t cols, int block_mode,
                                      int rounding, uint64_t seed, uint8_t* packed,
                                      uint8_t* scales, float* tensor_scale,
                                      nvfp4_stream_t stream) {
    static_assert(kNeededBytes <= kScratchBytes, "scratch array smaller than one call needs");
    if (!x || !packed || !scales || !tensor_scale) return NVFP4_ERR_ARG;
    if (block_mode != NVFP4_BLOCK_1X16 && block_mode != NVFP4_BLOCK_16X16) return NVFP4_ERR_ARG;
    if (rounding != NVFP4_ROUND_RNE && rounding != NVFP4_ROUND_SR) return NVFP4_ERR_ARG;
    if (rows < 1 || cols < 16 || cols % 16 != 0) return NVFP4_ERR_SHAPE;
    if (block_mode == NVFP4_BLOCK_16X16 && (rows % 16 != 0 || rows > kMaxTileRows)) return NVFP4_ERR_SHAPE;
    // the scratch this call needs must fit the static array (it needs the same 64
    // bytes for every tensor size today; a larger need is refused, not truncated)
    const size_t needed = kNeededBytes;
    if (needed > kScratchBytes) return NVFP4_ERR_WORKSPACE;
    if (!is_aligned(x, 16) || !is_aligned(packed, 16) || !is_aligned(scales, 16) ||
        !is_aligned(tensor_scale, 4))
        return NVFP4_ERR_ALIGN;
    uint32_t* words = nullptr;
    int sms = 0;
    int rc = scratch_for_current_device(&words, &sms);
    if (rc) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // the amax words accumulate with atomicMax and the status word keeps the first
    // error, so both must start at zero: clear them on this call's stream
    if (cudaMemsetAsync(words, 0, kNeededBytes, st) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (launch_amax(static_cast<const uint16_t*>(x), rows, cols, false, 0u, words, sms, st) !=
        cudaSuccess)
        return NVFP4_ERR_CUDA;
    QuantParams p = {};
    p.x = static_cast<const uint16_t*>(x);
    p.rows = rows;
    p.cols = cols;
    p.row_data = packed;
    p.row_sf = scales;
    p.row_g = tensor_scale;
    p.amax_words = words;
    p.status = reinterpret_cast<int*>(words + kStatusWord);
    p.seed = seed;
    p.row_sr = rounding == NVFP4_ROUND_SR;
    cudaError_t e = (block_mode == NVFP4_BLOCK_1X16) ? launch_quant_rows(p, sms, st)
                                                     : launch_quant_tile(p, true, sms, st);
    if (e != cudaSuccess) return NVFP4_ERR_CUDA;
    if (launch_sf_pad(scales, rows, cols / 16, sms, st) != cudaSuccess) return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}
