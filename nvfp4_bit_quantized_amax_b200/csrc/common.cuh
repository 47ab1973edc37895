// common.cuh -- device helpers shared by the libnvfp4 kernels (sm_100a only).
//
// Numeric helpers implement the fixed readings of the NVFP4 encoding
// ("Nemotron NVFP4" explainer, "What NVFP4 actually is"):
//   E2M1 element codes, E4M3 block scales (bias 7, max 448), fp32 tensor scale.
// Conversions use the sm_100a cvt instructions by name; the parity tests check
// them against the CPU oracle bit for bit.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libnvfp4 kernels are written for sm_100a (B200) only"
#endif

namespace nvfp4 {

// ---------------------------------------------------------------- status codes
constexpr int kStatusNonFinite = -5;
constexpr int kStatusTimeout = -6;
constexpr int kStatusIndex = -9;
constexpr int kStatusRhtRange = -10;

// Record the first device-side error in a status word (0 = ok).
__device__ __forceinline__ void set_status(int* status, int code) {
    if (status != nullptr) atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------- bf16 / fp32
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 16-byte streaming load of data read once.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// ---------------------------------------------------------------- mbarriers, bulk copies
// Default bound of every wait on an mbarrier (clock cycles, ~1 s at 2 GHz).
constexpr long long kWaitCycles = 1ll << 31;
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait for the phase with the given parity to complete: false once
// `budget` clock cycles have passed without it.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, long long budget) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > budget) return false;
    return true;
}
// Wait, at exit after a timeout, for this CTA's own asynchronous work (copies it
// issued, MMAs it committed) to finish.  That work always completes, so the bound
// is the long default, never the (possibly short) budget of the pipeline waits.
__device__ __forceinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity) {
    (void)mbar_wait(bar, parity, kWaitCycles);
}
// Asynchronous copy of `bytes` (a multiple of 16; both addresses 16-byte aligned)
// from global to shared memory, completing as transaction bytes on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// ---------------------------------------------------------------- E2M1 / E4M3
// Eight fp32 values -> eight E2M1 codes, round-to-nearest-even with saturation
// to +-6; element i lands in bits [4i, 4i+4).
__device__ __forceinline__ uint32_t e2m1x8_rn(const float (&v)[8]) {
    uint32_t out;
    asm("{\n\t"
        ".reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t"
        "}"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
          "f"(v[7]));
    return out;
}

// fp32 t >= 0 -> E4M3 code, round-to-nearest-even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_rn_satfinite(float t) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(t));
    return (uint32_t)(r & 0xFFu);
}

// E4M3 code -> fp32 (exact).
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
    uint32_t h2;
    uint16_t c = (uint16_t)code;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// ---------------------------------------------------------------- tensor scale
// Per-tensor constants: decode scale g = amax / 2688 and encode factor
// enc = 2688 / amax (0 for an all-zero tensor, clamped to FLT_MAX).
struct TensorScale {
    float g;
    float enc;
};
__device__ __forceinline__ TensorScale tensor_scale_from_amax(float amax) {
    TensorScale s;
    s.g = __fdiv_rn(amax, 2688.0f);
    if (amax == 0.0f) {
        s.enc = 0.0f;
    } else {
        float e = __fdiv_rn(2688.0f, amax);
        s.enc = fminf(e, 3.402823466e38f);
    }
    return s;
}

// ---------------------------------------------------------------- Philox4x32-10
// Salmon et al., "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11): four
// 32-bit counter words, two key words, 10 rounds of two 32x32->64 multiplies.
struct Philox4 {
    uint32_t x, y, z, w;
};

// Philox4x32-10 with the key schedule taken from rk: round r uses
// (rk[2r], rk[2r+1]) = (k0 + r * 0x9E3779B9, k1 + r * 0xBB67AE85).  The
// schedule depends on the seed alone, so the host computes it once per launch
// and the kernels read it from their parameters.
__device__ __forceinline__ Philox4 philox4x32_10_rk(uint32_t c0, uint32_t c1, uint32_t c2,
                                                    uint32_t c3, const uint32_t (&rk)[20]) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint32_t hi0 = __umulhi(0xD2511F53u, c0), lo0 = 0xD2511F53u * c0;
        const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2), lo1 = 0xCD9E8D57u * c2;
        const uint32_t n0 = hi1 ^ c1 ^ rk[2 * r];
        const uint32_t n2 = hi0 ^ c3 ^ rk[2 * r + 1];
        c0 = n0;
        c1 = lo1;
        c2 = n2;
        c3 = lo0;
    }
    return Philox4{c0, c1, c2, c3};
}

// The Philox block of the 8 consecutive elements 8*group .. 8*group+7 of random
// stream `stream`: counter (group lo, group hi, stream, 0).  Its words serve the
// element pairs (0,2), (1,3), (4,6), (5,7), 16 bits per element (sr_codes8).
__device__ __forceinline__ Philox4 sr_draws8(const uint32_t (&rk)[20], uint32_t stream,
                                             uint64_t group) {
    return philox4x32_10_rk((uint32_t)group, (uint32_t)(group >> 32), stream, 0u, rk);
}

// ---------------------------------------------------------------- scale layout
// Byte offset of the scale of (row r, 16-block kb) in the block-scaled MMA
// layout: 512-byte atoms of 128 rows x 4 blocks; inside an atom row r sits in
// 16-byte line (r % 32) at word (r / 32), block kb at byte (kb % 4); atoms run
// along the blocks first, then by 128-row groups.  katoms = ceil(nblocks / 4).
__device__ __forceinline__ uint64_t sf_offset(int64_t r, int64_t kb, int64_t katoms) {
    const int64_t atom = (r >> 7) * katoms + (kb >> 2);
    const int64_t rr = r & 127;
    return (uint64_t)(atom * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (kb & 3));
}

}  // namespace nvfp4
