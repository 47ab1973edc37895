// gemm.cu -- block-scaled NVFP4 GEMM on the sm_100a 5th-generation tensor cores.
//
// D[m][n] = alpha * gA * gB * sum_k a[m][k] * b[n][k], with a, b the decoded
// E2M1 codes times their E4M3 16-element block scales, fp32 accumulation.  The
// fprop, dgrad and wgrad GEMMs of the NVFP4 linear layer all take this form
// ("NVIDIA's 4-bit floating point pushes AI training limits", artiverse.ca).
//
// Design: a persistent kernel, one CTA per SM, 448 threads; CTA c computes the
// 128 x BN output tiles c, c + gridDim.x, ... in turn.
//   warp 0 lane 0   TMA producer: A/B tiles (128-byte swizzled K-major boxes of
//                   256 FP4 along K) and the matching 512-byte scale atoms
//                   (bulk copies) into a STAGES-deep shared-memory ring, running
//                   ahead across tile boundaries.
//   warps 2-5       scale writers: copy each stage's scale atoms from shared memory
//                   into a 4-deep ring of TMEM scale regions with tcgen05.st (each
//                   warp its 32-lane quadrant, every quadrant a full copy), so the
//                   tensor pipe spends no cycles on scale copies.
//   warp 1 lane 0   MMA issuer: four tcgen05.mma kind::mxf4nvf4 block_scale
//                   (K = 64 each) per stage into the fp32 accumulator in TMEM;
//                   one tcgen05.commit per stage frees the stage (and with it the
//                   scale region of the same index), and a commit per tile hands
//                   the accumulator to the epilogue.
//   warps 6-13      epilogue: two warps per TMEM quadrant, 128 columns each; they
//                   drain the accumulator into registers (scaled by alpha*gA*gB and
//                   rounded to bf16), release TMEM so the next tile's MMAs start,
//                   then write the tile through a swizzled shared-memory buffer
//                   with bulk tensor stores while the next tile's mainloop runs.
// Every wait is bounded: after ~1 s the kernel records NVFP4_ERR_TIMEOUT in the
// status word, stops issuing work, drains its own copies and frees TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace nvfp4 {

constexpr int kBM = 128;         // rows of A per tile (MMA M)
constexpr int kBKBytes = 128;    // bytes of K per stage per row (256 FP4)
constexpr int kKStep = 64;       // FP4 elements per MMA

// ---------------------------------------------------------------- PTX wrappers
// After a timeout: spin ~`cycles` so that mbarrier arrivals already on their way
// between the two CTAs of a pair land before either CTA can leave.
__device__ __forceinline__ void settle(long long cycles) {
    const long long t0 = clock64();
    while (clock64() - t0 < cycles) {
    }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(map), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}
// Write 16 / 32 consecutive TMEM columns of this warp's 32 lanes (lane i: row i of
// the quadrant), then wait for the writes to land.
__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tc_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X"
        " [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
        : "memory");
}

// The four K = 64 MMAs of one 256-deep k-tile in one statement: descriptors
// advance by 32 bytes (2 in the >> 4 address field), the A scales by 4 TMEM
// columns and the B scales by 4 * G columns per step; only the first MMA takes
// `accumulate` (0 on the first k-tile of a tile), the rest always accumulate.
template <int G>
__device__ __forceinline__ void tc_mma_nvf4_x4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        ".reg .b64 a1, a2, a3, b1, b2, b3;\n\t"
        ".reg .b32 sa1, sa2, sa3, sb1, sb2, sb3;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "setp.eq.b32 q, %3, %3;\n\t"
        "add.s64 a1, %1, 2;\n\tadd.s64 a2, %1, 4;\n\tadd.s64 a3, %1, 6;\n\t"
        "add.s64 b1, %2, 2;\n\tadd.s64 b2, %2, 4;\n\tadd.s64 b3, %2, 6;\n\t"
        "add.u32 sa1, %4, 4;\n\tadd.u32 sa2, %4, 8;\n\tadd.u32 sa3, %4, 12;\n\t"
        "add.u32 sb1, %5, %7;\n\tadd.u32 sb2, %5, %8;\n\tadd.u32 sb3, %5, %9;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], a1, b1, %3, [sa1], [sb1], q;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], a2, b2, %3, [sa2], [sb2], q;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], a3, b3, %3, [sa3], [sb3], q;\n\t"
        "}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate), "n"(4 * G),
        "n"(8 * G), "n"(12 * G)
        : "memory");
}

// MXFP4 (kMx): E2M1 operands with UE8M0 scales over 32-element blocks
// (block_scale.scale_vec::2X).  A 512-byte scale atom holds 4 blocks of 32 per row,
// i.e. two K = 64 steps; the instruction descriptor's scale-factor ids (bits 29-30
// for A, 4-5 for B) pick the byte pair of the step: 0 for the first, 2 for the
// second.  The four steps of a k-tile read atoms 0, 0, 1, 1.
__device__ __forceinline__ void tc_mma_mx(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::2X"
        " [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ uint32_t mx_sf_id(uint32_t idesc, uint32_t id) {
    return idesc | (id << 29) | (id << 4);
}
// The four K = 64 steps of one MX k-tile in one statement: scale ids 0, 2, 0, 2
// (idesc0 / idesc2), A scales advancing by 4 and B scales by 4 * G columns after the
// second step.
template <int G>
__device__ __forceinline__ void tc_mma_mx_x4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc0,
                                             uint32_t idesc2, uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        ".reg .b64 a1, a2, a3, b1, b2, b3;\n\t"
        ".reg .b32 sa2, sb2;\n\t"
        "setp.ne.b32 p, %7, 0;\n\t"
        "setp.eq.b32 q, %3, %3;\n\t"
        "add.s64 a1, %1, 2;\n\tadd.s64 a2, %1, 4;\n\tadd.s64 a3, %1, 6;\n\t"
        "add.s64 b1, %2, 2;\n\tadd.s64 b2, %2, 4;\n\tadd.s64 b3, %2, 6;\n\t"
        "add.u32 sa2, %5, 4;\n\tadd.u32 sb2, %6, %8;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], p;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::2X [%0], a1, b1, %4, [%5], [%6], q;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::2X [%0], a2, b2, %3, [sa2], [sb2], q;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::2X [%0], a3, b3, %4, [sa2], [sb2], q;\n\t"
        "}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc0), "r"(idesc2), "r"(sfa), "r"(sfb), "r"(accumulate), "n"(4 * G)
        : "memory");
}

// Bulk tensor store of a shared-memory box to global memory (async proxy), and
// its completion groups: .read waits until the source buffer may be reused.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
                 "r"(src), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Generic-proxy shared-memory writes made visible to the async proxy (TMA).
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t x, uint32_t y, uint32_t z,
                                             uint32_t w) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(x), "r"(y), "r"(z), "r"(w)
                 : "memory");
}

// Shared-memory matrix descriptor (tcgen05 format): start address, leading and
// stride byte offsets (all >> 4), descriptor version 1, layout type.
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                               uint32_t layout) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}
// K-major operand with 128-byte swizzle: 8-row x 128-byte atoms, 1024 B apart.
__device__ __forceinline__ uint64_t operand_desc(uint32_t saddr) {
    return make_sdesc(saddr, 16, 1024, 2);
}
// Instruction descriptor of kind::mxf4nvf4 block-scaled MMA: E2M1 A and B
// (format 1), K-major both, UE4M3 scales (scale format 0), M = 128, N = BN,
// K = 64 per instruction, dense.
template <int BN, bool kMx = false>
__host__ __device__ constexpr uint32_t nvf4_idesc() {
    return (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((kMx ? 1u : 0u) << 23) |
           ((uint32_t)(kBM >> 4) << 24);
}

// ---------------------------------------------------------------- shared memory
template <int BN, int STAGES>
struct __align__(1024) GemmSmem {
    uint8_t a[STAGES][kBM * kBKBytes];          // 16 KB / stage
    uint8_t b[STAGES][BN * kBKBytes];           // BN * 128 B / stage
    uint8_t dstage[8][32 * 32];                 // per epilogue warp: 32 rows x 16 bf16, 32B-swizzled
    uint8_t sfa[STAGES][4 * 512];               // 4 atoms: 128 rows x 16 blocks
    uint8_t sfb[STAGES][(BN / 128) * 4 * 512];  // per 128-row group, 4 atoms
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t sf_full[4];   // scale region r written (4 scale-writer warps arrive)
    uint64_t acc_full;   // accumulator of the current tile complete (MMA commit)
    uint64_t acc_empty;  // accumulator drained by the 8 epilogue warps
    uint64_t drain;      // after a timeout: every MMA issued so far complete
    uint32_t tmem_base;
};

template <int BN>
struct TmemLayout {
    static constexpr int kSfaCols = 16;                   // 4 k-steps x 4 columns
    static constexpr int kSfbCols = 4 * 4 * (BN / 128);   // 4 k-steps x 4 columns per group
    static constexpr int kRegion = kSfaCols + kSfbCols;   // scales of one stage
    static constexpr int kRegions = 4;                    // ring of scale regions
    static constexpr int kUsed = BN + kRegions * kRegion; // accumulator + scale ring
    static constexpr int kAlloc = kUsed <= 32 ? 32 : kUsed <= 64 ? 64 : kUsed <= 128 ? 128
                                : kUsed <= 256 ? 256 : 512;
};

// ---------------------------------------------------------------- epilogue
// 32 consecutive TMEM columns of this warp's 32 lanes (lane = row), one register
// each; the values are valid after tmem_wait_ld.
__device__ __forceinline__ void tmem_ld_32cols(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}
// Wait for this thread's TMEM loads; the registers of `r` pass through the wait so
// that no use of them is scheduled before it.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
                   "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]),
                   "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]),
                   "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]),
                   "+r"(r[31])
                 :
                 : "memory");
}
// One epilogue warp's share of a finished tile: its 32 TMEM lanes (rows row0 ..
// row0+31 of D, lane = row) by CW columns from col0; nothing is stored unless
// `store`, and `zero` writes zeros without reading the accumulator.  Drains the accumulator into
// registers (times alpha, rounded to bf16; the fp32 checking output is stored
// before the release), arrives on the accumulator-empty barrier (local, or the
// leader's at a cluster address when `remote`), then writes the bf16 tile 32 rows x 16 columns
// at a time through this warp's 1 KB buffer: 16-byte half j of a row at half
// j ^ ((row / 4) % 2), the 32-byte swizzle the store's tensor map undoes
// (conflict-free), one bulk tensor store each; rows and columns past M and N are
// clipped by the tensor map.
template <int CW>
__device__ __forceinline__ void epilogue_tile(uint32_t lane_base, int64_t row0, int64_t col0,
                                              const GemmParams& p, float alpha, bool store, bool zero,
                                              uint32_t acc_empty, uint32_t remote, uint32_t buf,
                                              const CUtensorMap* tmD) {
    constexpr int HC = CW;
    const int lane = threadIdx.x & 31;
    const int64_t row = row0 + lane;
    uint32_t packed[HC / 2];  // bf16 pairs of this thread's row
#pragma unroll
    for (int c = 0; c < HC / 32; ++c) {
        if (zero) {  // a tile with an empty reduction: D = 0, the accumulator is not read
#pragma unroll
            for (int i = 0; i < 16; ++i) packed[c * 16 + i] = 0u;
            continue;
        }
        uint32_t r[32];
        tmem_ld_32cols(lane_base + (uint32_t)(c * 32), r);
        tmem_wait_ld(r);
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(__uint_as_float(r[i]), alpha);
        if (p.D_f32 && store && row < p.M) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const int64_t col = col0 + c * 32 + 8 * g;
                if (col >= p.N) break;
                float4* d = reinterpret_cast<float4*>(p.D_f32 + row * p.N + col);
                d[0] = make_float4(v[8 * g], v[8 * g + 1], v[8 * g + 2], v[8 * g + 3]);
                d[1] = make_float4(v[8 * g + 4], v[8 * g + 5], v[8 * g + 6], v[8 * g + 7]);
            }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            packed[c * 16 + i] = *reinterpret_cast<const uint32_t*>(&h);
        }
    }
    // accumulator drained: the next tile's MMAs may overwrite it
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
        // a peer CTA's arrival needs no cluster-scope release: tcgen05.wait::ld
        // has completed the reads of the accumulator it announces
        if (remote)
            asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(acc_empty)
                         : "memory");
        else
            mbar_arrive(acc_empty);
    }
    if (p.D_bf16 && store) {
        const uint32_t sw = (uint32_t)((lane >> 2) & 1);
#pragma unroll
        for (int h = 0; h < HC / 16; ++h) {
            if (col0 + 16 * h >= p.N) break;
            if (lane == 0) bulk_wait_read_all();  // the previous store has read the buffer
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 2; ++j)
                st_shared_v4(buf + (uint32_t)lane * 32u + (((uint32_t)j ^ sw) << 4),
                             packed[8 * h + 4 * j], packed[8 * h + 4 * j + 1],
                             packed[8 * h + 4 * j + 2], packed[8 * h + 4 * j + 3]);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_2d(tmD, buf, (int)(col0 + 16 * h), (int)row0);
                bulk_commit();
            }
        }
    }
}

constexpr int kGemmThreads = 448;

// Operands and result of one 128 x BN output tile (see GemmParams' group modes).
struct TileJob {
    int64_t a_row, b_row, d_row, n0;  // first A / B / D row, first D column
    int64_t k0, k_len;                // reduction range
    int64_t bk0;                      // extra reduction offset into B
    int group;                        // -1 when not grouped
    bool valid;                       // the tile's first row lies inside its problem
};
template <int BN>
__device__ __forceinline__ TileJob tile_job(const GemmParams& p, int64_t tile, int64_t tiles_n,
                                            int64_t tiles_per_group) {
    TileJob j;
    const int64_t t = p.group_mode == 2 ? tile % tiles_per_group : tile;
    const int64_t m0 = (t / tiles_n) * kBM;
    j.n0 = (t % tiles_n) * BN;
    j.a_row = m0;
    j.b_row = j.n0;
    j.d_row = m0;
    j.k0 = 0;
    j.k_len = p.K;
    j.bk0 = 0;
    j.group = -1;
    j.valid = m0 < p.M;
    if (p.group_mode == 1) {
        j.group = p.mtile_group[m0 / kBM];
        j.b_row = (int64_t)j.group * p.b_group_rows + j.n0;
        j.bk0 = (int64_t)j.group * p.b_group_k;
    } else if (p.group_mode == 2) {
        j.group = (int)(tile / tiles_per_group);
        j.k0 = p.k_start[j.group];
        j.k_len = p.k_len[j.group];
        j.d_row = (int64_t)j.group * p.M + m0;
    }
    return j;
}

template <int BN, int STAGES, bool kMx>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_nvf4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmD, const GemmParams p) {
    using Smem = GemmSmem<BN, STAGES>;
    using TL = TmemLayout<BN>;
    constexpr int R = TL::kRegions;
    constexpr int G = BN / 128;  // 128-row groups of B per tile
    static_assert(R == STAGES, "scale regions are freed with their shared-memory stage");
    extern __shared__ uint8_t smem_raw[];
    Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // scale atoms per 128-row group of A and of B (an atom covers 64, or for MX 128,
    // reduction elements)
    constexpr int64_t kAtomK = kMx ? 128 : 64;
    const int64_t katoms = (p.K + kAtomK - 1) / kAtomK;
    const int64_t katoms_b = ((p.Kb ? p.Kb : p.K) + kAtomK - 1) / kAtomK;
    const int64_t nb_groups = (p.N + 127) / 128;     // 128-row groups of B (per group)
    const int64_t tiles_n = (p.N + BN - 1) / BN;
    const int64_t tiles_per_group = ((p.M + kBM - 1) / kBM) * tiles_n;
    const int64_t tiles = p.group_mode == 2 ? tiles_per_group * p.num_groups : tiles_per_group;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_addr(&S.full[s]), 1);
            mbar_init(smem_addr(&S.empty[s]), 1);
        }
        for (int r = 0; r < R; ++r) {
            mbar_init(smem_addr(&S.sf_full[r]), 4);
        }
        mbar_init(smem_addr(&S.acc_full), 1);
        mbar_init(smem_addr(&S.acc_empty), 8);
        mbar_init(smem_addr(&S.drain), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(&S.tmem_base)),
                     "r"((uint32_t)TL::kAlloc)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    __shared__ int timed_out;
    if (threadIdx.x == 0) timed_out = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const long long budget = p.wait_cycles > 0 ? p.wait_cycles : kWaitCycles;
    int64_t it = 0;  // producer thread: k-tiles whose copies it issued (all tiles)

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            for (int64_t tile = blockIdx.x; tile < tiles && !*(volatile int*)&timed_out; tile += gridDim.x) {
                const TileJob jb = tile_job<BN>(p, tile, tiles_n, tiles_per_group);
                const int KTt = (int)((jb.k_len + 255) / 256);
                for (int kt = 0; kt < KTt; ++kt, ++it) {
                    const int s = (int)(it % STAGES);
                    const uint32_t use = (uint32_t)(it / STAGES);
                    if (it >= STAGES && !mbar_wait(smem_addr(&S.empty[s]), (use & 1u) ^ 1u, budget)) {
                        timed_out = 1;
                        break;
                    }
                    const int64_t rem = (jb.k_len - (int64_t)kt * 256) / kKStep;
                    const int nks = rem < 4 ? (int)rem : 4;
                    const uint32_t sf_bytes = (uint32_t)(kMx ? (nks + 1) / 2 : nks) * 512u;
                    uint32_t bytes = kBM * kBKBytes + BN * kBKBytes + sf_bytes;
                    for (int g = 0; g < G; ++g)
                        if (jb.n0 / 128 + g < nb_groups) bytes += sf_bytes;
                    const uint32_t fb = smem_addr(&S.full[s]);
                    const int64_t katom = (jb.k0 + (int64_t)kt * 256) / kAtomK;  // first scale atom of the k-tile
                    mbar_expect_tx(fb, bytes);
                    tma_load_2d(smem_addr(S.a[s]), &tmA, (int)((jb.k0 / 2) + kt * kBKBytes), (int)jb.a_row, fb);
                    tma_load_2d(smem_addr(S.b[s]), &tmB, (int)((jb.bk0 + jb.k0) / 2 + kt * kBKBytes), (int)jb.b_row, fb);
                    bulk_load(smem_addr(S.sfa[s]), p.sfA + ((jb.a_row / 128) * katoms + katom) * 512,
                              sf_bytes, fb);
                    for (int g = 0; g < G; ++g)
                        if (jb.n0 / 128 + g < nb_groups)
                            bulk_load(smem_addr(S.sfb[s] + g * 2048),
                                      p.sfB + ((jb.b_row / 128 + g) * katoms_b + jb.bk0 / kAtomK + katom) * 512,
                                      sf_bytes, fb);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            // The block-scaled MMA does not queue ahead of its issuing thread:
            // every instruction this thread runs between two MMAs idles the
            // tensor pipe.  So the loop keeps stage, phase and descriptors in
            // registers and waits on one barrier per k-tile: the scale writers
            // arrive on sf_full only after they saw the stage's bytes land.
            constexpr uint32_t idesc = nvf4_idesc<BN, kMx>();
            constexpr uint64_t kAStep = (kBM * kBKBytes) >> 4, kBStep = (BN * kBKBytes) >> 4;
            const uint64_t adesc0 = operand_desc(smem_addr(S.a[0]));
            const uint64_t bdesc0 = operand_desc(smem_addr(S.b[0]));
            const uint32_t tsf0 = tmem + (uint32_t)BN;
            const uint32_t sf_full0 = smem_addr(&S.sf_full[0]), empty0 = smem_addr(&S.empty[0]);
            uint32_t s = 0, ph = 0;                 // stage (= scale region) and its phase
            uint32_t local = 0;  // tiles of this CTA so far
            for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++local) {
                const TileJob jb = tile_job<BN>(p, tile, tiles_n, tiles_per_group);
                const int KT = (int)((jb.k_len + 255) / 256);
                const int KT_full = (int)(jb.k_len / 256);  // k-tiles with all four K = 64 steps
                // the epilogue has drained the accumulator of the previous tile
                if (local > 0 && !mbar_wait(smem_addr(&S.acc_empty), (local - 1) & 1u, budget)) {
                    timed_out = 1;
                    break;
                }
                tc_fence_after();
                bool bad = false;
                for (int kt = 0; kt < KT; ++kt) {
                    if (!mbar_wait(sf_full0 + 8u * s, ph, budget)) {
                        bad = true;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = adesc0 + kAStep * s, bd = bdesc0 + kBStep * s;
                    const uint32_t t_sfa = tsf0 + (uint32_t)TL::kRegion * s;
                    const uint32_t t_sfb = t_sfa + TL::kSfaCols;
                    if (kMx && kt < KT_full) {
                        tc_mma_mx_x4<G>(tmem, ad, bd, mx_sf_id(idesc, 0u), mx_sf_id(idesc, 2u), t_sfa, t_sfb,
                                        kt > 0 ? 1u : 0u);
                    } else if (kMx) {  // K tail: 1 to 3 steps of 64
                        const int nks = (int)((jb.k_len - (int64_t)kt * 256) / kKStep);
                        for (int j = 0; j < nks; ++j)
                            tc_mma_mx(tmem, ad + 2u * j, bd + 2u * j, mx_sf_id(idesc, 2u * (j & 1)),
                                      t_sfa + 4 * (j >> 1), t_sfb + 4 * G * (j >> 1),
                                      (kt > 0 || j > 0) ? 1u : 0u);
                    } else if (kt < KT_full) {
                        tc_mma_nvf4_x4<G>(tmem, ad, bd, idesc, t_sfa, t_sfb, kt > 0 ? 1u : 0u);
                    } else {  // K tail: 1 to 3 steps of 64
                        const int nks = (int)((jb.k_len - (int64_t)kt * 256) / kKStep);
                        for (int j = 0; j < nks; ++j)
                            tc_mma_nvf4(tmem, ad + 2u * j, bd + 2u * j, idesc, t_sfa + 4 * j,
                                        t_sfb + 4 * G * j, (kt > 0 || j > 0) ? 1u : 0u);
                    }
                    tc_commit(empty0 + 8u * s);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                tc_commit(smem_addr(&S.acc_full));
                if (bad) {
                    timed_out = 1;
                    break;
                }
            }
        }
        __syncwarp();
    } else if (warp < 6) {
        // ---------------------------------------------------- scale writers (warps 2-5)
        // TMEM quadrant q = warp % 4 (lanes 32q .. 32q+31).  Scale atom j of a
        // stage holds, in 16-byte line l, the 4-block scales of rows l, l+32, l+64,
        // l+96; lane l of every quadrant gets line l in 4 consecutive columns, the
        // layout the block-scaled MMA reads (row l + 32i in column i).
        const int q = warp & 3;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        int64_t it = 0;
        bool stop = false;
        for (int64_t tile = blockIdx.x; tile < tiles && !stop; tile += gridDim.x)
        for (int kt = (int)((tile_job<BN>(p, tile, tiles_n, tiles_per_group).k_len + 255) / 256); kt > 0; --kt, ++it) {
            const int s = (int)(it % STAGES), r = (int)(it % R);
            // Region r was last read by the MMAs of k-tile it - R.  With R == STAGES
            // those MMAs completed before the producer could refill stage s (it
            // waited for their commit), so the arrival of k-tile it in stage s
            // also means that region r is free.
            if (!mbar_wait(smem_addr(&S.full[s]), (uint32_t)(it / STAGES) & 1u, budget)) {
                timed_out = 1;
                stop = true;
                break;
            }
            tc_fence_after();
            const uint32_t col = (uint32_t)(BN + r * TL::kRegion);
            uint32_t v[16];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 w = *reinterpret_cast<const uint4*>(S.sfa[s] + j * 512 + lane * 16);
                v[4 * j] = w.x; v[4 * j + 1] = w.y; v[4 * j + 2] = w.z; v[4 * j + 3] = w.w;
            }
            tc_st16(lane_base + col, v);
#pragma unroll
            for (int h = 0; h < G; ++h) {  // 16 columns: k-steps and groups, order 4*G*j + 4*g
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int idx = h * 4 + jj;
                    const int j = idx / G, g = idx % G;
                    const uint4 w = *reinterpret_cast<const uint4*>(S.sfb[s] + g * 2048 + j * 512 + lane * 16);
                    v[4 * jj] = w.x; v[4 * jj + 1] = w.y; v[4 * jj + 2] = w.z; v[4 * jj + 3] = w.w;
                }
                tc_st16(lane_base + col + TL::kSfaCols + 16 * h, v);
            }
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&S.sf_full[r]));
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------- epilogue (warps 6-13)
        const int q = warp & 3;                  // TMEM quadrant of this warp
        const int half = (warp - 6) >> 2;        // columns [half * BN/2, +BN/2)
        constexpr int HC = BN / 2;               // columns per epilogue warp
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(half * HC);
        uint32_t local = 0;
        for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++local) {
            if (*(volatile int*)&timed_out) break;  // a stage failed: no further tiles arrive
            const TileJob jb = tile_job<BN>(p, tile, tiles_n, tiles_per_group);
            float alpha = p.alpha;
            const int gs = jb.group < 0 ? 0 : jb.group;
            if (p.scale_a) alpha = __fmul_rn(alpha, p.scale_a[gs]);
            if (p.scale_b) alpha = __fmul_rn(alpha, p.scale_b[gs]);
            const bool acc_ok = mbar_wait(smem_addr(&S.acc_full), local & 1u, budget);
            tc_fence_after();
            __syncwarp();
            if (!acc_ok) timed_out = 1;
            // after a timeout the accumulator is neither read nor stored
            const bool bad = *(volatile int*)&timed_out != 0;
            const int64_t m_in = (jb.d_row - (jb.group >= 0 && p.group_mode == 2 ? (int64_t)jb.group * p.M : 0)) + 32 * q;
            epilogue_tile<HC>(lane_base, jb.d_row + 32 * q, jb.n0 + half * HC, p, alpha,
                              !bad && m_in < p.M, bad || jb.k_len == 0, smem_addr(&S.acc_empty), 0u,
                              smem_addr(S.dstage[warp - 6]), &tmD);
        }
        if (lane == 0) bulk_wait_all();  // every store of this warp has landed
        __syncwarp();
    }
    __syncthreads();
    // Every role has left its loop.  After a timeout some consumers stopped early,
    // so work this CTA issued may still be in flight: the producer waits for the
    // copies of its last STAGES k-tiles (earlier ones were waited for before their
    // stage was refilled), the MMA issuer commits once more and waits for that
    // commit (it arrives when every MMA issued so far has completed).  Only then
    // is TMEM freed and the CTA allowed to exit.
    if (*(volatile int*)&timed_out) {
        if (warp == 0 && lane == 0)
            for (int64_t k = (it > STAGES ? it - STAGES : 0); k < it; ++k)
                mbar_wait_drain(smem_addr(&S.full[k % STAGES]), (uint32_t)(k / STAGES) & 1u);
        if (warp == 1 && lane == 0) {
            tc_commit(smem_addr(&S.drain));
            mbar_wait_drain(smem_addr(&S.drain), 0u);
        }
        if (threadIdx.x == 0) set_status(p.status, kStatusTimeout);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"((uint32_t)TL::kAlloc)
                     : "memory");
    }
}

// ============================================================================
// Two-SM variant.  A cluster of two CTAs computes 256 x 256 output tiles with
// tcgen05.mma.cta_group::2 (M = 256, 128 rows per CTA; N = 256).  Each CTA
// loads its own 128 rows of A and its own 128 of the tile's 256 rows of B, so an
// SM streams 32 KB of operands per 256-deep k-tile instead of 48 KB, and the
// pair's MMA reads both halves of B.  The roles are those of the kernel above in
// each CTA; the leader (cluster rank 0) issues the MMAs, the operand copies of
// both CTAs complete on the leader's stage barrier, the scale writers and
// epilogue warps of both CTAs arrive on the leader's barriers, and the leader's
// commits arrive on the barriers of both CTAs.  No copy is multicast.
// ============================================================================
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on the peer's barrier without a cluster-scope release: used after
// tcgen05.wait::st, which has already completed the TMEM writes it announces.
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// Arrive (once the pair's MMAs issued so far complete) on the barrier at this
// shared-memory offset in both CTAs.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(bar),
        "h"((uint16_t)3)
        : "memory");
}
__device__ __forceinline__ void tc_mma_nvf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                 uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                                 uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X"
        " [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
        : "memory");
}
// The four K = 64 steps of one k-tile, as tc_mma_nvf4_x4 (N = 256: B scales
// advance by 8 columns per step).
__device__ __forceinline__ void tc_mma_nvf4_pair_x4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                    uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                                    uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        ".reg .b64 a1, a2, a3, b1, b2, b3;\n\t"
        ".reg .b32 sa1, sa2, sa3, sb1, sb2, sb3;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "setp.eq.b32 q, %3, %3;\n\t"
        "add.s64 a1, %1, 2;\n\tadd.s64 a2, %1, 4;\n\tadd.s64 a3, %1, 6;\n\t"
        "add.s64 b1, %2, 2;\n\tadd.s64 b2, %2, 4;\n\tadd.s64 b3, %2, 6;\n\t"
        "add.u32 sa1, %4, 4;\n\tadd.u32 sa2, %4, 8;\n\tadd.u32 sa3, %4, 12;\n\t"
        "add.u32 sb1, %5, 8;\n\tadd.u32 sb2, %5, 16;\n\tadd.u32 sb3, %5, 24;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], a1, b1, %3, [sa1], [sb1], q;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], a2, b2, %3, [sa2], [sb2], q;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], a3, b3, %3, [sa3], [sb3], q;\n\t"
        "}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
        : "memory");
}
// Pair MMA: M = 256 (both CTAs), N = 256, E2M1 x E2M1, UE4M3 scales, K-major.
constexpr uint32_t kIdescPair = (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) |
                                ((uint32_t)(256 >> 4) << 24);

// Epilogue warps of the pair kernel (EW, a template parameter): EW / 4 per TMEM lane
// quarter, each draining 256 / (EW / 4) columns of its 32 rows.  Sixteen release the
// accumulator sooner, which pays where tiles are short (the grouped GEMMs, 4-8 k-tiles
// per tile: MoE step 0.986 -> 0.976 ms); on the long dense tiles the extra waiting
// warps cost more than they save (MLP GEMMs 0.996 -> 1.020 ms), so those keep eight.
constexpr int kPairEpiWarpsMax = 16;
template <int EW>
constexpr int pair_threads() {
    return (6 + EW + 1) * 32;  // producer, issuer, 4 scale writers, epilogue, scale producer
}

template <int STAGES, int EW>
struct __align__(1024) PairSmem {
    uint8_t a[STAGES][128 * kBKBytes];       // this CTA's 128 rows of A, 16 KB / stage
    uint8_t b[STAGES][128 * kBKBytes];       // this CTA's 128 rows of B, 16 KB / stage
    uint8_t dstage[EW][32 * 32];             // per epilogue warp: 32 rows x 16 bf16, 32B-swizzled
    uint8_t sfa[STAGES][4 * 512];            // scales of this CTA's A rows
    uint8_t sfb[STAGES][2][4 * 512];         // scales of all 256 B rows of the tile
    uint64_t full[STAGES];       // this CTA's A/B boxes landed
    uint64_t sf_loaded[STAGES];  // this CTA's scale atoms landed
    uint64_t empty[STAGES];      // stage free (leader's commit, both CTAs)
    uint64_t sf_full[STAGES];    // leader: operands landed and TMEM scales written in both CTAs (8 warps)
    uint64_t acc_full;           // accumulator ready (leader's commit, both CTAs)
    uint64_t acc_empty;          // leader: accumulators of both CTAs drained (16 warps)
    uint64_t drain;              // leader, after a timeout: every MMA issued so far complete
    uint32_t tmem_base;
};


// Operands and result of one 256 x 256 output tile of the pair kernel (the group
// modes of GemmParams; mode 1 walks the 256-row tiles of every group, whose second
// half may lie past the group's rows).
struct PairJob {
    int64_t m0;     // first A row of the tile (CTA rank r owns rows m0 + 128 r ..)
    int64_t b_row;  // first B row of the tile (rank r loads rows b_row + 128 r ..)
    int64_t n0;     // first D column
    int64_t d_row;  // first D row
    int64_t k0;     // first reduction element of A (B adds bk0)
    int64_t bk0;    // extra reduction offset into B
    int64_t k_len;  // reduction length
    int64_t rows;   // rows from m0 that belong to the tile's problem (up to 256)
    int group;      // -1 when not grouped
};

// MXFP4 (kMx): one pair MMA K step with UE8M0 scales over 32-element blocks.
__device__ __forceinline__ void tc_mma_mx_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::2X"
        " [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
        : "memory");
}

// The four K = 64 steps of one MX k-tile: an E8M0 scale atom column serves two
// steps (scale ids 0 and 2 of the same columns), so the A scales advance by 4 and
// the B scales by 8 columns every second step.  idesc0 / idesc2 carry scale ids 0 / 2.
__device__ __forceinline__ void tc_mma_mx_pair_x4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                  uint32_t idesc0, uint32_t idesc2, uint32_t sfa, uint32_t sfb,
                                                  uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        ".reg .b64 a1, a2, a3, b1, b2, b3;\n\t"
        ".reg .b32 sa2, sb2;\n\t"
        "setp.ne.b32 p, %7, 0;\n\t"
        "setp.eq.b32 q, %3, %3;\n\t"
        "add.s64 a1, %1, 2;\n\tadd.s64 a2, %1, 4;\n\tadd.s64 a3, %1, 6;\n\t"
        "add.s64 b1, %2, 2;\n\tadd.s64 b2, %2, 4;\n\tadd.s64 b3, %2, 6;\n\t"
        "add.u32 sa2, %5, 4;\n\tadd.u32 sb2, %6, 8;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], p;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::2X [%0], a1, b1, %4, [%5], [%6], q;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::2X [%0], a2, b2, %3, [sa2], [sb2], q;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::2X [%0], a3, b3, %4, [sa2], [sb2], q;\n\t"
        "}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc0), "r"(idesc2), "r"(sfa), "r"(sfb), "r"(accumulate)
        : "memory");
}

template <int STAGES, bool kMx, int EW>
__global__ void __launch_bounds__(pair_threads<EW>(), 1)
    gemm_nvf4_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmD, const GemmParams p) {
    using Smem = PairSmem<STAGES, EW>;
    constexpr int BN = 256, G = 2;
    constexpr int kEpiCols = BN / (EW / 4);  // columns per epilogue warp
    constexpr int kScaleW = 6 + EW;          // the scale-atom producer, after the epilogue warps
    static_assert(EW % 4 == 0 && EW <= kPairEpiWarpsMax, "epilogue warps: a multiple of 4, at most 16");
    constexpr int kSfaCols = 16, kRegion = 48;              // per stage: A scales, then B scales
    constexpr int kUsed = BN + STAGES * kRegion;
    static_assert(kUsed <= 512, "TMEM holds 512 columns");
    constexpr uint32_t kAlloc = 512;
    constexpr uint32_t kIdesc = kIdescPair | ((kMx ? 1u : 0u) << 23);  // UE8M0 scales for MX
    constexpr int64_t kAtomK = kMx ? 128 : 64;  // reduction elements per scale atom
    extern __shared__ uint8_t smem_raw[];
    Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int64_t katoms = (p.K + kAtomK - 1) / kAtomK;                       // per 128-row group of A
    const int64_t katoms_b = ((p.Kb ? p.Kb : p.K) + kAtomK - 1) / kAtomK;     // ... of B
    const int64_t b_rows_total = p.group_mode == 1 && p.b_group_rows ? p.b_group_rows * p.num_groups : p.N;
    const int64_t na_groups = (p.M + 127) / 128, nb_groups = (b_rows_total + 127) / 128;
    const int64_t tiles_n = (p.N + BN - 1) / BN, tiles_m = (p.M + 255) / 256;
    const int64_t tiles = p.group_mode == 1 ? p.num_pair_tiles * tiles_n
                        : p.group_mode == 2 ? tiles_m * tiles_n * p.num_groups
                                            : tiles_m * tiles_n;
    const int64_t cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
    // Tile order of the ungrouped problem (chosen on the host, pair_tile_order): 0 N
    // fastest, 1 M fastest, 2 bands of tile_band 256-row tile rows with M fastest
    // inside a band, 3 bands of tile_band tile columns with N fastest inside.
    // Grouped problems go N fastest inside each 256-row tile of a group: the
    // group's B and the tile's A rows are reused from L2.
    const int order = p.tile_order;
    const int64_t band_len = p.tile_band > 0 ? p.tile_band : 1;
    auto job_of = [&](int64_t pt) {
        PairJob j;
        j.k0 = 0;
        j.bk0 = 0;
        j.k_len = p.K;
        j.group = -1;
        if (p.group_mode == 1) {
            const int64_t t = pt / tiles_n;
            j.n0 = (pt % tiles_n) * BN;
            j.m0 = p.pair_row0[t];
            j.group = p.pair_group[t];
            j.rows = p.pair_rows[t];
            j.b_row = (int64_t)j.group * p.b_group_rows + j.n0;
            j.bk0 = (int64_t)j.group * p.b_group_k;
            j.d_row = j.m0;
            return j;
        }
        int64_t tm, tn, t = pt;
        if (p.group_mode == 2) {
            j.group = (int)(pt / (tiles_m * tiles_n));
            t = pt % (tiles_m * tiles_n);
            tm = t / tiles_n;
            tn = t % tiles_n;
            j.k0 = p.k_start[j.group];
            j.k_len = p.k_len[j.group];
        } else if (order == 0) {  // N fastest
            tm = t / tiles_n;
            tn = t % tiles_n;
        } else if (order == 1) {  // M fastest
            tm = t % tiles_m;
            tn = t / tiles_m;
        } else if (order == 2) {  // bands of tile rows, M fastest inside a band
            const int64_t band = t / (band_len * tiles_n), w = t % (band_len * tiles_n);
            const int64_t rows = tiles_m - band * band_len < band_len ? tiles_m - band * band_len : band_len;
            tm = band * band_len + w % rows;
            tn = w / rows;
        } else {  // bands of tile columns, N fastest inside a band
            const int64_t band = t / (band_len * tiles_m), w = t % (band_len * tiles_m);
            const int64_t cols = tiles_n - band * band_len < band_len ? tiles_n - band * band_len : band_len;
            tn = band * band_len + w % cols;
            tm = w / cols;
        }
        j.m0 = tm * 256;
        j.n0 = tn * BN;
        j.b_row = j.n0;
        j.rows = p.M - j.m0 < 256 ? p.M - j.m0 : 256;
        j.d_row = (j.group > 0 ? (int64_t)j.group * p.M : 0) + j.m0;
        return j;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_addr(&S.full[s]), 1);
            mbar_init(smem_addr(&S.sf_loaded[s]), 1);
            mbar_init(smem_addr(&S.empty[s]), 1);
            mbar_init(smem_addr(&S.sf_full[s]), 8);
        }
        mbar_init(smem_addr(&S.acc_full), 1);
        mbar_init(smem_addr(&S.acc_empty), 2 * EW);
        mbar_init(smem_addr(&S.drain), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(&S.tmem_base)),
                     "r"(kAlloc)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    __shared__ int timed_out;
    if (threadIdx.x == 0) timed_out = 0;
    tc_fence_before();
    cluster_sync_all();  // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const long long budget = p.wait_cycles > 0 ? p.wait_cycles : kWaitCycles;
    int64_t issued_ab = 0;  // A/B producer thread: k-tiles whose boxes it issued
    int64_t issued_sf = 0;  // scale producer thread: k-tiles whose atoms it issued

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ A/B producer (each CTA its own)
            const uint32_t empty0 = smem_addr(&S.empty[0]);
            uint32_t s = 0, ph = 0;
            for (int64_t pt = cid; pt < tiles && !*(volatile int*)&timed_out; pt += ncl) {
                const PairJob jb = job_of(pt);
                const int KT = (int)((jb.k_len + 255) / 256);
                for (int kt = 0; kt < KT; ++kt, ++issued_ab) {
                    if (issued_ab >= STAGES && !mbar_wait(empty0 + 8u * s, ph ^ 1u, budget)) {
                        timed_out = 1;
                        break;
                    }
                    // this CTA's A and B boxes (rows past the tensors are zero-filled and count)
                    const uint32_t fb = smem_addr(&S.full[s]);
                    mbar_expect_tx(fb, 2u * 128u * kBKBytes);
                    tma_load_2d(smem_addr(S.a[s]), &tmA, (int)(jb.k0 / 2 + kt * kBKBytes),
                                (int)(jb.m0 + 128 * rank), fb);
                    tma_load_2d(smem_addr(S.b[s]), &tmB, (int)((jb.bk0 + jb.k0) / 2 + kt * kBKBytes),
                                (int)(jb.b_row + 128 * rank), fb);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == kScaleW) {
        if (lane == 0) {
            // ------------------------------------------------ scale-atom producer (both CTAs)
            // One thread issuing every copy of a stage was the pipeline's limit;
            // the scale atoms have their own thread and barrier.
            const uint32_t sfl0 = smem_addr(&S.sf_loaded[0]), empty0 = smem_addr(&S.empty[0]);
            uint32_t s = 0, ph = 0;
            for (int64_t pt = cid; pt < tiles && !*(volatile int*)&timed_out; pt += ncl) {
                const PairJob jb = job_of(pt);
                const int KT = (int)((jb.k_len + 255) / 256);
                const int64_t a_group = (jb.m0 + 128 * rank) / 128;
                for (int kt = 0; kt < KT; ++kt, ++issued_sf) {
                    if (issued_sf >= STAGES && !mbar_wait(empty0 + 8u * s, ph ^ 1u, budget)) {
                        timed_out = 1;
                        break;
                    }
                    const int64_t rem = (jb.k_len - (int64_t)kt * 256) / kKStep;
                    const int nks = rem < 4 ? (int)rem : 4;
                    const uint32_t sf_bytes = (uint32_t)(kMx ? (nks + 1) / 2 : nks) * 512u;
                    const int64_t katom = (jb.k0 + (int64_t)kt * 256) / kAtomK;  // first atom of the k-tile
                    uint32_t bytes = a_group < na_groups ? sf_bytes : 0u;
                    for (int g = 0; g < G; ++g)
                        if (jb.b_row / 128 + g < nb_groups) bytes += sf_bytes;
                    const uint32_t sb = sfl0 + 8u * s;
                    mbar_expect_tx(sb, bytes);
                    if (a_group < na_groups)
                        bulk_load(smem_addr(S.sfa[s]), p.sfA + (a_group * katoms + katom) * 512, sf_bytes, sb);
                    for (int g = 0; g < G; ++g)
                        if (jb.b_row / 128 + g < nb_groups)
                            bulk_load(smem_addr(S.sfb[s][g]),
                                      p.sfB + ((jb.b_row / 128 + g) * katoms_b + jb.bk0 / kAtomK + katom) * 512,
                                      sf_bytes, sb);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------------------------ MMA issuer (leader)
            constexpr uint64_t kStep = (128 * kBKBytes) >> 4;
            const uint64_t adesc0 = operand_desc(smem_addr(S.a[0]));
            const uint64_t bdesc0 = operand_desc(smem_addr(S.b[0]));
            const uint32_t tsf0 = tmem + (uint32_t)BN;
            const uint32_t sf_full0 = smem_addr(&S.sf_full[0]), empty0 = smem_addr(&S.empty[0]);
            uint32_t s = 0, ph = 0;
            uint32_t local = 0;
            for (int64_t pt = cid; pt < tiles; pt += ncl, ++local) {
                const PairJob jb = job_of(pt);
                const int KT = (int)((jb.k_len + 255) / 256);
                const int KT_full = (int)(jb.k_len / 256);  // k-tiles with all four K = 64 steps
                if (local > 0 && !mbar_wait(smem_addr(&S.acc_empty), (local - 1) & 1u, budget)) {
                    timed_out = 1;
                    break;
                }
                tc_fence_after();
                bool bad = false;
                for (int kt = 0; kt < KT; ++kt) {
                    if (!mbar_wait(sf_full0 + 8u * s, ph, budget)) {
                        bad = true;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = adesc0 + kStep * s, bd = bdesc0 + kStep * s;
                    const uint32_t t_sfa = tsf0 + (uint32_t)kRegion * s;
                    const uint32_t t_sfb = t_sfa + kSfaCols;
                    if (!kMx && kt < KT_full) {
                        tc_mma_nvf4_pair_x4(tmem, ad, bd, kIdesc, t_sfa, t_sfb, kt > 0 ? 1u : 0u);
                    } else if (kMx && kt < KT_full) {
                        tc_mma_mx_pair_x4(tmem, ad, bd, mx_sf_id(kIdesc, 0u), mx_sf_id(kIdesc, 2u), t_sfa, t_sfb,
                                          kt > 0 ? 1u : 0u);
                    } else if (kMx) {  // K tail: 1 to 3 steps of 64
                        // an atom serves two K = 64 steps: steps 0, 1 read atom 0 (scale
                        // ids 0, 2), steps 2, 3 atom 1
                        const int nks = (int)((jb.k_len - (int64_t)kt * 256) / kKStep);
                        for (int j = 0; j < nks; ++j)
                            tc_mma_mx_pair(tmem, ad + 2u * j, bd + 2u * j, mx_sf_id(kIdesc, 2u * (j & 1)),
                                           t_sfa + 4 * (j >> 1), t_sfb + 4 * G * (j >> 1),
                                           (kt > 0 || j > 0) ? 1u : 0u);
                    } else {  // K tail: 1 to 3 steps of 64
                        const int nks = (int)((jb.k_len - (int64_t)kt * 256) / kKStep);
                        for (int j = 0; j < nks; ++j)
                            tc_mma_nvf4_pair(tmem, ad + 2u * j, bd + 2u * j, kIdesc, t_sfa + 4 * j,
                                             t_sfb + 4 * G * j, (kt > 0 || j > 0) ? 1u : 0u);
                    }
                    tc_commit_pair(empty0 + 8u * s);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                tc_commit_pair(smem_addr(&S.acc_full));
                if (bad) {
                    timed_out = 1;
                    break;
                }
            }
        }
        __syncwarp();
    } else if (warp < 6) {
        // ---------------------------------------------------- scale writers (warps 2-5, both CTAs)
        // Into this CTA's TMEM: the A scales of its own 128 rows and the B scales
        // of all 256 rows of the tile, in the layout of the one-SM kernel.  The
        // writers of each CTA also wait for that CTA's A/B boxes, so the leader's
        // sf_full (all eight writer warps) means both CTAs' operands have landed and
        // the issuer needs no other barrier.  Region s was last read by the
        // previous use of stage s, whose commit the producer waited for before
        // refilling the stage's scale atoms.
        const int q = warp & 3;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        const uint32_t sfl0 = smem_addr(&S.sf_loaded[0]), full0 = smem_addr(&S.full[0]);
        const uint32_t sf_full_local0 = smem_addr(&S.sf_full[0]);
        const uint32_t sf_full_l0 = mapa_shared(sf_full_local0, 0);
        uint32_t s = 0, ph = 0;
        bool stop = false;
        for (int64_t pt = cid; pt < tiles && !stop; pt += ncl)
        for (int kt = (int)((job_of(pt).k_len + 255) / 256); kt > 0; --kt) {
            if (!mbar_wait(sfl0 + 8u * s, ph, budget) || !mbar_wait(full0 + 8u * s, ph, budget)) {
                timed_out = 1;
                stop = true;
                break;
            }
            tc_fence_after();
            const uint32_t col = (uint32_t)(BN + kRegion * s);
            uint32_t v[16];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 w = *reinterpret_cast<const uint4*>(S.sfa[s] + j * 512 + lane * 16);
                v[4 * j] = w.x; v[4 * j + 1] = w.y; v[4 * j + 2] = w.z; v[4 * j + 3] = w.w;
            }
            tc_st16(lane_base + col, v);
#pragma unroll
            for (int h = 0; h < G; ++h) {  // 16 columns: k-steps and groups, order 4*G*j + 4*g
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int idx = h * 4 + jj;
                    const int j = idx / G, g = idx % G;
                    const uint4 w = *reinterpret_cast<const uint4*>(S.sfb[s][g] + j * 512 + lane * 16);
                    v[4 * jj] = w.x; v[4 * jj + 1] = w.y; v[4 * jj + 2] = w.z; v[4 * jj + 3] = w.w;
                }
                tc_st16(lane_base + col + kSfaCols + 16 * h, v);
            }
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader)
                    mbar_arrive(sf_full_local0 + 8u * s);
                else
                    mbar_arrive_cluster_relaxed(sf_full_l0 + 8u * s);
            }
            if (++s == STAGES) {
                s = 0;
                ph ^= 1u;
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------- epilogue (warps 6 .. 5 + EW, both CTAs)
        const int q = warp & 3;                // TMEM lane quarter
        const int part = (warp - 6) >> 2;      // columns [part * kEpiCols, + kEpiCols)
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(part * kEpiCols);
        const uint32_t acc_empty_l = leader ? smem_addr(&S.acc_empty) : mapa_shared(smem_addr(&S.acc_empty), 0);
        uint32_t local = 0;
        for (int64_t pt = cid; pt < tiles; pt += ncl, ++local) {
            if (*(volatile int*)&timed_out) break;
            const PairJob jb = job_of(pt);
            float alpha = p.alpha;
            const int gs = jb.group < 0 ? 0 : jb.group;
            if (p.scale_a) alpha = __fmul_rn(alpha, p.scale_a[gs]);
            if (p.scale_b) alpha = __fmul_rn(alpha, p.scale_b[gs]);
            const bool acc_ok = mbar_wait(smem_addr(&S.acc_full), local & 1u, budget);
            tc_fence_after();
            __syncwarp();
            if (!acc_ok) timed_out = 1;
            // after a timeout the accumulator is neither read nor stored
            const bool bad = *(volatile int*)&timed_out != 0;
            const int64_t r_in = 128 * rank + 32 * q;  // this warp's first row inside the tile
            epilogue_tile<kEpiCols>(lane_base, jb.d_row + r_in, jb.n0 + part * kEpiCols, p, alpha,
                                        !bad && r_in < jb.rows,
                              bad || jb.k_len == 0, acc_empty_l, leader ? 0u : 1u,
                              smem_addr(S.dstage[warp - 6]), &tmD);
        }
        if (lane == 0) bulk_wait_all();
        __syncwarp();
    }
    __syncthreads();
    // Every role of this CTA has left its loop.  A CTA that saw no timeout has
    // consumed every copy it issued (its scale writers waited for each stage) and,
    // on the leader, its epilogue waited for the last MMA commit.  After a timeout
    // each producer waits for the copies of its last STAGES k-tiles (they complete
    // on this CTA's own barriers), the leader's issuer commits once more and waits
    // for that commit (every MMA issued so far complete), and the CTA spins a few
    // microseconds so that arrivals already sent to the other CTA land.  Only then
    // do the two CTAs meet, free TMEM and exit.
    if (*(volatile int*)&timed_out) {
        if (warp == 0 && lane == 0)
            for (int64_t k = (issued_ab > STAGES ? issued_ab - STAGES : 0); k < issued_ab; ++k)
                mbar_wait_drain(smem_addr(&S.full[k % STAGES]), (uint32_t)(k / STAGES) & 1u);
        if (warp == kScaleW && lane == 0)
            for (int64_t k = (issued_sf > STAGES ? issued_sf - STAGES : 0); k < issued_sf; ++k)
                mbar_wait_drain(smem_addr(&S.sf_loaded[k % STAGES]), (uint32_t)(k / STAGES) & 1u);
        if (warp == 1 && lane == 0 && leader) {
            asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                             smem_addr(&S.drain))
                         : "memory");
            mbar_wait_drain(smem_addr(&S.drain), 0u);
        }
        if (threadIdx.x == 0) {
            set_status(p.status, kStatusTimeout);
            settle(20000);
        }
    }
    __syncthreads();
    tc_fence_before();
    cluster_sync_all();  // both CTAs done: no copy, MMA, commit or remote arrive pending
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kAlloc)
                     : "memory");
    }
}

// ---------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 2-D byte tensor [rows][row_bytes], box = 128 bytes x box_rows, 128-byte swizzle.
static bool make_operand_map(CUtensorMap* map, const void* base, int64_t rows, int64_t row_bytes,
                             int box_rows) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {(cuuint32_t)kBKBytes, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// bf16 output [M][N] (N % 8 == 0), box = 16 columns x 32 rows, 32-byte swizzle.
static bool make_output_map(CUtensorMap* map, void* base, int64_t M, int64_t N) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)N * 2};
    cuuint32_t box[2] = {16, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int BN, int STAGES, bool kMx>
static cudaError_t launch_gemm_cfg(const GemmParams& p, int sm_count, cudaStream_t st) {
    CUtensorMap ma, mb, md;
    const int64_t b_rows = p.group_mode == 1 && p.b_group_rows ? p.b_group_rows * p.num_groups : p.N;
    const int64_t kb = p.Kb ? p.Kb : p.K;
    if (!make_operand_map(&ma, p.A, p.M, p.K / 2, kBM) || !make_operand_map(&mb, p.B, b_rows, kb / 2, BN))
        return cudaErrorInvalidValue;
    memset(&md, 0, sizeof(md));
    const int64_t d_rows = p.group_mode == 2 ? p.M * p.num_groups : p.M;
    if (p.D_bf16 && !make_output_map(&md, p.D_bf16, d_rows, p.N)) return cudaErrorInvalidValue;
    const size_t smem = sizeof(GemmSmem<BN, STAGES>) + 1024;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gemm_nvf4_kernel<BN, STAGES, kMx>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    int64_t tiles = ((p.M + kBM - 1) / kBM) * ((p.N + BN - 1) / BN);
    if (p.group_mode == 2) tiles *= p.num_groups;
    const unsigned grid = (unsigned)(tiles < sm_count ? tiles : sm_count);
    gemm_nvf4_kernel<BN, STAGES, kMx><<<grid, kGemmThreads, smem, st>>>(ma, mb, md, p);
    return cudaGetLastError();
}

// Tile order of an ungrouped pair GEMM, for reuse of the operands in L2 (measured
// on the DRAM counters).  If the smaller operand (codes + scales) fits in a quarter
// of L2, the clusters sweep along its dimension first: it is re-read from L2 and
// the larger one streams from DRAM once.  Otherwise the tiles go in bands: a band
// of one operand (up to 40% of L2) stays resident while the other operand streams
// past it once per band; the banded operand and the band width are the ones with
// the fewer bytes read in total.
static void pair_tile_order(GemmParams& g, int64_t l2_bytes) {
    const int64_t row_bytes = g.K / 2 + g.K / 16 * (g.mx ? 1 : 2) / 2;
    const int64_t a = g.M * row_bytes, b = g.N * row_bytes;
    const int64_t tiles_m = (g.M + 255) / 256, tiles_n = (g.N + 255) / 256;
    if ((a < b ? a : b) <= l2_bytes / 4) {
        g.tile_order = g.M < g.N ? 1 : 0;
        g.tile_band = 0;
        return;
    }
    // A fifth of L2 per resident band: at two fifths (a 50 MB band of the 8192 x 20480
    // dgrad operand) the band thrashed (453 MB of DRAM traffic for a modelled 296 MB);
    // at a fifth the measured 407 MB matches the model's 414 MB.
    int64_t band = (l2_bytes / 5) / (256 * row_bytes);
    if (band < 1) band = 1;
    const int64_t bm = band < tiles_m ? band : tiles_m, bn = band < tiles_n ? band : tiles_n;
    const int64_t reads_m = a + (tiles_m + bm - 1) / bm * b;  // A bands resident, B streamed per band
    const int64_t reads_n = b + (tiles_n + bn - 1) / bn * a;
    g.tile_order = reads_m <= reads_n ? 2 : 3;
    g.tile_band = reads_m <= reads_n ? bm : bn;
}

template <int STAGES, bool kMx, int EW>
static cudaError_t launch_gemm_pair(const GemmParams& params, int sm_count, cudaStream_t st) {
    GemmParams p = params;
    if (p.group_mode == 0) {
        static int64_t l2 = 0;
        if (l2 == 0) {
            int dev = 0, v = 0;
            if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&v, cudaDevAttrL2CacheSize, dev) != cudaSuccess || v <= 0)
                v = 126 << 20;
            l2 = v;
        }
        pair_tile_order(p, l2);
    }
    CUtensorMap ma, mb, md;
    const int64_t b_rows = p.group_mode == 1 && p.b_group_rows ? p.b_group_rows * p.num_groups : p.N;
    const int64_t kb = p.Kb ? p.Kb : p.K;
    if (!make_operand_map(&ma, p.A, p.M, p.K / 2, 128) || !make_operand_map(&mb, p.B, b_rows, kb / 2, 128))
        return cudaErrorInvalidValue;
    memset(&md, 0, sizeof(md));
    const int64_t d_rows = p.group_mode == 2 ? p.M * p.num_groups : p.M;
    if (p.D_bf16 && !make_output_map(&md, p.D_bf16, d_rows, p.N)) return cudaErrorInvalidValue;
    const size_t smem = sizeof(PairSmem<STAGES, EW>) + 1024;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gemm_nvf4_pair_kernel<STAGES, kMx, EW>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    const int64_t tiles_n = (p.N + 255) / 256, tiles_m = (p.M + 255) / 256;
    const int64_t tiles = p.group_mode == 1 ? p.num_pair_tiles * tiles_n
                        : p.group_mode == 2 ? tiles_m * tiles_n * p.num_groups
                                            : tiles_m * tiles_n;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(pair_threads<EW>());
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // persistent: as many clusters as can be resident at once (an SM left over
    // in a GPC cannot host half a pair), never more than there are tiles
    static int resident = 0;
    if (resident == 0) {
        cfg.gridDim = dim3((unsigned)(2 * (sm_count / 2)));
        if (cudaOccupancyMaxActiveClusters(&resident, gemm_nvf4_pair_kernel<STAGES, kMx, EW>, &cfg) != cudaSuccess ||
            resident < 1)
            resident = sm_count / 2;
    }
    const int64_t clusters = tiles < resident ? (tiles > 0 ? tiles : 1) : resident;
    cfg.gridDim = dim3((unsigned)(2 * clusters));
    return cudaLaunchKernelEx(&cfg, gemm_nvf4_pair_kernel<STAGES, kMx, EW>, ma, mb, md, p);
}

cudaError_t launch_gemm(const GemmParams& p, int sm_count, cudaStream_t st) {
    // two-SM pairs for every problem taller than one 128-row tile, and for the grouped
    // problems (mode 1 needs its table of 256-row group tiles)
    const bool pair = sm_count >= 2 && (p.group_mode == 0 ? p.M > 128
                                        : p.group_mode == 2 || p.pair_row0 != nullptr);
    if (pair) {
        if (p.mx) return launch_gemm_pair<5, true, 8>(p, sm_count, st);
        return p.group_mode != 0 ? launch_gemm_pair<5, false, 16>(p, sm_count, st)
                                 : launch_gemm_pair<5, false, 8>(p, sm_count, st);
    }
    if (p.mx) return launch_gemm_cfg<256, 4, true>(p, sm_count, st);
    return launch_gemm_cfg<256, 4, false>(p, sm_count, st);
}

}  // namespace nvfp4
