// Building blocks of the tcgen05 projection kernels: the tile shape, the
// instruction and shared-memory descriptors of a bf16 x bf16 -> fp32
// tcgen05.mma with 128-byte-swizzled K-major operands, the MMA / commit /
// tensor-memory-load instructions, and the host-side helpers that encode the
// TMA tensor maps and launch the row-statistics pass.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "qkn_common.cuh"

namespace qkn {
namespace gemm {

constexpr int BM = 128, BN = 256, BK = 64;             // bf16: BK * 2 B = one 128-byte swizzle row
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;                    // 16 KiB
constexpr int B_BYTES = BN * BK * 2;                    // 32 KiB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int UMMA_K = 16;                              // K of one kind::f16 MMA
constexpr int ACC_COLS = BN;                            // fp32 accumulator: one column per n
constexpr int TMEM_COLS = 2 * ACC_COLS;                 // double-buffered accumulator
static_assert(STAGE_BYTES % 1024 == 0, "stages must stay 1024-byte aligned for the 128B swizzle");

// Instruction descriptor of tcgen05.mma kind::f16: bf16 A and B (both
// K-major), fp32 accumulator, M = 128, N = 256.
constexpr uint32_t kInstrDesc = (1u << 4)                 // D format: f32
                              | (1u << 7)                 // A format: bf16
                              | (1u << 10)                // B format: bf16
                              | (0u << 15) | (0u << 16)   // A, B K-major
                              | ((uint32_t)(BN >> 3) << 17)
                              | ((uint32_t)(BM >> 4) << 24);

// Shared-memory matrix descriptor for a K-major operand stored as rows of 64
// bf16 (128 bytes) with the 128-byte swizzle: groups of 8 rows are 1024 bytes
// apart (stride byte offset); the leading byte offset is unused for this
// layout and set to 1.  Stage buffers are 1024-byte aligned, so the base
// offset field is 0.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;     // descriptor version for tcgen05
    d |= (uint64_t)2u << 61;     // swizzle mode: 128 bytes
    return d;
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(kInstrDesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 lanes x 32 consecutive fp32 columns: thread i gets row (lane base + i).
__device__ __forceinline__ void tmem_ld_32cols(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

}  // namespace gemm

// 2-D bf16 tensor [rows][inner] (inner contiguous) as a TMA tensor map: box
// of 64 (inner) x box_rows, 128-byte swizzle, out-of-range elements read as 0.
qkn_status make_tmap(CUtensorMap *m, const void *ptr, int64_t rows, int64_t inner, int box_rows);

// 2-D bf16 tensor [rows][cols] as the destination of TMA stores: box of
// 32 x 32, 64-byte swizzle (a 16-byte chunk j of staging row r sits at
// position j ^ ((r >> 1) & 3)); parts of a box outside the tensor are skipped.
qkn_status make_tmap_store(CUtensorMap *m, void *ptr, int64_t rows, int64_t cols);

// inv[m] = 1/sqrt(sum_k x[m][k]^2 / K + eps) for bf16 x [M][K] (K a multiple
// of 8, rows 16-byte aligned), on stream s.
qkn_status launch_inv_rms(const void *x, float *inv, int64_t M, int64_t K, float eps, cudaStream_t s);

// Reads (and clears) the device error word of the fused QKV + QK-Norm kernel.
qkn_status read_qkv_error(int *flag);

}  // namespace qkn
