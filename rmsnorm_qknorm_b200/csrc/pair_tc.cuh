// Building blocks of the CTA-pair projection kernel (gemm_pair.cuh): the
// pair tile shape and ring, the instruction descriptor of a bf16 tcgen05.mma
// with M = 256 over two CTAs, the CTA-pair form of the TMA load (bytes
// completing on the even CTA's barrier, each CTA loading only its own tile),
// the pair MMA and its commit.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "gemm_tc.cuh"
#include "qkn_sync.cuh"

namespace qkn {
namespace pair {

constexpr int BM = 128;                            // x rows per CTA (256 per pair)
constexpr int BN = 256;                            // columns per pair tile
constexpr int BN_CTA = 128;                        // W' rows loaded by each CTA
constexpr int BK = 64;                             // bf16: one 128-byte swizzle row
constexpr int STAGES = 6;
constexpr int A_BYTES = BM * BK * 2;               // 16 KiB
constexpr int B_BYTES = BN_CTA * BK * 2;           // 16 KiB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;     // 32 KiB per CTA
constexpr int PAIR_STAGE_BYTES = 2 * STAGE_BYTES;  // bytes completing on the even CTA's barrier
constexpr int ACC_COLS = BN;
constexpr int TMEM_COLS = 2 * ACC_COLS;            // double-buffered accumulator
constexpr int THREADS = 192;
constexpr int EPI_BYTES = 4 * 2 * 2048;            // two 32 x 32 bf16 staging tiles per epilogue warp
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 1024;  // + 1 KiB for alignment
// pair row blocks (256 rows) walked together down each column block: W'
// then streams from DRAM once per group (16: 353 MB read per 8192-row
// launch against 493 MB with 8, at the same speed)
constexpr int GROUP_M = 16;

static_assert(STAGE_BYTES % 1024 == 0, "stages must stay 1024-byte aligned for the 128B swizzle");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

// kind::f16 instruction descriptor: bf16 A and B (both K-major), fp32 D,
// M = 256 (the pair), N = 256.
constexpr uint32_t kInstrDesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                ((uint32_t)(2 * BM >> 4) << 24);

// 2-D tensor copy into this CTA's shared memory whose bytes complete on the
// barrier at shared::cluster address `bar` (the even CTA's).  The copy
// writes this CTA's shared memory only.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar) : "memory");
}

__device__ __forceinline__ void umma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(kInstrDesc), "r"(accumulate));
}

// Arrives on the barrier at shared::cluster address `bar` once every MMA
// this thread issued so far has completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(bar) : "memory");
}

}  // namespace pair
}  // namespace qkn
