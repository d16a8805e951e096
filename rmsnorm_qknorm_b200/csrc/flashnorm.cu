// FlashNorm (Graef, arXiv 2024), abstract: RMSNorm followed by a linear layer,
// reformulated exactly as
//   (i)  W' = diag(w) W                       -- flashnorm_fold_weights (offline)
//   (ii) y  = (x W') * 1/rms(x)               -- flashnorm_proj
// The projection is a dense contraction, so it runs on the 5th-generation
// tensor cores: a persistent, warp-specialised kernel in which one warp moves
// 128x64 / 256x64 bf16 tiles with TMA into a ring of shared-memory stages, one
// thread issues tcgen05.mma into a double-buffered fp32 accumulator in tensor
// memory, and four epilogue warps read the accumulator back (tcgen05.ld),
// multiply each row by its 1/rms and store bf16.  The 1/rms vector comes from
// a small row-statistics kernel (or from the caller).
#include <atomic>
#include <cuda.h>
#include <math.h>

#include <mutex>
#include <stdlib.h>
#include <string.h>

#include "gemm_tc.cuh"
#include "pair_tc.cuh"
#include "qkn_common.cuh"
#include "qkn_sync.cuh"

namespace qkn {

// Set by any bounded device-side wait that gave up; read by qkn_check_device.
__device__ int g_device_error = 0;

// ============================================================== fold (i)

// Row-major output: W'[k][n] = w[k] * W[k][n], 8 bf16 per thread.
template <typename TW>
__global__ void __launch_bounds__(256) fold_rowmajor_kernel(const TW *__restrict__ w,
                                                            const __nv_bfloat16 *__restrict__ W,
                                                            __nv_bfloat16 *__restrict__ Wf,
                                                            int64_t K, int64_t N) {
    const int64_t total = K * N;
    for (int64_t i = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x);
         i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t k = i / N;
        Wf[i] = __float2bfloat16_rn(to_f32<TW>(w[k]) * __bfloat162float(W[i]));
    }
}

// Transposed output: W'[n][k] = w[k] * W[k][n] through a 64x64 shared tile.
constexpr int kFoldTile = 64;

template <typename TW>
__global__ void __launch_bounds__(256) fold_transpose_kernel(const TW *__restrict__ w,
                                                             const __nv_bfloat16 *__restrict__ W,
                                                             __nv_bfloat16 *__restrict__ Wf,
                                                             int64_t K, int64_t N) {
    __shared__ __nv_bfloat16 tile[kFoldTile][kFoldTile + 2];
    const int64_t k0 = (int64_t)blockIdx.y * kFoldTile, n0 = (int64_t)blockIdx.x * kFoldTile;
    const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;  // 64 x 4
    for (int r = ty; r < kFoldTile; r += 4) {
        const int64_t k = k0 + r, n = n0 + tx;
        if (k < K && n < N)
            tile[r][tx] = __float2bfloat16_rn(to_f32<TW>(w[k]) * __bfloat162float(W[k * N + n]));
    }
    __syncthreads();
    for (int r = ty; r < kFoldTile; r += 4) {
        const int64_t n = n0 + r, k = k0 + tx;
        if (n < N && k < K) Wf[n * K + k] = tile[tx][r];
    }
}

// Two bf16 of a word scaled by s in fp32 and rounded back (RNE), the same
// rounding as the element-wise fold.
__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t v, float s) {
    return pack_bf16x2(s * bf16lo(v), s * bf16hi(v));
}

// Row-major output with 16-byte accesses (N a multiple of 8, buffers 16-byte
// aligned): chunks of 8 consecutive n of one k row, four per thread and step,
// all four loads issued before any arithmetic.
template <typename TW>
__global__ void __launch_bounds__(256) fold_rowmajor_vec_kernel(const TW *__restrict__ w,
                                                                const __nv_bfloat16 *__restrict__ W,
                                                                __nv_bfloat16 *__restrict__ Wf,
                                                                int64_t K, int64_t N) {
    const int64_t cpr = N / 8, chunks = K * cpr;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i0 < chunks; i0 += 4 * stride) {
        uint4 v[4];
        float sk[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t i = i0 + u * stride;
            if (i < chunks) {
                v[u] = __ldcs(reinterpret_cast<const uint4 *>(W) + i);
                sk[u] = to_f32<TW>(w[i / cpr]);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t i = i0 + u * stride;
            if (i < chunks)
                __stcs(reinterpret_cast<uint4 *>(Wf) + i,
                       make_uint4(scale_bf16x2(v[u].x, sk[u]), scale_bf16x2(v[u].y, sk[u]),
                                  scale_bf16x2(v[u].z, sk[u]), scale_bf16x2(v[u].w, sk[u])));
        }
    }
}

// W [K][N] -> W^T [N][K] (scaled by w[k] when SCALE) through a 64 (k) x 128
// (n) tile with 16-byte global accesses; K and N multiples of 8, buffers
// 16-byte aligned.  A thread first issues its four 16-byte loads (8
// consecutive n of one k row each), then scales them and parks them as
// words in shared memory (rows of 65 words); after the barrier it gathers
// one pair of n columns over 8 consecutive k, twice, and writes two 16-byte
// chunks each time, W^T[n][k0 .. k0+7] and W^T[n+1][k0 .. k0+7] (eight
// threads cover the 128 contiguous bytes of an output row's piece).
// blockIdx.x walks the k tiles, so blocks launched together write
// neighbouring pieces of the same output rows.  Measured on B200 for 4096 x
// 12288: 64 x 64 tiles 43.3 us, 64 x 128 36.3 us (5.5 TB/s), 64 x 256 40.4
// us, 128 x 128 41.3 us.
constexpr int kTransTK = 64, kTransTN = 128;
template <typename TW, bool SCALE>
__global__ void __launch_bounds__(256) transpose_tile_kernel(const TW *__restrict__ w,
                                                             const __nv_bfloat16 *__restrict__ W,
                                                             __nv_bfloat16 *__restrict__ Wt, int64_t K, int64_t N) {
    constexpr int TK = kTransTK, TN = kTransTN, CPR = TN / 8;  // 8-column chunks per tile row
    constexpr int LOADS = TK * CPR / 256, TASKS = (TN / 2) * (TK / 8) / 256;
    __shared__ uint32_t tile[TK][TN / 2 + 1];
    const int64_t k0 = (int64_t)blockIdx.x * TK, n0 = (int64_t)blockIdx.y * TN;
    const int t = threadIdx.x;
    uint4 v[LOADS];
#pragma unroll
    for (int h = 0; h < LOADS; ++h) {
        const int idx = t + h * 256;
        const int r = idx / CPR, c = idx % CPR;  // tile row (k) and chunk of 8 n
        const int64_t k = k0 + r, n = n0 + c * 8;
        v[h] = make_uint4(0u, 0u, 0u, 0u);
        if (k < K && n < N) v[h] = __ldcs(reinterpret_cast<const uint4 *>(W + k * N + n));
    }
#pragma unroll
    for (int h = 0; h < LOADS; ++h) {
        const int idx = t + h * 256;
        const int r = idx / CPR, c = idx % CPR;
        uint4 u = v[h];
        if constexpr (SCALE) {
            if (k0 + r < K) {
                const float sk = to_f32<TW>(w[k0 + r]);
                u = make_uint4(scale_bf16x2(u.x, sk), scale_bf16x2(u.y, sk), scale_bf16x2(u.z, sk),
                               scale_bf16x2(u.w, sk));
            }
        }
        tile[r][c * 4 + 0] = u.x;
        tile[r][c * 4 + 1] = u.y;
        tile[r][c * 4 + 2] = u.z;
        tile[r][c * 4 + 3] = u.w;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < TASKS; ++h) {
        const int task = t + h * 256;
        const int p = task / (TK / 8), kc = task % (TK / 8);  // pair of n columns, chunk of 8 k
        uint32_t wd[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) wd[j] = tile[kc * 8 + j][p];
        // low halves hold column n0 + 2p, high halves column n0 + 2p + 1
        const uint4 lo = make_uint4(__byte_perm(wd[0], wd[1], 0x5410), __byte_perm(wd[2], wd[3], 0x5410),
                                    __byte_perm(wd[4], wd[5], 0x5410), __byte_perm(wd[6], wd[7], 0x5410));
        const uint4 hi = make_uint4(__byte_perm(wd[0], wd[1], 0x7632), __byte_perm(wd[2], wd[3], 0x7632),
                                    __byte_perm(wd[4], wd[5], 0x7632), __byte_perm(wd[6], wd[7], 0x7632));
        const int64_t n = n0 + 2 * p, k = k0 + kc * 8;
        if (k < K) {
            if (n < N) __stcs(reinterpret_cast<uint4 *>(Wt + n * K + k), lo);
            if (n + 1 < N) __stcs(reinterpret_cast<uint4 *>(Wt + (n + 1) * K + k), hi);
        }
    }
}

// ======================================================= row statistics

// inv[m] = 1/sqrt(sum_k x[m][k]^2 / K + eps), one warp per row, 16-byte loads
// issued 8 deep per lane before any arithmetic (a 4096-wide row is then one
// round trip).  K is a multiple of 8 and rows are 16-byte aligned (checked by
// the caller).
__global__ void __launch_bounds__(256) inv_rms_kernel(const __nv_bfloat16 *__restrict__ x,
                                                      float *__restrict__ inv, int64_t M, int64_t K,
                                                      float eps) {
    constexpr int U = 8;
    // let the projection that follows launch now: it streams x and W' through
    // its MMAs while this pass runs, and only its epilogue waits for inv
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= M) return;  // whole warp leaves together
    const uint8_t *xr = reinterpret_cast<const uint8_t *>(x + row * K);
    const int64_t nchunks = K / 8;
    float2 s2 = make_float2(0.f, 0.f);
    for (int64_t c0 = 0; c0 < nchunks; c0 += 32 * U) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t c = c0 + u * 32 + lane;
            v[u] = c < nchunks ? __ldcs(reinterpret_cast<const uint4 *>(xr + c * 16)) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const float2 p0 = make_float2(bf16lo(v[u].x), bf16hi(v[u].x));
            const float2 p1 = make_float2(bf16lo(v[u].y), bf16hi(v[u].y));
            const float2 p2 = make_float2(bf16lo(v[u].z), bf16hi(v[u].z));
            const float2 p3 = make_float2(bf16lo(v[u].w), bf16hi(v[u].w));
            s2 = __ffma2_rn(p0, p0, s2);
            s2 = __ffma2_rn(p1, p1, s2);
            s2 = __ffma2_rn(p2, p2, s2);
            s2 = __ffma2_rn(p3, p3, s2);
        }
    }
    float s = s2.x + s2.y;
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) inv[row] = rsqrtf(s / (float)K + eps);
}

// ===================================================== tcgen05 GEMM (ii)

namespace gemm {

constexpr int THREADS = 256;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue, warps 6-7 row statistics
constexpr int BAR_BYTES = 256;
constexpr int INV_BYTES = 2 * BM * 4;                   // 1/rms of the rows of both accumulator tiles
constexpr int EPI_BYTES = 4 * 2 * 2048;  // two 32x32 bf16 staging tiles per epilogue warp
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + INV_BYTES + 1024;  // + 1 KiB for alignment
constexpr int GROUP_M = 16;  // tiles are walked in groups of 16 row blocks so concurrent tiles share operands in L2

static_assert(STAGE_BYTES % 1024 == 0, "stages must stay 1024-byte aligned for the 128B swizzle");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

struct Args {
    const float *inv_rms;   // [M] given 1/rms (used when compute_inv == 0)
    float *inv_out;         // [M] optional: receives the 1/rms computed in-kernel
    __nv_bfloat16 *y;       // [M][N]
    int M, N, K;
    int m_blocks, n_blocks, k_blocks, num_tiles;
    int compute_inv;        // 1: rows' 1/rms from the x tiles streaming through shared memory
    int unit_scale;         // 1: no row scaling at all (y = x W'^T)
    float eps;
};

// Tile index -> (row block, column block), walking GROUP_M row blocks at a
// time down each column block: the ~148 tiles in flight at once then touch
// at most GROUP_M x-blocks and a handful of W'-blocks.
__device__ __forceinline__ void tile_coords(int tile, const Args &g, int &m_blk, int &n_blk) {
    const int group_tiles = GROUP_M * g.n_blocks;
    const int group = tile / group_tiles;
    const int first_m = group * GROUP_M;
    const int rows_in_group = min(g.m_blocks - first_m, GROUP_M);
    const int in_group = tile - group * group_tiles;
    m_blk = first_m + in_group % rows_in_group;
    n_blk = in_group / rows_in_group;
}

__global__ void __launch_bounds__(THREADS, 1)
flashnorm_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                      const __grid_constant__ CUtensorMap tmap_y, const Args g) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES + EPI_BYTES);
    uint64_t *full = bars, *empty = bars + STAGES;
    uint64_t *acc_full = bars + 2 * STAGES, *acc_empty = bars + 2 * STAGES + 2;
    uint64_t *stats_full = bars + 2 * STAGES + 4;
    uint64_t *drained = bars + 2 * STAGES + 6;  // every MMA this CTA issued has completed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 7);
    float *inv_buf = reinterpret_cast<float *>(smem + STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES);  // [2][BM]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&full[s]), 1);    // producer's arrive + TMA bytes
            // one tcgen05.commit, plus one arrive per statistics warp when they read x
            mbar_init(smem_u32(&empty[s]), g.compute_inv ? 3 : 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&acc_full[a]), 1);    // one tcgen05.commit
            mbar_init(smem_u32(&acc_empty[a]), 4);   // one arrive per epilogue warp
            mbar_init(smem_u32(&stats_full[a]), 2);  // one arrive per statistics warp
        }
        mbar_init(smem_u32(drained), 1);             // the MMA warp's final tcgen05.commit
        mbar_init_fence();
    }
    if (warp == 1) {  // whole warp: allocate the two accumulators in tensor memory
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        // One lane runs the ring: nothing here needs the other 31, and a
        // single-thread loop keeps the per-k-block path short.
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed = 0, armed_parity = 0;  // per stage: loads issued; parity of the phase they complete
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < g.num_tiles; tile += gridDim.x) {
                int m_blk, n_blk;
                tile_coords(tile, g, m_blk, n_blk);
                for (int kb = 0; kb < g.k_blocks; ++kb) {
                    if (!mbar_wait_fast(smem_u32(&empty[stage]), phase ^ 1u, &g_device_error)) { ok = false; break; }
                    const uint32_t fb = smem_u32(&full[stage]);
                    uint8_t *sa = smem + stage * STAGE_BYTES;
                    mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    tma_load_2d(smem_u32(sa), &tmap_x, kb * BK, m_blk * BM, fb);
                    tma_load_2d(smem_u32(sa + A_BYTES), &tmap_w, kb * BK, n_blk * BN, fb);
                    armed |= 1u << stage;
                    armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            // No copy may still be writing shared memory when the CTA exits:
            // wait (bounded) for the last phase armed on every stage.  On the
            // normal path the MMA warp consumed them all and these return at
            // once; after a wait gave up they catch loads nobody will consume.
            for (int s2 = 0; s2 < STAGES; ++s2)
                if (armed & (1u << s2)) mbar_wait(smem_u32(&full[s2]), (armed_parity >> s2) & 1u, &g_device_error);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        // One lane waits and issues.  The shared-memory descriptors of stage 0
        // are formed once; a stage or a 16-wide K step moves only their start
        // address field (address / 16, far from overflowing its 14 bits).
        if (lane == 0) {
            const uint64_t a_desc0 = sw128_kmajor_desc(smem_u32(smem));
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < g.num_tiles; tile += gridDim.x, ++it) {
                const int acc = it & 1;
                const uint32_t acc_phase = (it >> 1) & 1;
                if (!mbar_wait_fast(smem_u32(&acc_empty[acc]), acc_phase ^ 1u, &g_device_error)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
                for (int kb = 0; kb < g.k_blocks; ++kb) {
                    if (!mbar_wait_fast(smem_u32(&full[stage]), phase, &g_device_error)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t ad = a_desc0 + (uint64_t)((stage * STAGE_BYTES) >> 4);
                    const uint64_t bd = ad + (uint64_t)(A_BYTES >> 4);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k)  // K by 16 bf16 = 32 bytes inside the swizzle row
                        umma_bf16(d_tmem, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), (kb | k) != 0 ? 1u : 0u);
                    umma_commit(smem_u32(&empty[stage]));  // frees the stage once these MMAs read it
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit(smem_u32(&acc_full[acc]));  // accumulator ready
            }
            // Tensor memory is released only after every MMA issued here has
            // completed, also when a wait above gave up with MMAs in flight.
            umma_commit(smem_u32(drained));
            mbar_wait(smem_u32(drained), 0u, &g_device_error);
        }
        __syncwarp();
    } else if (warp < 6) {
        // ---------------------------------------------------------------- epilogue (warps 2..5)
        // Launched right behind the statistics pass (programmatic dependent
        // launch), only these warps wait for that pass to finish and its 1/rms
        // to be visible; the loads and MMAs above never read its output.  A
        // no-op when the kernel was launched normally.
        asm volatile("griddepcontrol.wait;" ::: "memory");
        // Each 32 x 32 block of y is staged in shared memory and written by one
        // TMA store (whole lines, instead of 16 bytes to each of 32 rows).  The
        // 64-byte swizzle puts a warp's 16-byte writes in the fewest wavefronts;
        // a warp's two staging buffers alternate, and one is rewritten only
        // after the store issued two blocks earlier has read it.
        const int quarter = warp & 3;  // TMEM lanes this warp may access: 32 * quarter ...
        const uint32_t epi = smem_u32(smem + STAGES * STAGE_BYTES) + (uint32_t)quarter * 4096u;
        int issued = 0;
        int it = 0;
        for (int tile = blockIdx.x; tile < g.num_tiles; tile += gridDim.x, ++it) {
            int m_blk, n_blk;
            tile_coords(tile, g, m_blk, n_blk);
            const int acc = it & 1;
            const uint32_t acc_phase = (it >> 1) & 1;
            if (!mbar_wait(smem_u32(&acc_full[acc]), acc_phase, &g_device_error)) break;
            tc_fence_after();
            const int row0 = m_blk * BM + quarter * 32;
            const int row = row0 + lane;
            const bool row_ok = row < g.M;
            float r;
            if (g.unit_scale) {
                r = 1.f;
            } else if (g.compute_inv) {
                if (!mbar_wait(smem_u32(&stats_full[acc]), acc_phase, &g_device_error)) break;
                r = inv_buf[acc * BM + quarter * 32 + lane];
            } else {
                r = row_ok ? __ldg(g.inv_rms + row) : 0.f;
            }
            const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * ACC_COLS;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32];
                tmem_ld_32cols(tbase + c * 32, v);
                const int col0 = n_blk * BN + c * 32;
                const uint32_t buf = epi + (uint32_t)(issued & 1) * 2048u;
                if (lane == 0 && issued >= 2) bulk_wait_read1();  // the store that used this buffer has read it
                __syncwarp();
                const uint32_t rowaddr = buf + (uint32_t)lane * 64u;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint4 o;
                    o.x = pack_bf16x2(__uint_as_float(v[8 * j + 0]) * r, __uint_as_float(v[8 * j + 1]) * r);
                    o.y = pack_bf16x2(__uint_as_float(v[8 * j + 2]) * r, __uint_as_float(v[8 * j + 3]) * r);
                    o.z = pack_bf16x2(__uint_as_float(v[8 * j + 4]) * r, __uint_as_float(v[8 * j + 5]) * r);
                    o.w = pack_bf16x2(__uint_as_float(v[8 * j + 6]) * r, __uint_as_float(v[8 * j + 7]) * r);
                    const uint32_t dst = rowaddr + (uint32_t)((j ^ ((lane >> 1) & 3)) * 16);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                                 ::"r"(dst), "r"(o.x), "r"(o.y), "r"(o.z), "r"(o.w) : "memory");
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if (col0 < g.N && row0 < g.M) tma_store_2d(&tmap_y, buf, col0, row0);
                    bulk_commit();
                }
                ++issued;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&acc_empty[acc]));
        }
        if (lane == 0) bulk_wait_all();
    } else if (g.compute_inv) {
        // ---------------------------------------------------------------- row statistics (warps 6, 7)
        // FlashNorm's RMS runs beside the matmul: each x tile the TMA brings in
        // for the MMA is also read here, and every row's sum of squares over K
        // accumulates while the tensor cores work.  The 128-byte swizzle only
        // permutes the 16-byte chunks inside a row, so a row's chunks are read
        // in logical order j at physical position j ^ (row & 7).  Lane l of
        // statistics warp sw owns rows sw*64 + l and sw*64 + l + 32.
        const int sw = warp - 6;
        int stage = 0;
        uint32_t phase = 0;
        int it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < g.num_tiles; tile += gridDim.x, ++it) {
            int m_blk, n_blk;
            tile_coords(tile, g, m_blk, n_blk);
            const int acc = it & 1;
            const uint32_t acc_phase = (it >> 1) & 1;
            float2 ssq[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            for (int kb = 0; kb < g.k_blocks; ++kb) {
                if (!mbar_wait(smem_u32(&full[stage]), phase, &g_device_error)) { ok = false; break; }
                const uint8_t *a_tile = smem + stage * STAGE_BYTES;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int r = sw * 64 + lane + 32 * i;
                    const uint8_t *arow = a_tile + r * (BK * 2);
                    uint4 v[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) v[j] = *reinterpret_cast<const uint4 *>(arow + ((j ^ (r & 7)) * 16));
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float2 p0 = make_float2(bf16lo(v[j].x), bf16hi(v[j].x));
                        const float2 p1 = make_float2(bf16lo(v[j].y), bf16hi(v[j].y));
                        const float2 p2 = make_float2(bf16lo(v[j].z), bf16hi(v[j].z));
                        const float2 p3 = make_float2(bf16lo(v[j].w), bf16hi(v[j].w));
                        ssq[i] = __ffma2_rn(p0, p0, ssq[i]);
                        ssq[i] = __ffma2_rn(p1, p1, ssq[i]);
                        ssq[i] = __ffma2_rn(p2, p2, ssq[i]);
                        ssq[i] = __ffma2_rn(p3, p3, ssq[i]);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&empty[stage]));
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
            // inv_buf[acc] is free once the epilogue has finished tile it - 2
            if (!mbar_wait(smem_u32(&acc_empty[acc]), acc_phase ^ 1u, &g_device_error)) break;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int r = sw * 64 + lane + 32 * i;
                const float inv = rsqrtf((ssq[i].x + ssq[i].y) / (float)g.K + g.eps);
                inv_buf[acc * BM + r] = inv;
                const int row = m_blk * BM + r;
                if (g.inv_out != nullptr && n_blk == 0 && row < g.M) g.inv_out[row] = inv;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&stats_full[acc]));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                     : "memory");
    }
}

}  // namespace gemm


// ----------------------------------------------------------- host helpers

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {  // looked up once, thread-safe
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(p);
        return nullptr;
    }();
    return fn;
}

}  // namespace

// 2-D bf16 tensor [rows][inner] (inner contiguous), box inner 64 x box_rows,
// 128-byte swizzle; out-of-range elements of a box read as zero.
qkn_status make_tmap(CUtensorMap *m, const void *ptr, int64_t rows, int64_t inner, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr) return fail(QKN_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(inner * 2)};
    cuuint32_t box[2] = {(cuuint32_t)gemm::BK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(QKN_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    return QKN_OK;
}

qkn_status make_tmap_store(CUtensorMap *m, void *ptr, int64_t rows, int64_t cols) {
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr) return fail(QKN_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols * 2)};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(QKN_ERR_CUDA, "cuTensorMapEncodeTiled (y) failed (CUresult %d)", (int)r);
    return QKN_OK;
}

qkn_status launch_inv_rms(const void *x, float *inv, int64_t M, int64_t K, float eps, cudaStream_t s) {
    const int64_t blocks = (M + 7) / 8;
    if (blocks > 0x7fffffffLL) return fail(QKN_ERR_SHAPE, "flashnorm_proj: M too large");
    inv_rms_kernel<<<(unsigned)blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(x), inv, M, K, eps);
    return check_launch("inv_rms_kernel launch");
}

#include "gemm_pair.cuh"

// Which projection kernel serves the calls with a given 1/rms (or none):
// the CTA-pair kernel by default (same-box interleaved runs: 616 vs 631 us
// for the single-CTA kernel on the 8192 x 4096 x 12288 projection, outputs
// bit-identical); QKN_GEMM_KERNEL=single selects the single-CTA kernel.
// Read on every call (a getenv), so a process can compare both.  The
// in-kernel statistics form always runs on the single-CTA kernel.
bool use_pair_kernel() {
    const char *v = getenv("QKN_GEMM_KERNEL");
    return !(v != nullptr && strcmp(v, "single") == 0);
}

namespace {

// inv == nullptr (and not unit_scale): the single-CTA kernel computes every
// row's 1/rms itself (eps) and, when inv_out is given, stores it there.
// after_stats: the launch just before on `s` is this library's statistics
// pass writing `inv` (and nothing the projection reads before its epilogue),
// so the projection is launched as its programmatic dependent and overlaps it.
qkn_status launch_gemm(const void *x, const void *Wf, void *y, const float *inv, int64_t M, int64_t N, int64_t K,
                       float eps, float *inv_out, cudaStream_t s, bool unit_scale = false, bool after_stats = false) {
    CUtensorMap tx, tw;
    if (qkn_status st = make_tmap(&tx, x, M, K, gemm::BM)) return st;
    if (qkn_status st = make_tmap(&tw, Wf, N, K, gemm::BN)) return st;
    CUtensorMap ty;
    if (qkn_status st = make_tmap_store(&ty, y, M, N)) return st;
    gemm::Args g;
    g.inv_rms = inv;
    g.inv_out = inv_out;
    g.unit_scale = unit_scale ? 1 : 0;
    g.compute_inv = (inv == nullptr && !unit_scale) ? 1 : 0;
    g.eps = eps;
    g.y = static_cast<__nv_bfloat16 *>(y);
    g.M = (int)M;
    g.N = (int)N;
    g.K = (int)K;
    g.m_blocks = (int)((M + gemm::BM - 1) / gemm::BM);
    g.n_blocks = (int)((N + gemm::BN - 1) / gemm::BN);
    g.k_blocks = (int)((K + gemm::BK - 1) / gemm::BK);
    g.num_tiles = g.m_blocks * g.n_blocks;
    if (!g.compute_inv && use_pair_kernel() && sm_count() >= 2)
        return launch_gemm_pair(x, Wf, y, inv, M, N, K, unit_scale, s, after_stats);
    static std::atomic<bool> attr_set[64];  // per device: the attribute has been set
    int dev = 0;
    cudaGetDevice(&dev);
    const bool known = dev >= 0 && dev < 64;
    if (!known || !attr_set[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(gemm::flashnorm_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             gemm::SMEM_BYTES);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(flashnorm_gemm_kernel)");
        if (known) attr_set[dev].store(true, std::memory_order_release);
    }
    const int grid = g.num_tiles < sm_count() ? g.num_tiles : sm_count();
    if (after_stats) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)grid, 1, 1);
        cfg.blockDim = dim3(gemm::THREADS, 1, 1);
        cfg.dynamicSmemBytes = gemm::SMEM_BYTES;
        cfg.stream = s;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr.val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        const cudaError_t e = cudaLaunchKernelEx(&cfg, gemm::flashnorm_gemm_kernel, tx, tw, ty, g);
        if (e != cudaSuccess) return cuda_fail(e, "flashnorm_gemm_kernel launch");
    } else {
        gemm::flashnorm_gemm_kernel<<<grid, gemm::THREADS, gemm::SMEM_BYTES, s>>>(tx, tw, ty, g);
    }
    return check_launch("flashnorm_gemm_kernel launch");
}

}  // namespace
}  // namespace qkn

using namespace qkn;

extern "C" QKN_API qkn_status flashnorm_fold_weights(const void *w, const void *W, void *W_folded, int64_t K,
                                                     int64_t N, qkn_dtype wdt, int out_k_major, void *stream) {
    if (!valid_dtype(wdt)) return fail(QKN_ERR_DTYPE, "flashnorm_fold_weights: unknown dtype %d", (int)wdt);
    if (w == nullptr || W == nullptr || W_folded == nullptr)
        return fail(QKN_ERR_NULL, "flashnorm_fold_weights: w, W and W_folded are required");
    if (K < 0 || N < 0) return fail(QKN_ERR_SHAPE, "flashnorm_fold_weights: negative size");
    if (!aligned(w, dtype_size(wdt)) || !aligned(W, 2) || !aligned(W_folded, 2))
        return fail(QKN_ERR_ALIGN, "flashnorm_fold_weights: pointers must be aligned to their element size");
    if (K == 0 || N == 0) return QKN_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const __nv_bfloat16 *Wb = static_cast<const __nv_bfloat16 *>(W);
    __nv_bfloat16 *Wo = static_cast<__nv_bfloat16 *>(W_folded);
    const __nv_bfloat16 *wb = static_cast<const __nv_bfloat16 *>(w);
    const float *wf = static_cast<const float *>(w);
    // 16-byte chunks of 8 bf16 when the layout allows (element-wise otherwise)
    const bool vec = aligned(W, 16) && aligned(W_folded, 16) && N % 8 == 0 && (!out_k_major || K % 8 == 0);
    if (out_k_major) {
        const int64_t gx = (N + kFoldTile - 1) / kFoldTile, gy = (K + kFoldTile - 1) / kFoldTile;
        const int64_t tx = (K + kTransTK - 1) / kTransTK, ty = (N + kTransTN - 1) / kTransTN;
        if (gx > 0x7fffffffLL || gy > 65535 || (vec && (tx > 0x7fffffffLL || ty > 65535)))
            return fail(QKN_ERR_SHAPE, "flashnorm_fold_weights: too large");
        dim3 grid((unsigned)gx, (unsigned)gy), tgrid((unsigned)tx, (unsigned)ty);  // tile kernel: k tiles in x
        if (vec && wdt == QKN_BF16)
            transpose_tile_kernel<__nv_bfloat16, true><<<tgrid, 256, 0, s>>>(wb, Wb, Wo, K, N);
        else if (vec)
            transpose_tile_kernel<float, true><<<tgrid, 256, 0, s>>>(wf, Wb, Wo, K, N);
        else if (wdt == QKN_BF16)
            fold_transpose_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(wb, Wb, Wo, K, N);
        else
            fold_transpose_kernel<float><<<grid, 256, 0, s>>>(wf, Wb, Wo, K, N);
    } else {
        const int blocks = 4 * sm_count();
        if (vec && wdt == QKN_BF16)
            fold_rowmajor_vec_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(wb, Wb, Wo, K, N);
        else if (vec)
            fold_rowmajor_vec_kernel<float><<<blocks, 256, 0, s>>>(wf, Wb, Wo, K, N);
        else if (wdt == QKN_BF16)
            fold_rowmajor_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(wb, Wb, Wo, K, N);
        else
            fold_rowmajor_kernel<float><<<blocks, 256, 0, s>>>(wf, Wb, Wo, K, N);
    }
    return check_launch("flashnorm_fold_weights launch");
}

extern "C" QKN_API qkn_status flashnorm_proj(const void *x, const void *W_folded, void *y, int64_t M, int64_t N,
                                             int64_t K, int w_k_major, float eps, const float *inv_rms,
                                             float *inv_rms_out, void *stream) {
    if (x == nullptr || W_folded == nullptr || y == nullptr)
        return fail(QKN_ERR_NULL, "flashnorm_proj: x, W_folded and y are required");
    if (M < 1 || N < 1 || K < 1 || M > 0x7fffffffLL || N > 0x7fffffffLL || K > 0x7fffffffLL)
        return fail(QKN_ERR_SHAPE, "flashnorm_proj: bad sizes M=%lld N=%lld K=%lld", (long long)M, (long long)N,
                    (long long)K);
    if (K % 8 != 0 || N % 8 != 0)
        return fail(QKN_ERR_SHAPE, "flashnorm_proj: K=%lld and N=%lld must be multiples of 8", (long long)K,
                    (long long)N);
    if (inv_rms == nullptr && (!(eps >= 0.f) || isinf(eps)))
        return fail(QKN_ERR_EPS, "flashnorm_proj: eps must be finite and >= 0");
    if (!aligned(x, 16) || !aligned(W_folded, 16) || !aligned(y, 16) || (inv_rms && !aligned(inv_rms, 4)) ||
        (inv_rms_out && !aligned(inv_rms_out, 4)))
        return fail(QKN_ERR_ALIGN, "flashnorm_proj: x, W_folded and y must be 16-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // W' given row-major ([K][N]): a stream-ordered K-major copy first, before
    // the statistics pass, so the projection's early reads (it overlaps that
    // pass) only see finished data
    const void *Wk = W_folded;
    void *tmp = nullptr;
    if (!w_k_major) {
        const int64_t gx = (N + kFoldTile - 1) / kFoldTile, gy = (K + kFoldTile - 1) / kFoldTile;
        if (gy > 0x7fffffffLL || gx > 65535) return fail(QKN_ERR_SHAPE, "flashnorm_proj: W_folded too large to transpose");
        cudaError_t e = cudaMallocAsync(&tmp, (size_t)(N * K * 2), s);
        if (e != cudaSuccess) return cuda_fail(e, "flashnorm_proj: K-major copy of W_folded");
        // K, N multiples of 8 and 16-byte aligned buffers (checked above)
        transpose_tile_kernel<__nv_bfloat16, false><<<dim3((unsigned)gy, (unsigned)gx), 256, 0, s>>>(
            nullptr, static_cast<const __nv_bfloat16 *>(W_folded), static_cast<__nv_bfloat16 *>(tmp), K, N);
        if (qkn_status st = check_launch("transpose_tile_kernel launch")) {
            cudaFreeAsync(tmp, s);
            return st;
        }
        Wk = tmp;
    }
    qkn_status st;
    if (inv_rms == nullptr && inv_rms_out != nullptr) {
        // the caller's buffer is the workspace of a separate row-statistics
        // pass, which leaves the matmul's shared-memory bandwidth to the MMA
        st = launch_inv_rms(x, inv_rms_out, M, K, eps, s);
        // FlashNorm (abstract, item (ii)): with the scaling deferred, the row
        // statistic and the matmul can run at the same time, so the projection
        // starts while the statistics pass runs and waits for it only in its
        // epilogue
        if (st == QKN_OK) st = launch_gemm(x, Wk, y, inv_rms_out, M, N, K, eps, nullptr, s, false, true);
    } else {
        // with no 1/rms at all the GEMM computes it beside the matmul (no workspace)
        st = launch_gemm(x, Wk, y, inv_rms, M, N, K, eps, nullptr, s);
    }
    if (tmp != nullptr) {
        const cudaError_t e = cudaFreeAsync(tmp, s);
        if (e != cudaSuccess && st == QKN_OK) st = cuda_fail(e, "flashnorm_proj: releasing the K-major copy");
    }
    return st;
}

extern "C" QKN_API qkn_status qkn_check_device(void *stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "qkn_check_device: stream synchronisation");
    int flag = 0;
    e = cudaMemcpyFromSymbol(&flag, g_device_error, sizeof flag);
    if (e != cudaSuccess) return cuda_fail(e, "qkn_check_device: reading the device error word");
    if (flag != 0) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero);
    }
    int norm_flag = 0, qkv_flag = 0;
    if (qkn_status st = read_norm_error(&norm_flag)) return st;
    if (qkn_status st = read_qkv_error(&qkv_flag)) return st;
    if (flag != 0 || norm_flag != 0 || qkv_flag != 0)
        return fail(QKN_ERR_TIMEOUT, "a bounded device-side wait gave up (projection %d, norm %d, fused QKV %d)", flag,
                    norm_flag, qkv_flag);
    return QKN_OK;
}

// ===================================================== no-allocation variant
//
// Some callers cannot allocate device memory at call time: serving runtimes
// that plan every byte of the GPU up front and forbid allocations on the hot
// path (so the footprint stays fixed and no allocator lock is taken), callers
// running under a framework whose own allocator owns the whole device, and
// real-time loops that cannot afford an allocator's latency spikes.  For them
// flashnorm_proj_noalloc keeps the 1/rms vector in the fixed array below
// instead of taking scratch from the CUDA memory pool.
//
// The array is a file-scope device variable: every GPU that loads this
// library holds it (1 MiB) until the process exits, and every call on that
// GPU shares it, so calls that overlap on the GPU race on it.  Each call
// overwrites the entries it uses before reading them, so nothing has to start
// at zero.  In host code the name g_noalloc_inv_rms is only a host-side
// stand-in; its device address is fetched with cudaGetSymbolAddress on the
// first call made with a device current and cached together with the CUDA
// context it belongs to.  A later call that finds another context current on
// that device (the primary context was reset and the module loaded again,
// possibly at another address) fetches the address again.

namespace qkn {
namespace {

constexpr int64_t kNoAllocMaxRows = 262144;  // 1 MiB of fp32

static __device__ __align__(256) float g_noalloc_inv_rms[kNoAllocMaxRows];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
struct NoAllocSlot {
    CUcontext ctx;  // context the cached address belongs to
    float *ptr;
};
NoAllocSlot g_noalloc_slot[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

// The driver's cuCtxGetCurrent, looked up once through the runtime (the
// library does not link libcuda directly).
CtxGetCurrentFn ctx_get_current_fn() {
    static const CtxGetCurrentFn fn = []() -> CtxGetCurrentFn {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<CtxGetCurrentFn>(p);
        return nullptr;
    }();
    return fn;
}

// Device address of g_noalloc_inv_rms in the current device's current context.
qkn_status noalloc_scratch(float **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "flashnorm_proj_noalloc: cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(QKN_ERR_UNSUPPORTED, "flashnorm_proj_noalloc: device %d", dev);
    CtxGetCurrentFn get_ctx = ctx_get_current_fn();
    if (get_ctx == nullptr) return fail(QKN_ERR_CUDA, "flashnorm_proj_noalloc: cuCtxGetCurrent is unavailable");
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) return fail(QKN_ERR_CUDA, "flashnorm_proj_noalloc: cuCtxGetCurrent failed");
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoAllocSlot &slot = g_noalloc_slot[dev];
    if (slot.ptr == nullptr || ctx == nullptr || slot.ctx != ctx) {
        // also makes the runtime bind the device's primary context when none was current yet
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_inv_rms);
        if (e != cudaSuccess || p == nullptr)
            return cuda_fail(e, "flashnorm_proj_noalloc: cudaGetSymbolAddress(scratch)");
        if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr)
            return fail(QKN_ERR_CUDA, "flashnorm_proj_noalloc: no current context after the symbol lookup");
        slot.ctx = ctx;
        slot.ptr = static_cast<float *>(p);
    }
    *out = slot.ptr;
    return QKN_OK;
}

}  // namespace
}  // namespace qkn

extern "C" QKN_API qkn_status flashnorm_proj_noalloc(const void *x, const void *W_folded, void *y, int64_t M,
                                                     int64_t N, int64_t K, int w_k_major, float eps,
                                                     void *stream) {
    if (x == nullptr || W_folded == nullptr || y == nullptr)
        return fail(QKN_ERR_NULL, "flashnorm_proj_noalloc: x, W_folded and y are required");
    if (M < 1 || N < 1 || K < 1 || N > 0x7fffffffLL || K > 0x7fffffffLL)
        return fail(QKN_ERR_SHAPE, "flashnorm_proj_noalloc: bad sizes M=%lld N=%lld K=%lld", (long long)M,
                    (long long)N, (long long)K);
    if (M > kNoAllocMaxRows)
        return fail(QKN_ERR_SHAPE,
                    "flashnorm_proj_noalloc: M=%lld rows exceed the fixed scratch of %lld rows; split the "
                    "call or use flashnorm_proj", (long long)M, (long long)kNoAllocMaxRows);
    if (K % 8 != 0 || N % 8 != 0)
        return fail(QKN_ERR_SHAPE, "flashnorm_proj_noalloc: K=%lld and N=%lld must be multiples of 8",
                    (long long)K, (long long)N);
    if (!w_k_major) return fail(QKN_ERR_UNSUPPORTED, "flashnorm_proj_noalloc: W_folded must be K-major ([N][K])");
    if (!(eps >= 0.f) || isinf(eps)) return fail(QKN_ERR_EPS, "flashnorm_proj_noalloc: eps must be finite and >= 0");
    if (!aligned(x, 16) || !aligned(W_folded, 16) || !aligned(y, 16))
        return fail(QKN_ERR_ALIGN, "flashnorm_proj_noalloc: x, W_folded and y must be 16-byte aligned");
    float *inv = nullptr;
    if (qkn_status st = noalloc_scratch(&inv)) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (qkn_status st = launch_inv_rms(x, inv, M, K, eps, s)) return st;
    return launch_gemm(x, W_folded, y, inv, M, N, K, eps, nullptr, s, false, /*after_stats=*/true);
}

// ===================================================== RMSNorm elimination
//
// FlashNorm, abstract: by the scale invariance of RMS, RMSNorm -> linear ->
// RMSNorm lets the first RMSNorm be dropped.  With q, k and v each
// RMS-normalised after the projection (QKV-normalisation), the pre-attention
// RMSNorm reduces to its weights, already folded into W', and its 1/rms(x)
// disappears: per row, RMSNorm(c * u) = RMSNorm(u) for the scale c = 1/rms(x)
// (exactly when that norm's eps is 0; otherwise up to the relative size of
// eps next to the rows' mean square).  So: y = x W'^T with no row scaling,
// then the q / k / v row groups normalised in place.
extern "C" QKN_API qkn_status qkv_norm_proj(const void *x, const void *W_folded, void *y, int64_t M, int64_t K,
                                            int64_t nq, int64_t nk, int64_t nv, const void *wq, const void *wk,
                                            const void *wv, qkn_dtype wdt, float eps, int n_seg, void *stream) {
    if (!valid_dtype(wdt)) return fail(QKN_ERR_DTYPE, "qkv_norm_proj: unknown dtype %d", (int)wdt);
    if (x == nullptr || W_folded == nullptr || y == nullptr || wq == nullptr || wk == nullptr ||
        (nv > 0 && wv == nullptr))
        return fail(QKN_ERR_NULL, "qkv_norm_proj: x, W_folded, y, wq, wk (and wv when nv > 0) are required");
    const int64_t N = nq + nk + nv;
    if (M < 1 || K < 1 || nq < 1 || nk < 1 || nv < 0 || M > 0x7fffffffLL || N > 0x7fffffffLL || K > 0x7fffffffLL)
        return fail(QKN_ERR_SHAPE, "qkv_norm_proj: bad sizes M=%lld K=%lld nq=%lld nk=%lld nv=%lld", (long long)M,
                    (long long)K, (long long)nq, (long long)nk, (long long)nv);
    if (K % 8 != 0 || N % 8 != 0)
        return fail(QKN_ERR_SHAPE, "qkv_norm_proj: K and nq + nk + nv must be multiples of 8");
    if (n_seg < 1 || n_seg > QKN_MAX_SEG || nq % n_seg || nk % n_seg || nv % n_seg)
        return fail(QKN_ERR_SHAPE, "qkv_norm_proj: nq, nk, nv must be multiples of n_seg=%d", n_seg);
    if (!(eps >= 0.f) || isinf(eps)) return fail(QKN_ERR_EPS, "qkv_norm_proj: eps must be finite and >= 0");
    if (!aligned(x, 16) || !aligned(W_folded, 16) || !aligned(y, 16))
        return fail(QKN_ERR_ALIGN, "qkv_norm_proj: x, W_folded and y must be 16-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (qkn_status st = launch_gemm(x, W_folded, y, nullptr, M, N, K, 0.f, nullptr, s, /*unit_scale=*/true))
        return st;
    __nv_bfloat16 *yb = static_cast<__nv_bfloat16 *>(y);
    if (qkn_status st = qknorm_fused(yb, yb + nq, wq, wk, nullptr, nullptr, M, nq, nk, N, N, N, N, QKN_BF16, wdt,
                                     eps, n_seg, stream))
        return st;
    if (nv > 0)
        return qknorm_fused(yb + nq + nk, nullptr, wv, nullptr, nullptr, nullptr, M, nv, 0, N, 0, N, 0, QKN_BF16,
                            wdt, eps, n_seg, stream);
    return QKN_OK;
}
