// QKV projection with QK-Norm in the GEMM epilogue.
//
// Pre-attention path of a block that normalises queries and keys:
//   u = RMSNorm(x; w_in) W          -- FlashNorm (abstract): w_in folded into W',
//                                     1/rms(x) applied to the matmul output
//   y_q = RMSNorm(u_q; wq), y_k = RMSNorm(u_k; wk), y_v = u_v
//                                  -- layerwise QK-Norm over each token's full
//                                     query and key vectors (SwiftQK, abstract)
// The QK-Norm factor of a row needs the sum of squares over all nq (nk)
// columns, which the GEMM computes in 256-column tiles on different CTAs.
// SwiftQK's observation carries over from GPUs to CTAs: only one scalar per
// row and tile has to be exchanged.  Every epilogue warp publishes its rows'
// partial sums of squares for its tile, counts itself in with a release
// add, waits (bounded) until all tiles of the row block's q (k) section have
// arrived, adds the partials in tile order -- a fixed order, so the result is
// deterministic -- and only then scales its accumulator and stores bf16.  The
// q and k values never go to HBM unnormalised.
//
// Progress: the kernel is persistent with at most one CTA per SM, launched
// cooperatively, so all CTAs are resident together.  CTA c handles tiles
// c, c + G, c + 2G, ... (G = grid size) in order and always publishes before
// it waits.  The tiles of one row block's section are consecutive tile
// indices, at most G of them, so they sit on distinct CTAs; the unfinished
// tile with the lowest index therefore waits only for tiles that their CTAs
// reach without waiting on anything later, and every wait ends.  Each wait is
// also bounded in time and records a failure in g_qkv_error.
#include <atomic>
#include <cuda.h>
#include <math.h>

#include "gemm_tc.cuh"
#include "qkn_common.cuh"
#include "qkn_sync.cuh"

namespace qkn {

// Set when a bounded wait of the fused kernel gave up; read by qkn_check_device.
__device__ int g_qkv_error = 0;

namespace qkvn {

using gemm::A_BYTES;
using gemm::ACC_COLS;
using gemm::BK;
using gemm::BM;
using gemm::BN;
using gemm::STAGE_BYTES;
using gemm::STAGES;
using gemm::TMEM_COLS;
using gemm::UMMA_K;

constexpr int THREADS = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int BAR_BYTES = 256;
constexpr int EPI_BYTES = 4 * 2 * 2048;  // two 32x32 bf16 staging tiles per epilogue warp
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 1024;  // + 1 KiB for alignment
constexpr int GROUP_M = 64;  // row blocks walked together: W' is read from DRAM about once per 64 row blocks

static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

struct Args {
    const float *inv_rms;  // [M] 1/rms of the rows of x, or null: no input scaling
    const void *wq;        // [nq] QK-Norm weights of q (fp32 or bf16)
    const void *wk;        // [nk]
    __nv_bfloat16 *y;      // [M][N], N = nq + nk + nv
    float *partial;        // [2][m_blocks * BM][pstride] per-tile row sums of squares
    unsigned *count;       // [m_blocks][2][4] arrivals per (row block, section, lane quarter)
    int M, K, N, nq, nk;
    int m_blocks, k_blocks;
    int tq, tk, tv;        // tiles per row block in the q, k and v sections
    int tiles_per_row, num_tiles, pstride;
    int w_f32;             // 1: fp32 QK-Norm weights, 0: bf16
    float eps;             // QK-Norm eps
    uint64_t wait_ns;      // limit of every wait
    int skip_arrival;      // testing only: CTA 0's first epilogue warp does not count in on its first tile
};

struct Tile {
    int m_blk, sec, n;  // row block; section 0 q, 1 k, 2 v; tile within the section
    int col0, col_end;  // first column of the tile; end of its section
};

// Tiles are dealt in groups of GROUP_M row blocks.  Inside a group come the
// q tiles (row block by row block, each row block's q tiles consecutive),
// then the k tiles, then the v tiles, in the same arrangement.
__device__ __forceinline__ Tile tile_of(int tile, const Args &g) {
    const int group_tiles = GROUP_M * g.tiles_per_row;
    const int group = tile / group_tiles;
    const int first_m = group * GROUP_M;
    const int rows = min(g.m_blocks - first_m, GROUP_M);
    int r = tile - group * group_tiles;
    Tile t;
    if (r < rows * g.tq) {
        t.sec = 0;
        t.m_blk = first_m + r / g.tq;
        t.n = r % g.tq;
        t.col0 = t.n * BN;
        t.col_end = g.nq;
        return t;
    }
    r -= rows * g.tq;
    if (r < rows * g.tk) {
        t.sec = 1;
        t.m_blk = first_m + r / g.tk;
        t.n = r % g.tk;
        t.col0 = g.nq + t.n * BN;
        t.col_end = g.nq + g.nk;
        return t;
    }
    r -= rows * g.tk;
    t.sec = 2;
    t.m_blk = first_m + r / g.tv;
    t.n = r % g.tv;
    t.col0 = g.nq + g.nk + t.n * BN;
    t.col_end = g.N;
    return t;
}

__device__ __forceinline__ void red_release_add(unsigned *p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Whole warp: waits until *cnt >= target.  Every lane's own acquire load sees
// the final count, so the partial sums published before the release adds are
// visible to all lanes afterwards.  Returns false after wait_ns, or as soon as
// another wait of this launch has given up (so one failure costs one limit,
// not one per tile).
__device__ __noinline__ bool wait_count(const unsigned *cnt, unsigned target, uint64_t wait_ns) {
    if (__all_sync(0xffffffffu, ld_acquire(cnt) >= target)) return true;
    const uint64_t t0 = global_timer();
    while (true) {
        for (int i = 0; i < 16; ++i) {
            __nanosleep(64);
            if (__all_sync(0xffffffffu, ld_acquire(cnt) >= target)) return true;
        }
        const int give_up =
            (global_timer() - t0 > wait_ns || *static_cast<volatile int *>(&g_qkv_error) != 0) ? 1 : 0;
        if (__shfl_sync(0xffffffffu, give_up, 0)) return false;
    }
}

// 8 consecutive QK-Norm weights as fp32 (all lanes read the same address).
__device__ __forceinline__ void load_w8(const void *w, int w_f32, int c, float (&f)[8]) {
    if (w_f32) {
        const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(w) + c);
        const float4 a = __ldg(p), b = __ldg(p + 1);
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    } else {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(w) + c));
        f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
        f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
    }
}

// The epilogue of one accumulator tile for the 32 rows of this warp (TMEM
// lane quarter `quarter` of the tile's 128-row block `mb`): QK-Norm's tile
// partials published and exchanged for q and k tiles, then the scaled tile
// stored in bf16.  `skip` (testing only) leaves this warp's arrival out.
__device__ __forceinline__ void epilogue_tile(const Args &g, const CUtensorMap *tmap_y, int mb, const Tile &t,
                                              uint32_t acc_tmem, uint32_t epi, int &issued, int quarter, int lane,
                                              bool skip) {
    const int lrow = quarter * 32 + lane;
    const int row = mb * BM + lrow;
    const bool row_ok = row < g.M;
    const float r = g.inv_rms == nullptr ? 1.f : (row_ok ? __ldg(g.inv_rms + row) : 0.f);
    const uint32_t tbase = acc_tmem + ((uint32_t)(quarter * 32) << 16);
    const int ncols = min(BN, t.col_end - t.col0);  // columns of this tile inside its section
    const int nchunks = (ncols + 31) / 32;
    float inv_qk = 1.f;
    const void *w = nullptr;
    int w0 = 0;
    if (t.sec < 2) {
        // pass 1: this tile's share of the row's sum of squares of u = r * acc
        float2 ss = make_float2(0.f, 0.f);
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
            uint32_t v[32];
            gemm::tmem_ld_32cols(tbase + c * 32, v);
            const int valid = ncols - c * 32;  // a multiple of 8
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                if (j < valid) {
                    const float2 u = make_float2(__uint_as_float(v[j]) * r, __uint_as_float(v[j + 1]) * r);
                    ss = __ffma2_rn(u, u, ss);
                }
            }
        }
        float *prow = g.partial + ((size_t)t.sec * g.m_blocks * BM + (size_t)row) * g.pstride;
        prow[t.n] = ss.x + ss.y;
        __threadfence();
        __syncwarp();
        unsigned *cnt = g.count + (mb * 2 + t.sec) * 4 + quarter;
        if (lane == 0 && !skip) red_release_add(cnt, 1u);
        const int ntiles = t.sec == 0 ? g.tq : g.tk;
        if (!wait_count(cnt, (unsigned)ntiles, g.wait_ns) && lane == 0) atomicExch(&g_qkv_error, 1);
        // fixed-order combine of the row's per-tile partial sums: sixteen at
        // a time loaded first (four 16-byte loads: a row's partials are
        // contiguous and pstride is a multiple of 4), then added in order
        float S = 0.f;
        const float4 *p4 = reinterpret_cast<const float4 *>(prow);
        for (int i0 = 0; i0 < ntiles; i0 += 16) {
            float4 q4[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (i0 + 4 * u < ntiles) q4[u] = __ldcg(p4 + i0 / 4 + u);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float e[4] = {q4[u].x, q4[u].y, q4[u].z, q4[u].w};
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (i0 + 4 * u + c < ntiles) S += e[c];
            }
        }
        const int d = t.sec == 0 ? g.nq : g.nk;
        inv_qk = rsqrtf(S / (float)d + g.eps);
        w = t.sec == 0 ? g.wq : g.wk;
        w0 = t.col0 - (t.sec == 0 ? 0 : g.nq);
    }
    // pass 2: y = ((r * acc) * inv_qk) * w for q and k, r * acc for v; bf16 out
    const int row0 = mb * BM + quarter * 32;
    __nv_bfloat16 *yrow = g.y + (int64_t)(row_ok ? row : 0) * g.N;
#pragma unroll 1
    for (int c = 0; c < nchunks; ++c) {
        uint32_t v[32];
        gemm::tmem_ld_32cols(tbase + c * 32, v);
        const int base = c * 32;
        const bool whole = base + 32 <= ncols;  // the same for the whole warp
        const uint32_t buf = epi + (uint32_t)(issued & 1) * 2048u;
        if (whole) {
            if (lane == 0 && issued >= 2) bulk_wait_read1();  // the store two blocks back has read it
            __syncwarp();
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int off = base + j * 8;
            if (whole || (row_ok && off < ncols)) {
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * j + e]) * r;
                if (t.sec < 2) {
                    float wv[8];
                    load_w8(w, g.w_f32, w0 + off, wv);
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = (f[e] * inv_qk) * wv[e];
                }
                uint4 o;
                o.x = pack_bf16x2(f[0], f[1]);
                o.y = pack_bf16x2(f[2], f[3]);
                o.z = pack_bf16x2(f[4], f[5]);
                o.w = pack_bf16x2(f[6], f[7]);
                if (whole) {
                    const uint32_t dst = buf + (uint32_t)lane * 64u + (uint32_t)((j ^ ((lane >> 1) & 3)) * 16);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                                 ::"r"(dst), "r"(o.x), "r"(o.y), "r"(o.z), "r"(o.w) : "memory");
                } else {
                    *reinterpret_cast<uint4 *>(yrow + t.col0 + off) = o;
                }
            }
        }
        if (whole) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                if (row0 < g.M) tma_store_2d(tmap_y, buf, t.col0 + base, row0);
                bulk_commit();
            }
            ++issued;
        }
    }
}

__global__ void __launch_bounds__(THREADS, 1)
qkv_qknorm_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                       const __grid_constant__ CUtensorMap tmap_y, const Args g) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES + EPI_BYTES);
    uint64_t *full = bars, *empty = bars + STAGES;
    uint64_t *acc_full = bars + 2 * STAGES, *acc_empty = bars + 2 * STAGES + 2;
    uint64_t *drained = bars + 2 * STAGES + 4;  // every MMA this CTA issued has completed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 5);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&full[s]), 1);   // producer's arrive + TMA bytes
            mbar_init(smem_u32(&empty[s]), 1);  // one tcgen05.commit
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&acc_full[a]), 1);   // one tcgen05.commit
            mbar_init(smem_u32(&acc_empty[a]), 4);  // one arrive per epilogue warp
        }
        mbar_init(smem_u32(drained), 1);            // the MMA warp's final tcgen05.commit
        mbar_init_fence();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    gemm::tc_fence_before();
    __syncthreads();
    gemm::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {  // one lane runs the ring
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed = 0, armed_parity = 0;  // per stage: loads issued; parity of the phase they complete
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < g.num_tiles; tile += gridDim.x) {
                const Tile t = tile_of(tile, g);
                for (int kb = 0; kb < g.k_blocks; ++kb) {
                    if (!mbar_wait_fast(smem_u32(&empty[stage]), phase ^ 1u, &g_qkv_error, g.wait_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full[stage]);
                    uint8_t *sa = smem + stage * STAGE_BYTES;
                    mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    tma_load_2d(smem_u32(sa), &tmap_x, kb * BK, t.m_blk * BM, fb);
                    tma_load_2d(smem_u32(sa + A_BYTES), &tmap_w, kb * BK, t.col0, fb);
                    armed |= 1u << stage;
                    armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            // No copy may still be writing shared memory when the CTA exits:
            // wait (bounded) for the last phase armed on every stage
            // (immediate on the normal path, where the MMA warp consumed them all).
            for (int s2 = 0; s2 < STAGES; ++s2)
                if (armed & (1u << s2))
                    mbar_wait(smem_u32(&full[s2]), (armed_parity >> s2) & 1u, &g_qkv_error, g.wait_ns);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {  // one lane waits and issues; stages move the descriptors' address field
            const uint64_t a_desc0 = gemm::sw128_kmajor_desc(smem_u32(smem));
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < g.num_tiles; tile += gridDim.x, ++it) {
                const int acc = it & 1;
                const uint32_t acc_phase = (it >> 1) & 1;
                if (!mbar_wait_fast(smem_u32(&acc_empty[acc]), acc_phase ^ 1u, &g_qkv_error, g.wait_ns)) break;
                gemm::tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
                for (int kb = 0; kb < g.k_blocks; ++kb) {
                    if (!mbar_wait_fast(smem_u32(&full[stage]), phase, &g_qkv_error, g.wait_ns)) { ok = false; break; }
                    gemm::tc_fence_after();
                    const uint64_t ad = a_desc0 + (uint64_t)((stage * STAGE_BYTES) >> 4);
                    const uint64_t bd = ad + (uint64_t)(A_BYTES >> 4);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k)
                        gemm::umma_bf16(d_tmem, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), (kb | k) != 0 ? 1u : 0u);
                    gemm::umma_commit(smem_u32(&empty[stage]));
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                gemm::umma_commit(smem_u32(&acc_full[acc]));
            }
            // Tensor memory is released only after every MMA issued here has
            // completed, also when a wait above gave up with MMAs in flight.
            gemm::umma_commit(smem_u32(drained));
            mbar_wait(smem_u32(drained), 0u, &g_qkv_error, g.wait_ns);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue (warps 2..5)
        const int quarter = warp & 3;  // TMEM lanes 32 * quarter ... of the accumulator
        // 32 x 32 output blocks go out through shared memory and one TMA store
        // each (two alternating staging buffers per warp, 64-byte swizzle); a
        // block that a section ends inside is stored lane by lane instead
        const uint32_t epi = smem_u32(smem + STAGES * STAGE_BYTES) + (uint32_t)quarter * 4096u;
        int issued = 0;
        int it = 0;
        for (int tile = blockIdx.x; tile < g.num_tiles; tile += gridDim.x, ++it) {
            const Tile t = tile_of(tile, g);
            const int acc = it & 1;
            const uint32_t acc_phase = (it >> 1) & 1;
            if (!mbar_wait(smem_u32(&acc_full[acc]), acc_phase, &g_qkv_error, g.wait_ns)) break;
            gemm::tc_fence_after();
            epilogue_tile(g, &tmap_y, t.m_blk, t, tmem_base + acc * ACC_COLS, epi, issued, quarter, lane,
                          g.skip_arrival && blockIdx.x == 0 && it == 0 && quarter == 0);
            gemm::tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&acc_empty[acc]));
        }
        if (lane == 0) bulk_wait_all();
    }

    gemm::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        gemm::tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                     : "memory");
    }
}

// Workspace layout: the partial sums, then the arrival counters.
struct Layout {
    int m_blocks, tq, tk, tv, pstride;
    size_t partial_bytes, count_bytes, total;
};

Layout layout(int64_t M, int64_t nq, int64_t nk, int64_t nv) {
    Layout l;
    l.m_blocks = (int)((M + BM - 1) / BM);
    l.tq = (int)((nq + BN - 1) / BN);
    l.tk = (int)((nk + BN - 1) / BN);
    l.tv = (int)((nv + BN - 1) / BN);
    l.pstride = ((l.tq > l.tk ? l.tq : l.tk) + 3) / 4 * 4;
    l.partial_bytes = (size_t)2 * l.m_blocks * BM * l.pstride * sizeof(float);
    l.count_bytes = (size_t)l.m_blocks * 8 * sizeof(unsigned);
    l.total = l.partial_bytes + (l.count_bytes + 255) / 256 * 256;
    return l;
}

}  // namespace qkvn

// Testing hook: the next qkv_proj_qknorm call on this host thread runs with
// a short wait limit and one missing arrival (a count nothing completes).
thread_local uint64_t t_exchange_fault_ns = 0;

qkn_status read_qkv_error(int *flag) {
    cudaError_t e = cudaMemcpyFromSymbol(flag, g_qkv_error, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "reading the fused QKV kernel's device error word");
    if (*flag) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_qkv_error, &zero, sizeof zero);
    }
    return QKN_OK;
}

}  // namespace qkn

using namespace qkn;

extern "C" QKN_API size_t qkv_proj_qknorm_workspace_bytes(int64_t M, int64_t nq, int64_t nk, int64_t nv) {
    if (M < 1 || nq < 1 || nk < 1 || nv < 0) return 0;
    return qkvn::layout(M, nq, nk, nv).total;
}

extern "C" QKN_API qkn_status qkv_proj_qknorm(const void *x, const void *W_folded, void *y, int64_t M, int64_t K,
                                              int64_t nq, int64_t nk, int64_t nv, const void *wq, const void *wk,
                                              qkn_dtype wdt, float eps, float eps_qk, const float *inv_rms,
                                              float *inv_rms_out, void *workspace, size_t workspace_bytes,
                                              void *stream) {
    if (!valid_dtype(wdt)) return fail(QKN_ERR_DTYPE, "qkv_proj_qknorm: unknown dtype %d", (int)wdt);
    if (x == nullptr || W_folded == nullptr || y == nullptr || wq == nullptr || wk == nullptr)
        return fail(QKN_ERR_NULL, "qkv_proj_qknorm: x, W_folded, y, wq and wk are required");
    const int64_t N = nq + nk + nv;
    if (M < 1 || K < 1 || nq < 1 || nk < 1 || nv < 0 || M > 0x7fffffffLL || K > 0x7fffffffLL || N > 0x7fffffffLL)
        return fail(QKN_ERR_SHAPE, "qkv_proj_qknorm: bad sizes M=%lld K=%lld nq=%lld nk=%lld nv=%lld",
                    (long long)M, (long long)K, (long long)nq, (long long)nk, (long long)nv);
    if (K % 8 || nq % 8 || nk % 8 || nv % 8)
        return fail(QKN_ERR_SHAPE, "qkv_proj_qknorm: K, nq, nk and nv must be multiples of 8");
    if (!(eps_qk >= 0.f) || isinf(eps_qk) || (inv_rms == nullptr && inv_rms_out != nullptr && (!(eps >= 0.f) || isinf(eps))))
        return fail(QKN_ERR_EPS, "qkv_proj_qknorm: eps and eps_qk must be finite and >= 0");
    if (!aligned(x, 16) || !aligned(W_folded, 16) || !aligned(y, 16) || !aligned(wq, 16) || !aligned(wk, 16) ||
        (inv_rms && !aligned(inv_rms, 4)) || (inv_rms_out && !aligned(inv_rms_out, 4)) ||
        (workspace && !aligned(workspace, 16)))
        return fail(QKN_ERR_ALIGN, "qkv_proj_qknorm: x, W_folded, y, wq, wk and workspace must be 16-byte aligned");
    const qkvn::Layout l = qkvn::layout(M, nq, nk, nv);
    if (workspace != nullptr && workspace_bytes < l.total)
        return fail(QKN_ERR_SHAPE, "qkv_proj_qknorm: workspace of %zu bytes, %zu needed", workspace_bytes, l.total);
    const int sms = sm_count();
    const int64_t num_tiles = (int64_t)l.m_blocks * (l.tq + l.tk + l.tv);
    if (num_tiles > 0x7fffffffLL) return fail(QKN_ERR_SHAPE, "qkv_proj_qknorm: too many tiles");
    const int grid = num_tiles < sms ? (int)num_tiles : sms;
    // the exchange needs every tile of a row block's q (k) section on a distinct resident CTA
    if (l.tq > grid || l.tk > grid)
        return fail(QKN_ERR_UNSUPPORTED, "qkv_proj_qknorm: nq=%lld or nk=%lld spans more tiles than the %d CTAs",
                    (long long)nq, (long long)nk, grid);
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    static std::atomic<bool> attr_set[64];  // per device: the attribute has been set
    int dev = 0;
    cudaGetDevice(&dev);
    const bool known = dev >= 0 && dev < 64;
    if (!known || !attr_set[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(qkvn::qkv_qknorm_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             qkvn::SMEM_BYTES);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(qkv_qknorm_gemm_kernel)");
        if (known) attr_set[dev].store(true, std::memory_order_release);
    }

    if (inv_rms == nullptr && inv_rms_out != nullptr) {
        if (qkn_status st = launch_inv_rms(x, inv_rms_out, M, K, eps, s)) return st;
        inv_rms = inv_rms_out;
    }
    CUtensorMap tx, tw;
    if (qkn_status st = make_tmap(&tx, x, M, K, gemm::BM)) return st;
    if (qkn_status st = make_tmap(&tw, W_folded, N, K, gemm::BN)) return st;
    CUtensorMap ty;
    if (qkn_status st = make_tmap_store(&ty, y, M, N)) return st;

    void *ws = workspace;
    bool owned = false;
    cudaError_t e;
    if (ws == nullptr) {
        if ((e = cudaMallocAsync(&ws, l.total, s)) != cudaSuccess) return cuda_fail(e, "qkv_proj_qknorm: workspace");
        owned = true;
    }
    float *partial = static_cast<float *>(ws);
    unsigned *count = reinterpret_cast<unsigned *>(static_cast<uint8_t *>(ws) + l.partial_bytes);
    e = cudaMemsetAsync(count, 0, l.count_bytes, s);
    qkn_status st = QKN_OK;
    if (e != cudaSuccess) {
        st = cuda_fail(e, "qkv_proj_qknorm: clearing the arrival counters");
    } else {
        qkvn::Args g;
        g.inv_rms = inv_rms;
        g.wq = wq;
        g.wk = wk;
        g.y = static_cast<__nv_bfloat16 *>(y);
        g.partial = partial;
        g.count = count;
        g.M = (int)M;
        g.K = (int)K;
        g.N = (int)N;
        g.nq = (int)nq;
        g.nk = (int)nk;
        g.m_blocks = l.m_blocks;
        g.k_blocks = (int)((K + gemm::BK - 1) / gemm::BK);
        g.tq = l.tq;
        g.tk = l.tk;
        g.tv = l.tv;
        g.tiles_per_row = l.tq + l.tk + l.tv;
        g.num_tiles = (int)num_tiles;
        g.pstride = l.pstride;
        g.w_f32 = wdt == QKN_F32 ? 1 : 0;
        g.eps = eps_qk;
        g.wait_ns = kWaitTimeoutNs;
        g.skip_arrival = 0;
        if (t_exchange_fault_ns != 0) {  // one-shot test hook
            g.wait_ns = t_exchange_fault_ns;
            g.skip_arrival = 1;
            t_exchange_fault_ns = 0;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)grid, 1, 1);
        cfg.blockDim = dim3(qkvn::THREADS, 1, 1);
        cfg.dynamicSmemBytes = qkvn::SMEM_BYTES;
        cfg.stream = s;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeCooperative;  // all CTAs resident at once, or the launch fails
        attr.val.cooperative = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, qkvn::qkv_qknorm_gemm_kernel, tx, tw, ty, g);
        if (e != cudaSuccess) st = cuda_fail(e, "qkv_qknorm_gemm_kernel launch");
    }
    if (owned) {
        e = cudaFreeAsync(ws, s);
        if (e != cudaSuccess && st == QKN_OK) st = cuda_fail(e, "qkv_proj_qknorm: releasing the workspace");
    }
    return st;
}

extern "C" QKN_API qkn_status qkn_testing_arm_exchange_fault(uint64_t wait_ns) {
    if (wait_ns == 0 || wait_ns > qkn::kWaitTimeoutNs)
        return fail(QKN_ERR_SHAPE, "qkn_testing_arm_exchange_fault: wait_ns must be in (0, %llu]",
                    (unsigned long long)qkn::kWaitTimeoutNs);
    qkn::t_exchange_fault_ns = wait_ns;
    return QKN_OK;
}
