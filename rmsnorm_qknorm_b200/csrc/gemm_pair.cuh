// FlashNorm projection y = (x W'^T) * 1/rms(x) on CTA pairs.
//
// Included by flashnorm.cu (it shares that file's device error word).
//
// The default kernel of the projection (the single-CTA kernel in
// flashnorm.cu serves the in-kernel statistics form).  Two CTAs of a
// cluster (the two SMs of a TPC) compute one 256 x 256 tile with
// tcgen05.mma.cta_group::2: each CTA loads only its own 128 x rows and its
// own 128 W' rows (32 KiB per k-block instead of the single-CTA kernel's
// 48 KiB), the MMA reads both CTAs' tiles, and each CTA's tensor memory
// holds the fp32 accumulator of its own 128 rows over all 256 columns.  The
// smaller stages give a 6-deep ring: what limits these kernels is the round
// trip a stage makes (MMAs complete, commit, refill, next MMAs), and a
// deeper ring hides more of it.
//
// Roles (192 threads per CTA):
//   warp 0     TMA producer, both CTAs: this CTA's x and W' tiles of a stage
//              land in its own shared memory; their bytes complete on the
//              even CTA's stage barrier (.cta_group::2 form of the load).
//   warp 1     even CTA: one lane issues the M = 256, N = 256 MMAs and the
//              commits that free a stage (or publish an accumulator) in both
//              CTAs -- one commit per CTA's barrier.
//              Both CTAs: allocate / free the pair's tensor memory.
//   warps 2-5  epilogue, both CTAs: tensor memory -> registers, times the
//              row's 1/rms, bf16, staged 32 x 32 blocks stored with TMA;
//              then released on the even CTA's accumulator barrier.
// Every wait is bounded and records a failure in g_device_error; before the
// pair frees tensor memory and exits, the even CTA waits for all of its MMAs
// and each producer for all the copies it issued.
#pragma once

// (pair_tc.cuh, the tile shape and helpers, is included at file scope by flashnorm.cu)

namespace pair {

struct Args {
    const float *inv_rms;  // [M] 1/rms per row (unit_scale == 0)
    int M, N, K;
    int pm_blocks, n_blocks, k_blocks, num_tiles;  // pm: 256-row blocks of the pair
    int unit_scale;        // 1: y = x W'^T, no row scaling
};

// Pair tile -> (256-row block, column block), GROUP_M row blocks at a time
// down each column block so the tiles in flight share operands in L2.
__device__ __forceinline__ void tile_coords(int tile, const Args &g, int &pm, int &n) {
    const int group_tiles = GROUP_M * g.n_blocks;
    const int group = tile / group_tiles;
    const int first = group * GROUP_M;
    const int rows_in_group = min(g.pm_blocks - first, GROUP_M);
    const int in_group = tile - group * group_tiles;
    pm = first + in_group % rows_in_group;
    n = in_group / rows_in_group;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
flashnorm_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                           const __grid_constant__ CUtensorMap tmap_y, const Args g) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES + EPI_BYTES);
    uint64_t *full = bars, *empty = bars + STAGES;
    uint64_t *acc_full = bars + 2 * STAGES, *acc_empty = bars + 2 * STAGES + 2;
    uint64_t *drained = bars + 2 * STAGES + 4;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 5);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int pair_id = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&full[s]), 1);   // even CTA: its producer's arrive + both CTAs' bytes
            mbar_init(smem_u32(&empty[s]), 1);  // the even CTA's commit
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&acc_full[a]), 1);   // the even CTA's commit
            mbar_init(smem_u32(&acc_empty[a]), 8);  // even CTA: four epilogue warps of each CTA
        }
        mbar_init(smem_u32(drained), 1);
        mbar_init_fence();
    }
    if (warp == 1) {  // whole warp, in both CTAs: the pair's tensor memory
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    gemm::tc_fence_before();
    cluster_sync();  // both CTAs' barriers exist before any remote arrive or copy
    gemm::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer (both CTAs)
        if (lane == 0) {  // one lane runs the ring
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed = 0, armed_parity = 0;  // per stage: loads issued; parity of the phase they complete
            bool ok = true;
            const uint32_t fb0 = map_to_rank(smem_u32(&full[0]), 0);  // the even CTA's stage barriers
            for (int tile = pair_id; ok && tile < g.num_tiles; tile += num_pairs) {
                int pm, n;
                tile_coords(tile, g, pm, n);
                for (int kb = 0; kb < g.k_blocks; ++kb) {
                    if (!mbar_wait_fast(smem_u32(&empty[stage]), phase ^ 1u, &g_device_error)) { ok = false; break; }
                    if (leader) mbar_arrive_expect_tx(smem_u32(&full[stage]), PAIR_STAGE_BYTES);
                    const uint32_t fb = fb0 + (uint32_t)stage * 8u;
                    uint8_t *sa = smem + stage * STAGE_BYTES;
                    tma_load_2d_pair(smem_u32(sa), &tmap_x, kb * BK, pm * 2 * BM + (int)rank * BM, fb);
                    tma_load_2d_pair(smem_u32(sa + A_BYTES), &tmap_w, kb * BK, n * BN + (int)rank * BN_CTA, fb);
                    armed |= 1u << stage;
                    armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            // The even CTA tracks every copy of the pair on its own stage
            // barriers: before exiting it waits (bounded) for the last phase
            // it armed on each stage, so no copy of either CTA is still in
            // flight (immediate on the normal path, where the MMA consumed
            // them all).  The odd CTA stays resident until then (cluster
            // barrier below).
            if (leader)
                for (int s2 = 0; s2 < STAGES; ++s2)
                    if (armed & (1u << s2))
                        mbar_wait(smem_u32(&full[s2]), (armed_parity >> s2) & 1u, &g_device_error);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer (even CTA)
        if (leader && lane == 0) {  // one lane waits and issues
            const uint32_t peer_empty0 = map_to_rank(smem_u32(&empty[0]), 1);
            const uint32_t peer_acc_full0 = map_to_rank(smem_u32(&acc_full[0]), 1);
            const uint64_t a_desc0 = gemm::sw128_kmajor_desc(smem_u32(smem));  // stage 0; stages move the address field
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            bool ok = true;
            for (int tile = pair_id; ok && tile < g.num_tiles; tile += num_pairs, ++it) {
                const int acc = it & 1;
                const uint32_t acc_phase = (it >> 1) & 1;
                if (!mbar_wait_cluster(smem_u32(&acc_empty[acc]), acc_phase ^ 1u, &g_device_error)) break;
                gemm::tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
                for (int kb = 0; kb < g.k_blocks; ++kb) {
                    if (!mbar_wait_fast(smem_u32(&full[stage]), phase, &g_device_error)) { ok = false; break; }
                    gemm::tc_fence_after();
                    const uint64_t ad = a_desc0 + (uint64_t)((stage * STAGE_BYTES) >> 4);
                    const uint64_t bd = ad + (uint64_t)(A_BYTES >> 4);
#pragma unroll
                    for (int k = 0; k < BK / gemm::UMMA_K; ++k)
                        umma_pair(d_tmem, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), (kb | k) != 0 ? 1u : 0u);
                    // the stage is free in both CTAs once these MMAs have read it
                    umma_commit_pair(smem_u32(&empty[stage]));
                    umma_commit_pair(peer_empty0 + (uint32_t)stage * 8u);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                // both CTAs' accumulators of this tile are complete
                umma_commit_pair(smem_u32(&acc_full[acc]));
                umma_commit_pair(peer_acc_full0 + (uint32_t)acc * 8u);
            }
            // tensor memory is released only after every MMA issued here has completed
            umma_commit_pair(smem_u32(drained));
            mbar_wait(smem_u32(drained), 0u, &g_device_error);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue (warps 2..5, both CTAs)
        // Launched right behind the statistics pass (programmatic dependent
        // launch), only these warps wait for its 1/rms to be visible.  A no-op
        // when the kernel was launched normally.
        asm volatile("griddepcontrol.wait;" ::: "memory");
        const int quarter = warp & 3;  // TMEM lanes this warp may access: 32 * quarter ...
        const uint32_t epi = smem_u32(smem + STAGES * STAGE_BYTES) + (uint32_t)quarter * 4096u;
        const uint32_t acc_empty_leader0 = map_to_rank(smem_u32(&acc_empty[0]), 0);
        int issued = 0;
        int it = 0;
        for (int tile = pair_id; tile < g.num_tiles; tile += num_pairs, ++it) {
            int pm, n;
            tile_coords(tile, g, pm, n);
            const int acc = it & 1;
            const uint32_t acc_phase = (it >> 1) & 1;
            if (!mbar_wait(smem_u32(&acc_full[acc]), acc_phase, &g_device_error)) break;
            gemm::tc_fence_after();
            const int row0 = pm * 2 * BM + (int)rank * BM + quarter * 32;
            const int row = row0 + lane;
            const float r = g.unit_scale ? 1.f : (row < g.M ? __ldg(g.inv_rms + row) : 0.f);
            const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * ACC_COLS;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32];
                gemm::tmem_ld_32cols(tbase + c * 32, v);
                const int col0 = n * BN + c * 32;
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
            gemm::tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty_leader0 + (uint32_t)acc * 8u);
        }
        if (lane == 0) bulk_wait_all();
    }

    gemm::tc_fence_before();
    __syncthreads();
    cluster_sync();  // the even CTA's MMAs and copies, which use both CTAs' memory, are done
    if (warp == 1) {
        gemm::tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                     : "memory");
    }
}

}  // namespace pair

// ----------------------------------------------------------------- host side

// The pair projection with a given 1/rms (or unit_scale).  after_stats: the
// launch just before on `s` is the statistics pass writing `inv`; the pair
// kernel is launched as its programmatic dependent (only its epilogue waits).
inline qkn_status launch_gemm_pair(const void *x, const void *Wf, void *y, const float *inv, int64_t M, int64_t N,
                                   int64_t K, bool unit_scale, cudaStream_t s, bool after_stats) {
    CUtensorMap tx, tw, ty;
    if (qkn_status st = make_tmap(&tx, x, M, K, pair::BM)) return st;
    if (qkn_status st = make_tmap(&tw, Wf, N, K, pair::BN_CTA)) return st;
    if (qkn_status st = make_tmap_store(&ty, y, M, N)) return st;
    pair::Args g;
    g.inv_rms = inv;
    g.unit_scale = unit_scale ? 1 : 0;
    g.M = (int)M;
    g.N = (int)N;
    g.K = (int)K;
    g.pm_blocks = (int)((M + 2 * pair::BM - 1) / (2 * pair::BM));
    g.n_blocks = (int)((N + pair::BN - 1) / pair::BN);
    g.k_blocks = (int)((K + pair::BK - 1) / pair::BK);
    g.num_tiles = g.pm_blocks * g.n_blocks;
    static std::atomic<int> max_pairs[64];  // per device: resident clusters of two (0 until measured)
    int dev = 0;
    cudaGetDevice(&dev);
    const bool known = dev >= 0 && dev < 64;
    int pairs = known ? max_pairs[dev].load(std::memory_order_acquire) : 0;
    if (pairs == 0) {
        cudaError_t e = cudaFuncSetAttribute(pair::flashnorm_gemm_pair_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, pair::SMEM_BYTES);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(flashnorm_gemm_pair_kernel)");
        // a persistent grid must be resident at once: as many pairs as the
        // device keeps resident together (a pair needs both SMs of a TPC)
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (unsigned)(sm_count() / 2), 1, 1);
        cfg.blockDim = dim3(pair::THREADS, 1, 1);
        cfg.dynamicSmemBytes = pair::SMEM_BYTES;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, pair::flashnorm_gemm_pair_kernel, &cfg);
        if (e != cudaSuccess || n <= 0) return cuda_fail(e, "cudaOccupancyMaxActiveClusters(flashnorm_gemm_pair_kernel)");
        pairs = n;
        if (known) max_pairs[dev].store(n, std::memory_order_release);
    }
    const int grid = 2 * (g.num_tiles < pairs ? g.num_tiles : pairs);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(pair::THREADS, 1, 1);
    cfg.dynamicSmemBytes = pair::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = after_stats ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, pair::flashnorm_gemm_pair_kernel, tx, tw, ty, g);
    if (e != cudaSuccess) return cuda_fail(e, "flashnorm_gemm_pair_kernel launch");
    return check_launch("flashnorm_gemm_pair_kernel launch");
}
