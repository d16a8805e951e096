// Cluster row kernel: a row spread over the CTAs of a thread-block cluster.
//
// Included by qknorm.cu only: the kernels are instantiated by its dispatch
// and share its device error word g_norm_error (one translation unit).
#pragma once

#include "qkn_common.cuh"
#include "qkn_sync.cuh"
#include "rownorm_register.cuh"

namespace qkn {

// ---------------------------------------------------------------------------
// Rows spread over the CTAs of a thread-block cluster: SwiftQK's shard
// structure on one GPU.  CTA k of a cluster of C holds the contiguous slice
// of chunks [k*per, (k+1)*per) of a row in registers, like a tensor-parallel
// shard, and forms one partial sum of squares for every segment its slice
// touches.  Those scalars are all that is exchanged: thread 0 writes them into
// every CTA's shared memory of the cluster (distributed shared memory) and
// arrives on every CTA's mbarrier; once its own barrier completes, each CTA
// adds the pieces segment by segment and, inside a segment, slice by slice --
// the same fixed order everywhere, so every CTA scales the row by the same
// 1/rms -- and applies the weights to its slice.  Serves rows wider than one
// CTA holds and rows with more than 8 segments.  The exchange buffers
// alternate with the row's parity, every wait is bounded, and a cluster-wide
// barrier before exit keeps each CTA's shared memory alive while peers may
// still write to it.
namespace cl {

constexpr int kBlock = 256;
constexpr int kCpt = 8;                              // chunks per thread
constexpr int kMaxChunksPerCta = kBlock * kCpt;      // 2048 chunks (16384 bf16) per slice
constexpr int kMaxCluster = 8;                       // portable cluster size

struct Job {
    const uint8_t *x;
    uint8_t *y;
    const void *w;
    int64_t ld_bytes, ldo_bytes, rows;
    int d, nchunks, seg_chunks, per_cta;
};

struct Args {
    Job job[2];
    int n_seg;
    float eps;
    float *partial;   // STATS: [rows][n_seg] (one job)
    uint64_t wait_ns;
};

__device__ __forceinline__ Job pick(const Args &a, int which) {
    const Job &j0 = a.job[0], &j1 = a.job[1];
    Job J;
    J.x = which ? j1.x : j0.x;
    J.y = which ? j1.y : j0.y;
    J.w = which ? j1.w : j0.w;
    J.ld_bytes = which ? j1.ld_bytes : j0.ld_bytes;
    J.ldo_bytes = which ? j1.ldo_bytes : j0.ldo_bytes;
    J.rows = which ? j1.rows : j0.rows;
    J.d = which ? j1.d : j0.d;
    J.nchunks = which ? j1.nchunks : j0.nchunks;
    J.seg_chunks = which ? j1.seg_chunks : j0.seg_chunks;
    J.per_cta = which ? j1.per_cta : j0.per_cta;
    return J;
}

template <typename TA, typename TW, bool STATS>
__global__ void __launch_bounds__(kBlock) rownorm_cluster_kernel(const Args a) {
    constexpr int E = Chunk<TA>::E;
    __shared__ float sq[kMaxChunksPerCta];                // sums of squares of this slice's chunks
    __shared__ float piece[QKN_MAX_SEG];                  // this CTA's partial of each segment it touches
    __shared__ float part[2][kMaxCluster][QKN_MAX_SEG];   // every CTA's partials, by row parity
    __shared__ float seg_sum[QKN_MAX_SEG];                // the row's segment statistics
    __shared__ __align__(8) uint64_t bar[2];
    __shared__ float s_inv;

    const uint32_t rank = cluster_rank(), C = cluster_size();
    const int64_t cid = blockIdx.x / C, nclusters = gridDim.x / C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar[0]), C);  // one arrive per CTA of the cluster
        mbar_init(smem_u32(&bar[1]), C);
        mbar_init_fence();
    }
    cluster_sync();  // every CTA's barriers exist before any remote arrive

    const int64_t total = a.job[0].rows + a.job[1].rows;
    int it = 0;
    for (int64_t r = cid; r < total; r += nclusters, ++it) {
        const int which = r >= a.job[0].rows ? 1 : 0;
        const int64_t row = which ? r - a.job[0].rows : r;
        const Job J = pick(a, which);
        const int c_lo = (int)rank * J.per_cta;
        const int c_hi = min(J.nchunks, c_lo + J.per_cta);
        const uint8_t *xr = J.x + row * J.ld_bytes;

        // 1. this CTA's slice into registers, every load issued before any arithmetic
        uint4 v[kCpt];
#pragma unroll
        for (int i = 0; i < kCpt; ++i) {
            const int c = c_lo + i * kBlock + (int)threadIdx.x;
            v[i] = c < c_hi ? ld_stream(xr + (int64_t)c * 16) : make_uint4(0u, 0u, 0u, 0u);
        }
        const int j0 = c_lo < c_hi ? c_lo / J.seg_chunks : 0;
        const int npieces = c_lo < c_hi ? (c_hi - 1) / J.seg_chunks - j0 + 1 : 0;
        if (npieces == 1) {
            // 2-3. the slice lies in one segment: each thread adds its chunks'
            //      sums in order, a fixed butterfly per warp, the 8 warp sums in order
            float t = 0.f;
#pragma unroll
            for (int i = 0; i < kCpt; ++i) {
                const int c = c_lo + i * kBlock + (int)threadIdx.x;
                if (c < c_hi) {
                    float f[E];
                    Chunk<TA>::unpack(v[i], f);
                    float s = 0.f;
#pragma unroll
                    for (int e = 0; e < E; ++e) s = fmaf(f[e], f[e], s);
                    t += s;
                }
            }
            for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
            if (lane == 0) sq[warp] = t;
            __syncthreads();
            if (threadIdx.x == 0) {
                float s = 0.f;
                for (int w = 0; w < kBlock / 32; ++w) s += sq[w];
                piece[0] = s;
            }
        } else {
            // 2. sum of squares of every chunk
#pragma unroll
            for (int i = 0; i < kCpt; ++i) {
                const int c = c_lo + i * kBlock + (int)threadIdx.x;
                if (c < c_hi) {
                    float f[E];
                    Chunk<TA>::unpack(v[i], f);
                    float s = 0.f;
#pragma unroll
                    for (int e = 0; e < E; ++e) s = fmaf(f[e], f[e], s);
                    sq[c - c_lo] = s;
                }
            }
            __syncthreads();
            // 3. one partial per segment touched: lane l adds its contiguous share of
            //    the piece's chunks in order, then a fixed butterfly over the warp
            for (int p = warp; p < npieces; p += kBlock / 32) {
                const int j = j0 + p;
                const int lo = max(c_lo, j * J.seg_chunks) - c_lo;
                const int len = min(c_hi, (j + 1) * J.seg_chunks) - c_lo - lo;
                const int b0 = lo + (lane * len) / 32, b1 = lo + ((lane + 1) * len) / 32;
                float s = 0.f;
                for (int k = b0; k < b1; ++k) s += sq[k];
                for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
                if (lane == 0) piece[p] = s;
            }
        }
        __syncthreads();
        const int buf = it & 1;
        if (warp == 0) {
            if (C > 1) {
                // 4. the scalars to every CTA of the cluster (lanes share the stores),
                //    then one arrive on each CTA's barrier
                for (int idx = lane; idx < npieces * (int)C; idx += 32) {
                    const int p = idx % npieces;
                    const uint32_t q = (uint32_t)(idx / npieces);
                    st_cluster_f32(map_to_rank(smem_u32(&part[buf][rank][j0 + p]), q), piece[p]);
                }
                asm volatile("fence.acq_rel.cluster;" ::: "memory");
                __syncwarp();
                if (lane < (int)C) mbar_arrive_cluster(map_to_rank(smem_u32(&bar[buf]), (uint32_t)lane));
                mbar_wait_cluster(smem_u32(&bar[buf]), (uint32_t)(it >> 1) & 1u, &g_norm_error, a.wait_ns);
            }
            // 5. each segment from its slices in order (one lane per segment), then
            //    the segments left to right
            for (int j = lane; j < a.n_seg; j += 32) {
                float Sj = 0.f;
                if (C == 1) {
                    Sj += piece[j];  // one slice: the whole row, j0 == 0
                } else {
                    for (uint32_t k = 0; k < C; ++k) {
                        const int klo = (int)k * J.per_cta, khi = min(J.nchunks, klo + J.per_cta);
                        if (klo < khi && klo < (j + 1) * J.seg_chunks && j * J.seg_chunks < khi)
                            Sj += part[buf][k][j];
                    }
                }
                seg_sum[j] = Sj;
                if constexpr (STATS) {
                    if (rank == 0) a.partial[row * a.n_seg + j] = Sj;
                }
            }
            __syncwarp();
            if (lane == 0) {
                float S = 0.f;
                for (int j = 0; j < a.n_seg; ++j) S += seg_sum[j];
                s_inv = rsqrtf(S / (float)J.d + a.eps);
            }
        }
        __syncthreads();
        if constexpr (!STATS) {
            // 6. weights and one rounding per element, on this CTA's slice
            const float inv = s_inv;
            uint8_t *yr = J.y + row * J.ldo_bytes;
            const TW *w = static_cast<const TW *>(J.w);
#pragma unroll
            for (int i = 0; i < kCpt; ++i) {
                const int c = c_lo + i * kBlock + (int)threadIdx.x;
                if (c < c_hi) {
                    float f[E], wf[E];
                    Chunk<TA>::unpack_again(v[i], f);
                    load_weights<TW, E>(w + (int64_t)c * E, wf);
#pragma unroll
                    for (int e = 0; e < E; ++e) f[e] = (f[e] * inv) * wf[e];
                    st_stream(yr + (int64_t)c * 16, Chunk<TA>::pack(f));
                }
            }
        }
    }
    cluster_sync();  // no CTA leaves while a peer may still write to its shared memory
}

}  // namespace cl

}  // namespace qkn
