// Layerwise QK-Norm with segment-wise scalar statistics (SwiftQK, abstract),
// emulating n_seg tensor-parallel shards of each row on one GPU:
//
//   S_j = sum_{i in segment j} x_i^2   (fp32)
//   S   = ((S_0 + S_1) + ...) + S_{n_seg-1}   (fixed order)
//   y_i = (x_i * rsqrt(S/d + eps)) * w_i      (fp32, one rounding at the store)
//
// Memory-bound: every row is read once and written once.  This file holds
// the entry points qknorm_fused and rmsnorm_partial_stats and the choice of
// kernel, which depends on the row shape, alignment and n_seg only:
//   rownorm_staged.cuh    rows through shared memory by bulk copies (n_seg <= 8)
//   rownorm_register.cuh  a row in registers (wider rows), or element-wise
//                         (unaligned rows)
//   rownorm_cluster.cuh   a row over the CTAs of a cluster (more segments, or
//                         rows wider than a CTA holds)
// Query rows and key rows are two jobs of the same launch.
#include <atomic>
#include <math.h>

#include <mutex>

#include "qkn_common.cuh"
#include "qkn_sync.cuh"

namespace qkn {
// Set by a bounded wait of the staged or cluster kernel that gave up (see qkn_check_device).
__device__ int g_norm_error = 0;
}  // namespace qkn

#include "rownorm_register.cuh"
#include "rownorm_staged.cuh"
#include "rownorm_cluster.cuh"

namespace qkn {

// ---------------------------------------------------------------- host side

namespace {

struct Tensor2 {
    const void *x;
    void *y;
    const void *w;
    int64_t d, ld, ldo;
};

// Rows over the CTAs of C-CTA clusters (C a power of two <= 8).
template <typename TA, typename TW, bool STATS>
qkn_status launch_cluster(const Tensor2 *ts, int njobs, int64_t rows, int n_seg, float eps, float *partial, int C,
                          cudaStream_t s) {
    constexpr int E = Chunk<TA>::E;
    cl::Args a{};
    a.n_seg = n_seg;
    a.eps = eps;
    a.partial = partial;
    a.wait_ns = kWaitTimeoutNs;
    for (int i = 0; i < njobs; ++i) {
        const Tensor2 &t = ts[i];
        cl::Job &J = a.job[i];
        J.x = static_cast<const uint8_t *>(t.x);
        J.y = static_cast<uint8_t *>(t.y);
        J.w = t.w;
        J.ld_bytes = t.ld * (int64_t)sizeof(TA);
        J.ldo_bytes = t.ldo * (int64_t)sizeof(TA);
        J.rows = rows;
        J.d = (int)t.d;
        J.nchunks = (int)(t.d / E);
        J.seg_chunks = J.nchunks / n_seg;
        J.per_cta = (J.nchunks + C - 1) / C;
    }
    // as many clusters as rows, at most as many as are resident at once; each loops over rows
    static std::atomic<int> per_sm[64];  // per instantiation and device; 0 until measured
    int dev = 0;
    cudaGetDevice(&dev);
    const bool known = dev >= 0 && dev < 64;
    int blocks_per_sm = known ? per_sm[dev].load(std::memory_order_relaxed) : 0;
    if (blocks_per_sm == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_per_sm, cl::rownorm_cluster_kernel<TA, TW, STATS>,
                                                          cl::kBlock, 0) != cudaSuccess ||
            blocks_per_sm <= 0) {
            cudaGetLastError();
            blocks_per_sm = 1;
        }
        if (known) per_sm[dev].store(blocks_per_sm, std::memory_order_relaxed);
    }
    const int64_t total = rows * njobs;
    const int64_t fit = (int64_t)blocks_per_sm * sm_count() / C > 0 ? (int64_t)blocks_per_sm * sm_count() / C : 1;
    const int64_t clusters = total < fit ? total : fit;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(clusters * C), 1, 1);
    cfg.blockDim = dim3(cl::kBlock, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = (unsigned)C;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, cl::rownorm_cluster_kernel<TA, TW, STATS>, a);
    if (e != cudaSuccess) return cuda_fail(e, "rownorm_cluster_kernel launch");
    return check_launch("rownorm_cluster_kernel launch");
}

// Widest row (bytes, over the launch's jobs) that the register kernels take
// although the staged kernel's ring would hold it.
constexpr int64_t kRegisterMaxRowBytes = 4096;

// Vector-kernel configurations, tried in order: the first whose CPT covers
// the widest row with at most `max_tpr` threads per row is used.
struct VecCfg { int cpt, block; };
constexpr VecCfg kVecCfgs[] = {{8, 256}, {8, 1024}};
constexpr int kNumVecCfgs = sizeof(kVecCfgs) / sizeof(kVecCfgs[0]);

int ceil_log2(int64_t v) {
    int l = 0;
    while ((int64_t(1) << l) < v) ++l;
    return l;
}

template <typename TA, typename TW, int CPT, int BLOCK, bool STATS>
qkn_status launch_vec(RowArgs &a, int njobs, cudaStream_t s) {
    int64_t blocks = 0;
    for (int i = 0; i < njobs; ++i) blocks += a.job[i].nblocks;
    if (blocks > 0x7fffffffLL) return fail(QKN_ERR_SHAPE, "too many rows for one launch");
    rownorm_vec_kernel<TA, TW, CPT, BLOCK, STATS><<<(unsigned)blocks, BLOCK, 0, s>>>(a);
    return check_launch("rownorm_vec_kernel launch");
}

template <typename TA, typename TW, bool STATS, bool MANY = false>
qkn_status launch_vec_stream(RowArgs &a, int njobs, cudaStream_t s) {
    int64_t groups = 0;
    for (int i = 0; i < njobs; ++i) groups += a.job[i].nblocks;
    const int64_t cap = 2 * (int64_t)sm_count();  // two 256-thread blocks per SM
    const unsigned grid = (unsigned)(groups < cap ? groups : cap);
    // programmatic dependent launch: back-to-back launches overlap one's
    // last blocks with the next one's start (the kernel waits for the
    // previous grid before its first global access)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(stream::BLOCK, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, rownorm_vec_stream_kernel<TA, TW, STATS, MANY>, a);
    if (e != cudaSuccess) return cuda_fail(e, "rownorm_vec_stream_kernel launch");
    return check_launch("rownorm_vec_stream_kernel launch");
}

// Job geometry of the register kernels: a row in 2^tpr_log2 threads of `cpt`
// chunks each, `block` threads per CTA.
template <typename TA>
void setup_vec_jobs(RowArgs &a, const Tensor2 *ts, int njobs, int64_t rows, int n_seg, int cpt, int block) {
    constexpr int E = Chunk<TA>::E;
    for (int i = 0; i < njobs; ++i) {
        const Tensor2 &t = ts[i];
        RowJob &J = a.job[i];
        J.x = static_cast<const uint8_t *>(t.x);
        J.y = static_cast<uint8_t *>(t.y);
        J.w = t.w;
        J.ld_bytes = t.ld * (int64_t)sizeof(TA);
        J.ldo_bytes = t.ldo * (int64_t)sizeof(TA);
        J.rows = rows;
        J.d = (int)t.d;
        J.nchunks = (int)(t.d / E);
        J.seg_chunks = J.nchunks / n_seg;
        J.inv_seg_chunks = 1.0f / (float)J.seg_chunks;
        J.tpr_log2 = ceil_log2((J.nchunks + cpt - 1) / cpt);
        J.rows_per_cta = block >> J.tpr_log2;
        J.nblocks = (rows + J.rows_per_cta - 1) / J.rows_per_cta;
    }
}

// Ring geometry for the staged kernel: stage = the widest row (rounded up to
// 16 bytes); as many consumer warps (at most kMaxWarps) as allow two stages
// per warp next to the fp32 weights within the shared-memory limit.  Returns
// false when even 2 warps x 2 stages do not fit (the register or cluster
// kernel runs).  Each warp also keeps the segment scratch for n_seg.
bool staged_geometry(int64_t max_row_bytes, int64_t w_bytes, int n_seg, int *warps, int *spw, int *stage_bytes) {
    const int64_t sb = (max_row_bytes + 15) / 16 * 16;
    const int64_t scratch = (int64_t)staged::scratch_floats(n_seg) * 4;
    for (int w = staged::kMaxWarps; w >= 2; --w) {
        const int64_t fixed = w_bytes + w * scratch + 8 * w * staged::kMaxStagesPerWarp;
        int64_t per_warp = (staged::kSmemLimit - fixed) / (w * sb);
        if (per_warp > staged::kMaxStagesPerWarp) per_warp = staged::kMaxStagesPerWarp;
        if (per_warp >= 2) {
            *warps = w;
            *spw = (int)per_warp;
            *stage_bytes = (int)sb;
            return true;
        }
    }
    return false;
}

// One-shot fault injection for testing the bounded waits (this host thread's
// next staged-kernel launch); see qkn_testing_arm_wait_fault.
thread_local uint64_t t_fault_wait_ns = 0;

// One instantiation of the staged kernel, launched with programmatic stream
// serialisation, so back-to-back launches overlap one grid's launch and
// setup with the previous one's tail.
template <typename TA, typename TW, bool STATS, int FLAVOR>
qkn_status launch_staged_kernel(const staged::Args &a, int grid, int smem, cudaStream_t s) {
    // the attribute is a cap: set once per device to the whole budget the
    // geometry ever asks for
    static std::atomic<bool> attr_set[64];
    int dev = 0;
    cudaGetDevice(&dev);
    const bool known = dev >= 0 && dev < 64;
    if (!known || !attr_set[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(staged::rownorm_staged_kernel<TA, TW, STATS, FLAVOR>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, QKN_STAGED_SMEM_LIMIT);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(rownorm_staged_kernel)");
        if (known) attr_set[dev].store(true, std::memory_order_release);
    }
    static_assert(QKN_STAGED_SMEM_LIMIT <= 227 * 1024, "the staged geometry's budget is a valid attribute");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(32 * a.warps, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, staged::rownorm_staged_kernel<TA, TW, STATS, FLAVOR>, a);
    if (e != cudaSuccess) return cuda_fail(e, "rownorm_staged_kernel launch");
    return check_launch("rownorm_staged_kernel launch");
}

template <typename TA, typename TW, bool STATS>
qkn_status launch_staged(const Tensor2 *ts, int njobs, int64_t rows, int n_seg, float eps, float *partial,
                         int warps, int spw, int stage_bytes, cudaStream_t s) {
    constexpr int E = Chunk<TA>::E;
    staged::Args a{};
    a.njobs = njobs;
    a.n_seg = n_seg;
    a.eps = eps;
    a.partial = partial;
    a.total_tiles = 0;
    a.warps = warps;
    a.stages = warps * spw;
    a.stage_bytes = stage_bytes;
    a.w_bytes = 0;
    a.wait_ns = kWaitTimeoutNs;
    a.fault_warp = -1;
    a.scratch_floats = staged::scratch_floats(n_seg);
    if (t_fault_wait_ns != 0) {
        a.wait_ns = t_fault_wait_ns;
        a.fault_warp = 0;
        t_fault_wait_ns = 0;
    }
    for (int i = 0; i < njobs; ++i) {
        const Tensor2 &t = ts[i];
        staged::Job &J = a.job[i];
        J.x = static_cast<const uint8_t *>(t.x);
        J.y = static_cast<uint8_t *>(t.y);
        J.w = t.w;
        J.ld_bytes = t.ld * (int64_t)sizeof(TA);
        J.ldo_bytes = t.ldo * (int64_t)sizeof(TA);
        J.rows = rows;
        J.d = (int)t.d;
        J.row_bytes = (int)(t.d * (int64_t)sizeof(TA));
        J.nchunks = (int)(t.d / E);
        J.seg_chunks = J.nchunks / n_seg;
        J.w_offset = a.w_bytes;
        if (!STATS) a.w_bytes += (int)(t.d * 4);
        J.rows_per_tile = stage_bytes / J.row_bytes;
        // rows the register kernels take on their own keep those kernels'
        // arithmetic (staged::process_rows_reg), a whole number of warp
        // passes per tile (a stage holds at least one: 32 / tpr rows of at
        // most tpr x 128 bytes)
        J.reg_tpr_log2 = -1;
        J.inv_seg_chunks = 1.0f / (float)J.seg_chunks;
        if (n_seg <= kFastMaxSeg && J.nchunks <= 32 * stream::CPT) {
            J.reg_tpr_log2 = ceil_log2((J.nchunks + stream::CPT - 1) / stream::CPT);
            const int rpw = 32 >> J.reg_tpr_log2;
            if (J.rows_per_tile >= rpw) J.rows_per_tile = J.rows_per_tile / rpw * rpw;
        }
        J.ntiles = (rows + J.rows_per_tile - 1) / J.rows_per_tile;
        a.total_tiles += J.ntiles;
    }
    const int smem = staged::smem_bytes(a.warps, a.stages, a.stage_bytes, a.w_bytes, a.scratch_floats);
    const int64_t grid = a.total_tiles < sm_count() ? a.total_tiles : sm_count();
    if (n_seg > kFastMaxSeg)
        return launch_staged_kernel<TA, TW, STATS, staged::kFlavorManySeg>(a, (int)grid, smem, s);
    bool reg_rows = false;
    for (int i = 0; i < njobs; ++i) reg_rows = reg_rows || a.job[i].reg_tpr_log2 >= 0;
    if (reg_rows) return launch_staged_kernel<TA, TW, STATS, staged::kFlavorRegRows>(a, (int)grid, smem, s);
    return launch_staged_kernel<TA, TW, STATS, staged::kFlavorGeneric>(a, (int)grid, smem, s);
}

// rmsnorm_partial_stats on rows the staged kernel would take: rows read
// straight from global memory (rowstats_direct_kernel).
template <typename TA>
qkn_status launch_stats_direct(const Tensor2 &t, int64_t rows, int n_seg, float *partial, cudaStream_t s) {
    constexpr int E = Chunk<TA>::E;
    staged::Args a{};
    a.njobs = 1;
    a.n_seg = n_seg;
    a.partial = partial;
    staged::Job &J = a.job[0];
    J.x = static_cast<const uint8_t *>(t.x);
    J.ld_bytes = t.ld * (int64_t)sizeof(TA);
    J.rows = rows;
    J.d = (int)t.d;
    J.row_bytes = (int)(t.d * (int64_t)sizeof(TA));
    J.nchunks = (int)(t.d / E);
    J.seg_chunks = J.nchunks / n_seg;
    a.scratch_floats = staged::scratch_floats(n_seg);
    const int64_t need = (rows + 7) / 8, cap = 4 * (int64_t)sm_count();
    const unsigned grid = (unsigned)(need < cap ? need : cap);
    if (n_seg <= kFastMaxSeg) {
        staged::rowstats_direct_kernel<TA, false><<<grid, 256, 0, s>>>(a);
    } else {
        // up to 64 slots of 33 floats per warp: at most 8 warps x 8448 bytes,
        // above the default 48 KiB, so the cap is raised once per device
        const int smem = 8 * a.scratch_floats * 4;
        static std::atomic<bool> attr_set[64];
        int dev = 0;
        cudaGetDevice(&dev);
        const bool known = dev >= 0 && dev < 64;
        if (!known || !attr_set[dev].load(std::memory_order_acquire)) {
            const cudaError_t e = cudaFuncSetAttribute(staged::rowstats_direct_kernel<TA, true>,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       8 * staged::scratch_floats(QKN_MAX_SEG) * 4);
            if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(rowstats_direct_kernel)");
            if (known) attr_set[dev].store(true, std::memory_order_release);
        }
        staged::rowstats_direct_kernel<TA, true><<<grid, 256, smem, s>>>(a);
    }
    return check_launch("rowstats_direct_kernel launch");
}

// The kernel a set of rows takes, and its launch parameters.  The per-row
// arithmetic of each kind depends on the row's own width, dtype and n_seg
// (and, for clusters, on the cluster size), never on the rows that share
// the launch; dispatch keeps it that way for two jobs (below).
enum class Kernel { kRegisterMany, kStaged, kRegister, kCluster, kScalar };
struct Route {
    Kernel kind;
    int cfg;                 // kRegister: kVecCfgs entry
    bool stream;             // kRegister: the streaming form
    int cluster;             // kCluster: CTAs per row
    int warps, spw, sb;      // kStaged: ring geometry
};

template <typename TA, typename TW, bool STATS>
Route plan(const Tensor2 *ts, int njobs, int n_seg) {
    constexpr int E = Chunk<TA>::E;
    Route r{};
    // 16-byte rows with whole chunks per segment take the vector paths
    bool chunked = true;
    int64_t max_chunks = 0;
    for (int i = 0; i < njobs && chunked; ++i) {
        const Tensor2 &t = ts[i];
        const size_t es = sizeof(TA);
        const uintptr_t walign = (E * sizeof(TW)) < 16 ? E * sizeof(TW) : 16;
        chunked = aligned(t.x, 16) && (t.ld * es) % 16 == 0 && t.d % E == 0 &&
                  (t.d / n_seg) % E == 0 &&
                  (STATS || (aligned(t.w, walign) && aligned(t.y, 16) && (t.ldo * es) % 16 == 0));
        if (t.d / E > max_chunks) max_chunks = t.d / E;
    }
    if (max_chunks >= (1 << 22)) chunked = false;
    bool vec = chunked && n_seg <= kFastMaxSeg;

    int cfg = -1;
    if (vec) {
        for (int c = 0; c < kNumVecCfgs; ++c) {
            if (max_chunks <= (int64_t)kVecCfgs[c].cpt * kVecCfgs[c].block) { cfg = c; break; }
        }
        if (cfg < 0) vec = false;
    }

    int64_t max_row_bytes = 0;
    for (int i = 0; i < njobs; ++i)
        if (ts[i].d * (int64_t)sizeof(TA) > max_row_bytes) max_row_bytes = ts[i].d * (int64_t)sizeof(TA);
    // Narrow rows go to the register kernel: a stage of the staged kernel
    // holds one row of the launch's widest job, so rows of a few hundred bytes
    // would move in copies too small to keep HBM busy, and each warp would
    // walk its rows one by one.  The bound is where the kernels measured even
    // on B200 (2048 bf16 rows: 2048 + 2048 staged 3 % ahead, 2048 + 512 and
    // 2048 + 256 the streaming register kernel 17-23 % ahead).
    // The choice depends on the row widths alone, never on the row count.
    // More than 8 segments (the register kernel stops at 8) take the staged
    // kernel's many-segment statistic when its ring holds the rows.
    const bool many = chunked && n_seg > kFastMaxSeg;
    // Rows of at most 4 KiB with 9-64 segments: the streaming register kernel
    // with its many-segment statistic (per-chunk sums parked in shared memory,
    // each segment added in chunk order by one lane).
    if (many && max_chunks <= 32 * stream::CPT && max_row_bytes <= kRegisterMaxRowBytes) {
        r.kind = Kernel::kRegisterMany;
        return r;
    }
    if ((vec && max_row_bytes > kRegisterMaxRowBytes) || many) {
        // the ring is sized as for normalising also for the statistics alone,
        // so that both take the same kernel, and summation order, for a row
        int64_t w_bytes = 0;
        for (int i = 0; i < njobs; ++i) w_bytes += ts[i].d * 4;
        if (staged_geometry(max_row_bytes, w_bytes, n_seg, &r.warps, &r.spw, &r.sb)) {
            r.kind = Kernel::kStaged;
            return r;
        }
    }
    if (vec) {
        r.kind = Kernel::kRegister;
        r.cfg = cfg;
        // narrow rows (at most 32 threads per row) stream through persistent
        // blocks that load the next rows while they normalise the current ones
        // (the statistics alone keep the one-shot form, which measured faster
        // for them than the streaming form and than a ring of bulk copies)
        r.stream = !STATS && cfg == 0 && max_chunks <= 32 * stream::CPT;
        return r;
    }
    // chunked rows with more than 8 segments, or wider than one CTA's
    // registers hold: spread each row over the CTAs of a cluster
    if (chunked) {
        const int64_t need = (max_chunks + cl::kMaxChunksPerCta - 1) / cl::kMaxChunksPerCta;
        if (need <= cl::kMaxCluster) {
            int C = 1;
            while (C < need) C <<= 1;
            r.kind = Kernel::kCluster;
            r.cluster = C;
            return r;
        }
    }
    r.kind = Kernel::kScalar;
    return r;
}

template <typename TA, typename TW, bool STATS>
qkn_status launch_route(const Route &r, const Tensor2 *ts, int njobs, int64_t rows, int n_seg, float eps,
                        float *partial, cudaStream_t s) {
    RowArgs a{};
    a.n_seg = n_seg;
    a.eps = eps;
    a.partial = partial;
    switch (r.kind) {
    case Kernel::kRegisterMany:
        setup_vec_jobs<TA>(a, ts, njobs, rows, n_seg, stream::CPT, stream::BLOCK);
        return launch_vec_stream<TA, TW, STATS, true>(a, njobs, s);
    case Kernel::kStaged:
        if (STATS) return launch_stats_direct<TA>(ts[0], rows, n_seg, partial, s);
        return launch_staged<TA, TW, STATS>(ts, njobs, rows, n_seg, eps, partial, r.warps, r.spw, r.sb, s);
    case Kernel::kRegister:
        setup_vec_jobs<TA>(a, ts, njobs, rows, n_seg, kVecCfgs[r.cfg].cpt, kVecCfgs[r.cfg].block);
        if (r.stream) return launch_vec_stream<TA, TW, STATS>(a, njobs, s);
        if (r.cfg == 0) return launch_vec<TA, TW, 8, 256, STATS>(a, njobs, s);
        return launch_vec<TA, TW, 8, 1024, STATS>(a, njobs, s);
    case Kernel::kCluster:
        return launch_cluster<TA, TW, STATS>(ts, njobs, rows, n_seg, eps, partial, r.cluster, s);
    case Kernel::kScalar:
        break;
    }
    for (int i = 0; i < njobs; ++i) {
        const Tensor2 &t = ts[i];
        RowJob &J = a.job[i];
        J.x = static_cast<const uint8_t *>(t.x);
        J.y = static_cast<uint8_t *>(t.y);
        J.w = t.w;
        J.ld_bytes = t.ld * (int64_t)sizeof(TA);
        J.ldo_bytes = t.ldo * (int64_t)sizeof(TA);
        J.rows = rows;
        J.d = (int)t.d;
    }
    const int64_t blocks = rows * njobs;
    if (blocks > 0x7fffffffLL) return fail(QKN_ERR_SHAPE, "too many rows for one launch");
    rownorm_scalar_kernel<TA, TW, STATS><<<(unsigned)blocks, kScalarBlock, 0, s>>>(a);
    return check_launch("rownorm_scalar_kernel launch");
}

// q and k share one launch when each would take the same kind of kernel on
// its own (the same cluster size, for clusters), or when one would take the
// register kernels and the other the staged kernel with at most 8 segments:
// the staged kernel then keeps the register kernels' arithmetic for the
// narrow rows (the prefill arrangement, 5120 + 1024).  Otherwise each goes
// to its own kernel, one launch after the other on the stream.  So the bits
// of a row depend on its own tensor's width, dtype, alignment and n_seg
// only: normalised beside any partner, or alone, it comes out the same, and
// rmsnorm_partial_stats gives the partial sums it was normalised with.
template <typename TA, typename TW, bool STATS>
qkn_status dispatch(const Tensor2 *ts, int njobs, int64_t rows, int n_seg, float eps,
                    float *partial, cudaStream_t s) {
    const Route joint = plan<TA, TW, STATS>(ts, njobs, n_seg);
    if (njobs == 2) {
        const Route r0 = plan<TA, TW, STATS>(ts, 1, n_seg), r1 = plan<TA, TW, STATS>(ts + 1, 1, n_seg);
        const bool same = r0.kind == r1.kind && joint.kind == r0.kind &&
                          (r0.kind != Kernel::kCluster || (r0.cluster == r1.cluster && joint.cluster == r0.cluster));
        const bool reg_in_staged = joint.kind == Kernel::kStaged && n_seg <= kFastMaxSeg &&
                                   ((r0.kind == Kernel::kRegister && r1.kind == Kernel::kStaged) ||
                                    (r0.kind == Kernel::kStaged && r1.kind == Kernel::kRegister));
        if (!same && !reg_in_staged) {
            if (qkn_status st = launch_route<TA, TW, STATS>(r0, ts, 1, rows, n_seg, eps, partial, s)) return st;
            return launch_route<TA, TW, STATS>(r1, ts + 1, 1, rows, n_seg, eps, partial, s);
        }
    }
    return launch_route<TA, TW, STATS>(joint, ts, njobs, rows, n_seg, eps, partial, s);
}

template <bool STATS>
qkn_status dispatch_types(qkn_dtype act, qkn_dtype wdt, const Tensor2 *ts, int njobs, int64_t rows,
                          int n_seg, float eps, float *partial, cudaStream_t s) {
    if (act == QKN_BF16) {
        if (wdt == QKN_BF16) return dispatch<__nv_bfloat16, __nv_bfloat16, STATS>(ts, njobs, rows, n_seg, eps, partial, s);
        return dispatch<__nv_bfloat16, float, STATS>(ts, njobs, rows, n_seg, eps, partial, s);
    }
    if (wdt == QKN_BF16) return dispatch<float, __nv_bfloat16, STATS>(ts, njobs, rows, n_seg, eps, partial, s);
    return dispatch<float, float, STATS>(ts, njobs, rows, n_seg, eps, partial, s);
}

}  // namespace
}  // namespace qkn

using namespace qkn;

extern "C" QKN_API qkn_status qknorm_fused(const void *q, const void *k, const void *wq,
                                           const void *wk, void *q_out, void *k_out, int64_t T,
                                           int64_t dq, int64_t dk, int64_t ldq, int64_t ldk,
                                           int64_t ldq_out, int64_t ldk_out, qkn_dtype act,
                                           qkn_dtype wdt, float eps, int n_seg, void *stream) {
    if (!valid_dtype(act) || !valid_dtype(wdt))
        return fail(QKN_ERR_DTYPE, "qknorm_fused: unknown dtype (act=%d, wdt=%d)", (int)act, (int)wdt);
    const bool has_k = dk > 0;
    if (T < 0 || dq < 1 || dk < 0)
        return fail(QKN_ERR_SHAPE, "qknorm_fused: bad sizes T=%lld dq=%lld dk=%lld", (long long)T,
                    (long long)dq, (long long)dk);
    if (dq > 0x7fffffffLL || dk > 0x7fffffffLL) return fail(QKN_ERR_SHAPE, "qknorm_fused: row too wide");
    if (ldq < dq || (has_k && ldk < dk))
        return fail(QKN_ERR_SHAPE, "qknorm_fused: leading dimension smaller than the row width");
    if ((q_out != nullptr && ldq_out < dq) || (has_k && k_out != nullptr && ldk_out < dk))
        return fail(QKN_ERR_SHAPE, "qknorm_fused: output leading dimension smaller than the row width");
    if (qkn_status st = check_seg(n_seg)) return st;
    if (dq % n_seg != 0 || dk % n_seg != 0)
        return fail(QKN_ERR_SHAPE, "qknorm_fused: dq=%lld / dk=%lld not multiples of n_seg=%d",
                    (long long)dq, (long long)dk, n_seg);
    if (!(eps >= 0.f) || isinf(eps)) return fail(QKN_ERR_EPS, "qknorm_fused: eps must be finite and >= 0");
    if (T == 0) return QKN_OK;  // nothing is read or written: pointers may be NULL
    if (q == nullptr || wq == nullptr) return fail(QKN_ERR_NULL, "qknorm_fused: q and wq are required");
    if (has_k && (k == nullptr || wk == nullptr))
        return fail(QKN_ERR_NULL, "qknorm_fused: k and wk are required when dk > 0");
    const size_t es = dtype_size(act), ws = dtype_size(wdt);
    if (!aligned(q, es) || !aligned(wq, ws) || (q_out && !aligned(q_out, es)) ||
        (has_k && (!aligned(k, es) || !aligned(wk, ws) || (k_out && !aligned(k_out, es)))))
        return fail(QKN_ERR_ALIGN, "qknorm_fused: pointers must be aligned to their element size");

    Tensor2 ts[2];
    ts[0] = {q, q_out ? q_out : const_cast<void *>(q), wq, dq, ldq, q_out ? ldq_out : ldq};
    int njobs = 1;
    if (has_k) {
        ts[1] = {k, k_out ? k_out : const_cast<void *>(k), wk, dk, ldk, k_out ? ldk_out : ldk};
        njobs = 2;
    }
    return dispatch_types<false>(act, wdt, ts, njobs, T, n_seg, eps, nullptr,
                                 static_cast<cudaStream_t>(stream));
}

extern "C" QKN_API qkn_status rmsnorm_partial_stats(const void *x, int64_t rows, int64_t d, int64_t ld,
                                                    qkn_dtype act, int n_seg, float *partial,
                                                    void *stream) {
    if (!valid_dtype(act)) return fail(QKN_ERR_DTYPE, "rmsnorm_partial_stats: unknown dtype %d", (int)act);
    if (rows < 0 || d < 1 || d > 0x7fffffffLL || ld < d)
        return fail(QKN_ERR_SHAPE, "rmsnorm_partial_stats: bad sizes rows=%lld d=%lld ld=%lld",
                    (long long)rows, (long long)d, (long long)ld);
    if (qkn_status st = check_seg(n_seg)) return st;
    if (d % n_seg != 0)
        return fail(QKN_ERR_SHAPE, "rmsnorm_partial_stats: d=%lld not a multiple of n_seg=%d", (long long)d, n_seg);
    if (rows == 0) return QKN_OK;  // nothing is read or written: pointers may be NULL
    if (x == nullptr || partial == nullptr)
        return fail(QKN_ERR_NULL, "rmsnorm_partial_stats: x and partial are required");
    if (!aligned(x, dtype_size(act)) || !aligned(partial, 4))
        return fail(QKN_ERR_ALIGN, "rmsnorm_partial_stats: pointers must be aligned to their element size");
    // the weights are not read in this mode; any aligned pointer satisfies the checks
    Tensor2 t = {x, nullptr, partial, d, ld, 0};
    return dispatch_types<true>(act, act, &t, 1, rows, n_seg, 0.f, partial,
                                static_cast<cudaStream_t>(stream));
}

namespace qkn {
// Reads and clears the staged kernel's device error word (current device).
qkn_status read_norm_error(int *flag) {
    cudaError_t e = cudaMemcpyFromSymbol(flag, g_norm_error, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "reading the norm kernel's device error word");
    if (*flag) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_norm_error, &zero, sizeof zero);
    }
    return QKN_OK;
}
}  // namespace qkn

extern "C" QKN_API qkn_status qkn_testing_arm_wait_fault(uint64_t wait_ns) {
    if (wait_ns == 0 || wait_ns > qkn::kWaitTimeoutNs)
        return qkn::fail(QKN_ERR_SHAPE, "qkn_testing_arm_wait_fault: wait_ns must be in (0, 2e9]");
    qkn::t_fault_wait_ns = wait_ns;
    return QKN_OK;
}
