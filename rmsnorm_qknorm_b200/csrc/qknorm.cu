// Layerwise QK-Norm with segment-wise scalar statistics (SwiftQK, abstract),
// emulating n_seg tensor-parallel shards of each row on one GPU:
//
//   S_j = sum_{i in segment j} x_i^2   (fp32)
//   S   = ((S_0 + S_1) + ...) + S_{n_seg-1}   (fixed order)
//   y_i = (x_i * rsqrt(S/d + eps)) * w_i      (fp32, one rounding at the store)
//
// Memory-bound: every row is read once and written once.  The vectorised
// kernel keeps a whole row in registers (16-byte chunks spread over a group
// of `tpr` threads), so nothing is re-read from HBM between the statistic and
// the apply step.  Segment partials are reduced with warp shuffles (and shared
// memory when a row spans several warps), then combined left to right -- the
// on-chip analogue of the shards' scalar exchange.  Query rows and key rows
// are two jobs of the same launch.
#include <atomic>
#include <math.h>

#include <mutex>

#include "qkn_common.cuh"
#include "qkn_sync.cuh"

namespace qkn {

// Set by a bounded wait of the staged kernel that gave up (see qkn_check_device).
__device__ int g_norm_error = 0;

constexpr int kFastMaxSeg = 8;    // segments handled by the vectorised kernel
constexpr int kMaxWarps = 32;     // 1024-thread blocks at most

// One set of rows to normalise (the query rows or the key rows).
struct RowJob {
    const uint8_t *x;     // row 0 of the input
    uint8_t *y;           // row 0 of the output (may equal x: in place)
    const void *w;        // weights [d]
    int64_t ld_bytes;     // input row pitch in bytes
    int64_t ldo_bytes;    // output row pitch in bytes
    int64_t rows;
    int d;                // row width in elements
    int nchunks;          // d / elements-per-16-byte-chunk   (vector kernel)
    int seg_chunks;       // chunks per segment               (vector kernel)
    float inv_seg_chunks; // 1 / seg_chunks, for the segment index of a chunk
    int tpr_log2;         // log2(threads per row)            (vector kernel)
    int rows_per_cta;
    int64_t nblocks;
};

struct RowArgs {
    RowJob job[2];
    int n_seg;
    float eps;
    float *partial;       // [rows][n_seg] output of the statistics-only mode
};

// Field-wise select of job 0 or 1 (keeps the kernel parameters in the
// constant bank instead of copying the array to local memory).
__device__ __forceinline__ RowJob pick_job(const RowArgs &a, int which) {
    const RowJob &j0 = a.job[0], &j1 = a.job[1];
    RowJob J;
    J.x = which ? j1.x : j0.x;
    J.y = which ? j1.y : j0.y;
    J.w = which ? j1.w : j0.w;
    J.ld_bytes = which ? j1.ld_bytes : j0.ld_bytes;
    J.ldo_bytes = which ? j1.ldo_bytes : j0.ldo_bytes;
    J.rows = which ? j1.rows : j0.rows;
    J.d = which ? j1.d : j0.d;
    J.nchunks = which ? j1.nchunks : j0.nchunks;
    J.seg_chunks = which ? j1.seg_chunks : j0.seg_chunks;
    J.inv_seg_chunks = which ? j1.inv_seg_chunks : j0.inv_seg_chunks;
    J.tpr_log2 = which ? j1.tpr_log2 : j0.tpr_log2;
    J.rows_per_cta = which ? j1.rows_per_cta : j0.rows_per_cta;
    J.nblocks = which ? j1.nblocks : j0.nblocks;
    return J;
}

// ---------------------------------------------------------------------------
// Vectorised kernel: a row lives in the registers of 2^tpr_log2 threads, each
// holding up to CPT 16-byte chunks (chunk c of the row sits in thread c % tpr,
// slot c / tpr, so every load instruction of a warp is fully coalesced).
// STATS = true writes the n_seg partials instead of normalising.
// Register cap: 1024 / BLOCK blocks per SM, i.e. 64 registers per thread, so
// an SM keeps at least 1024 threads x CPT x 16 B of loads in flight.
template <typename TA, typename TW, int CPT, int BLOCK, bool STATS>
__global__ void __launch_bounds__(BLOCK, 1024 / BLOCK) rownorm_vec_kernel(const RowArgs a) {
    constexpr int E = Chunk<TA>::E;
    __shared__ float red[kMaxWarps][kFastMaxSeg];

    int64_t b = blockIdx.x;
    const int which = (b >= a.job[0].nblocks) ? 1 : 0;
    if (which) b -= a.job[0].nblocks;
    const RowJob J = pick_job(a, which);
    const int tpr_log2 = J.tpr_log2;
    const int tpr = 1 << tpr_log2;
    const int lrow = threadIdx.x >> tpr_log2;
    const int t = threadIdx.x & (tpr - 1);
    const int64_t row = b * J.rows_per_cta + lrow;
    const bool active = row < J.rows;
    const int nchunks = J.nchunks;

    // 1. issue every load of the row before any arithmetic
    const uint8_t *xr = J.x + (active ? row : 0) * J.ld_bytes;
    uint4 v[CPT];
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = i * tpr + t;
        if (active && c < nchunks) v[i] = ld_stream(xr + (int64_t)c * 16);
        else v[i] = make_uint4(0u, 0u, 0u, 0u);
    }

    // 2. per-thread partial sum of squares of each segment
    float acc[kFastMaxSeg];
#pragma unroll
    for (int j = 0; j < kFastMaxSeg; ++j) acc[j] = 0.f;
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = i * tpr + t;
        float f[E];
        Chunk<TA>::unpack(v[i], f);
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) s = fmaf(f[e], f[e], s);
        // floor(c / seg_chunks): (c + 0.5) / seg_chunks is never an integer, and
        // the fp32 error stays below 0.5 / seg_chunks for c < 2^22 (host-checked)
        const int seg = __float2int_rz(((float)c + 0.5f) * J.inv_seg_chunks);
#pragma unroll
        for (int j = 0; j < kFastMaxSeg; ++j) acc[j] += (j == seg) ? s : 0.f;
    }

    // 3. reduce each segment over the threads of the row (fixed tree)
    const int n_seg = a.n_seg;
    const int lanes = tpr < 32 ? tpr : 32;
#pragma unroll
    for (int j = 0; j < kFastMaxSeg; ++j) {
        if (j < n_seg) {
            for (int off = lanes >> 1; off > 0; off >>= 1)
                acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
        }
    }
    if (tpr > 32) {  // uniform per block: a block serves one job
        const int warp = threadIdx.x >> 5;
        if ((threadIdx.x & 31) == 0) {
#pragma unroll
            for (int j = 0; j < kFastMaxSeg; ++j)
                if (j < n_seg) red[warp][j] = acc[j];
        }
        __syncthreads();
        const int wpr = tpr >> 5;
        const int w0 = lrow * wpr;
#pragma unroll
        for (int j = 0; j < kFastMaxSeg; ++j) {
            if (j < n_seg) {
                float s = 0.f;
                for (int w = 0; w < wpr; ++w) s += red[w0 + w][j];
                acc[j] = s;
            }
        }
    }

    if constexpr (STATS) {
        if (active && t == 0) {
            float *p = a.partial + row * n_seg;
#pragma unroll
            for (int j = 0; j < kFastMaxSeg; ++j)
                if (j < n_seg) p[j] = acc[j];
        }
        return;
    } else {
        // 4. combine the segment statistics left to right, then scale
        float S = 0.f;
#pragma unroll
        for (int j = 0; j < kFastMaxSeg; ++j)
            if (j < n_seg) S += acc[j];
        const float inv = rsqrtf(S / (float)J.d + a.eps);

        // 5. apply the weights and store, one rounding per element
        uint8_t *yr = J.y + (active ? row : 0) * J.ldo_bytes;
        const TW *w = static_cast<const TW *>(J.w);
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int c = i * tpr + t;
            if (active && c < nchunks) {
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

// ---------------------------------------------------------------------------
// Staged kernel (rows up to ~40 KiB): persistent, one block per SM.
//
// Rows reach shared memory through 1-D bulk copies (cp.async.bulk, completion
// counted on an mbarrier per stage), so the loads in flight do not depend on
// what the threads are computing.  Every warp is both producer and consumer:
// warp w handles every W-th "tile" of the block (whole rows of one job, at
// most one stage of bytes) and owns `spw` stages of its own; as soon as it has
// read a stage it refills it with its tile spw steps ahead, so while it works
// on one stage the copies into its other stages are in flight, and no warp
// ever waits for another warp's progress.  A warp reads each row twice from
// shared memory -- the segment statistic, then the apply -- and writes the
// output from registers with streaming stores.  The weights of both jobs are
// widened to fp32 once per block and kept in shared memory, split into the
// low and high 16-byte halves of each chunk so a warp's weight loads are
// conflict-free.  Products use the packed fp32x2 pipe (two fp32 lanes per
// instruction, each rounded exactly like a scalar fp32 operation).
//
// Segment partials: a lane's chunks c = lane, lane + 32, ... visit segments
// in increasing order, so the lane keeps one running (even, odd) pair of sums
// and parks their total in a per-warp shared-memory slot [segment][lane] when
// it crosses a segment boundary.  The eight slots are then reduced over the
// warp by recursive halving (lane bit 4 splits segments 0-3 / 4-7, bit 3 and
// bit 2 split further, bits 1 and 0 finish the sum), after which lanes
// 4j .. 4j+3 hold segment j; the segments are combined left to right.
namespace staged {

#ifndef QKN_STAGED_SMEM_LIMIT
#define QKN_STAGED_SMEM_LIMIT (227 * 1024)
#endif
#ifndef QKN_STAGED_MAX_WARPS
#define QKN_STAGED_MAX_WARPS 8
#endif
#ifndef QKN_STAGED_MAX_SPW
#define QKN_STAGED_MAX_SPW 3
#endif

constexpr int kSmemLimit = QKN_STAGED_SMEM_LIMIT;    // whole dynamic shared memory
constexpr int kMaxWarps = QKN_STAGED_MAX_WARPS;       // consumer warps
constexpr int kMaxStagesPerWarp = QKN_STAGED_MAX_SPW;
constexpr int kMaxThreads = 32 * kMaxWarps;
#ifndef QKN_STAGED_UNROLL
#define QKN_STAGED_UNROLL 4
#endif
constexpr int kUnroll = QKN_STAGED_UNROLL;             // chunks per lane per group
static_assert(kFastMaxSeg == 8, "the warp reduction below is written for 8 segment slots");

struct Job {
    const uint8_t *x;
    uint8_t *y;
    const void *w;
    int64_t ld_bytes, ldo_bytes, rows;
    int d, row_bytes, nchunks, seg_chunks;
    int w_offset;        // byte offset of this job's fp32 weights in shared memory
    int rows_per_tile;
    int narrow_cpl;      // 1, 2 or 4: a narrow row whose segments are whole lane groups; 0 otherwise
    int64_t ntiles;
};

struct Args {
    Job job[2];
    int njobs;
    int64_t total_tiles;
    int n_seg;
    float eps;
    float *partial;
    int warps;        // consumer warps W
    int stages;       // W * stages per warp
    int stage_bytes;  // multiple of 16
    int w_bytes;      // fp32 weights of both jobs
    uint64_t wait_ns;  // limit of every mbarrier wait
    int fault_warp;   // testing only: this block*W+warp skips its first tile's copies (-1: none)
};

// Shared memory: [ring][fp32 weights][full bars][W x 8 x 32 floats scratch]
inline int smem_bytes(int warps, int stages, int stage_bytes, int w_bytes) {
    return stages * stage_bytes + w_bytes + stages * 8 + warps * kFastMaxSeg * 32 * 4;
}

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
    J.row_bytes = which ? j1.row_bytes : j0.row_bytes;
    J.nchunks = which ? j1.nchunks : j0.nchunks;
    J.seg_chunks = which ? j1.seg_chunks : j0.seg_chunks;
    J.w_offset = which ? j1.w_offset : j0.w_offset;
    J.rows_per_tile = which ? j1.rows_per_tile : j0.rows_per_tile;
    J.narrow_cpl = which ? j1.narrow_cpl : j0.narrow_cpl;
    J.ntiles = which ? j1.ntiles : j0.ntiles;
    return J;
}

// fp32 pairs of a 16-byte activation chunk.
template <typename TA> struct Pairs;
template <> struct Pairs<__nv_bfloat16> {
    static constexpr int P = 4;
    __device__ __forceinline__ static void get(const uint4 &v, float2 (&p)[P]) {
        p[0] = make_float2(bf16lo(v.x), bf16hi(v.x));
        p[1] = make_float2(bf16lo(v.y), bf16hi(v.y));
        p[2] = make_float2(bf16lo(v.z), bf16hi(v.z));
        p[3] = make_float2(bf16lo(v.w), bf16hi(v.w));
    }
    __device__ __forceinline__ static uint4 put(const float2 (&p)[P]) {
        return make_uint4(pack_bf16x2(p[0].x, p[0].y), pack_bf16x2(p[1].x, p[1].y),
                          pack_bf16x2(p[2].x, p[2].y), pack_bf16x2(p[3].x, p[3].y));
    }
};
template <> struct Pairs<float> {
    static constexpr int P = 2;
    __device__ __forceinline__ static void get(const uint4 &v, float2 (&p)[P]) {
        p[0] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
        p[1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
    }
    __device__ __forceinline__ static uint4 put(const float2 (&p)[P]) {
        return make_uint4(__float_as_uint(p[0].x), __float_as_uint(p[0].y), __float_as_uint(p[1].x),
                          __float_as_uint(p[1].y));
    }
};

// Sum of squares of one 16-byte chunk as an (even, odd) pair: a short
// dependency chain per chunk, so the chunks of a group overlap.
template <typename TA>
__device__ __forceinline__ float2 chunk_sumsq(const uint4 &v) {
    float2 p[Pairs<TA>::P];
    Pairs<TA>::get(v, p);
    float2 a = __fmul2_rn(p[0], p[0]);
#pragma unroll
    for (int i = 1; i < Pairs<TA>::P; ++i) a = __ffma2_rn(p[i], p[i], a);
    return a;
}

// Adds a chunk's sum into the running pair sum, parking the running sum of
// the segment being left whenever chunk c crosses a segment boundary.
__device__ __forceinline__ void accumulate(float2 sq, int c, float2 &cur, int &cur_seg, int &next_bound,
                                           int seg_chunks, float *part, int lane) {
    while (c >= next_bound) {
        part[cur_seg * 32 + lane] = cur.x + cur.y;
        cur = make_float2(0.f, 0.f);
        ++cur_seg;
        next_bound += seg_chunks;
    }
    cur = __fadd2_rn(cur, sq);
}

// y = (x * inv) * w for one chunk c, stored with a streaming store.
template <typename TA>
__device__ __forceinline__ void apply_chunk(const uint4 &v, int c, float2 inv2, const float4 *wsm, int nchunks,
                                            uint8_t *yr) {
    float4 w[Pairs<TA>::P / 2];
#pragma unroll
    for (int h = 0; h < Pairs<TA>::P / 2; ++h) w[h] = wsm[h * nchunks + c];
    float2 p[Pairs<TA>::P];
    Pairs<TA>::get(v, p);
#pragma unroll
    for (int h = 0; h < Pairs<TA>::P / 2; ++h) {
        p[2 * h] = __fmul2_rn(__fmul2_rn(p[2 * h], inv2), make_float2(w[h].x, w[h].y));
        p[2 * h + 1] = __fmul2_rn(__fmul2_rn(p[2 * h + 1], inv2), make_float2(w[h].z, w[h].w));
    }
    st_stream_batched(yr + (int64_t)c * 16, Pairs<TA>::put(p));
}

// Statistic of one row held in shared memory, by one warp (any width): lane
// l adds its chunks l, l + 32, ... in order into a running pair sum that is
// parked in the warp's [8][32] scratch `part` whenever a segment ends; the 8
// slots are reduced over the warp by recursive halving (lanes 4j .. 4j+3 end
// with segment j) and the segments added left to right.  Returns S.
template <typename TA, bool STATS>
__device__ __forceinline__ float row_statistic(const Args &a, const Job &J, const uint8_t *srow, int64_t row,
                                               int lane, float *part) {
    const int nchunks = J.nchunks;
    const int n_seg = a.n_seg;
    const int sc = J.seg_chunks;
#pragma unroll
    for (int j = 0; j < kFastMaxSeg; ++j) part[j * 32 + lane] = 0.f;
    float2 cur = make_float2(0.f, 0.f);
    int cur_seg = 0, next_bound = sc;
    int c0 = 0;
    constexpr int G = 32 * kUnroll;  // chunks per group
    if (nchunks >= G) {
        // groups of kUnroll chunks per lane; the next group's loads are issued
        // before the current group's arithmetic
        uint4 vn[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) vn[u] = *reinterpret_cast<const uint4 *>(srow + (u * 32 + lane) * 16);
        for (; c0 + G <= nchunks; c0 += G) {
            uint4 v[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) v[u] = vn[u];
            if (c0 + 2 * G <= nchunks) {
#pragma unroll
                for (int u = 0; u < kUnroll; ++u)
                    vn[u] = *reinterpret_cast<const uint4 *>(srow + (c0 + G + u * 32 + lane) * 16);
            }
            float2 sq[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) sq[u] = chunk_sumsq<TA>(v[u]);
            if (c0 + (kUnroll - 1) * 32 + lane < next_bound) {  // the whole group is in the current segment
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) cur = __fadd2_rn(cur, sq[u]);
            } else {
#pragma unroll
                for (int u = 0; u < kUnroll; ++u)
                    accumulate(sq[u], c0 + u * 32 + lane, cur, cur_seg, next_bound, sc, part, lane);
            }
        }
    }
    for (; c0 < nchunks; c0 += 32) {
        const int c = c0 + lane;
        if (c < nchunks)
            accumulate(chunk_sumsq<TA>(*reinterpret_cast<const uint4 *>(srow + c * 16)), c, cur, cur_seg,
                       next_bound, sc, part, lane);
    }
    part[cur_seg * 32 + lane] = cur.x + cur.y;
    __syncwarp();

    float S = 0.f;
    if (n_seg == 1) {
        float r = part[lane];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
        S = r;
        if constexpr (STATS) {
            if (lane == 0) a.partial[row] = r;
        }
    } else {
        float v8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v8[j] = part[j * 32 + lane];
        const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
        float k4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float give = b4 ? v8[i] : v8[i + 4];
            k4[i] = (b4 ? v8[i + 4] : v8[i]) + __shfl_xor_sync(0xffffffffu, give, 16);
        }
        float k2[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float give = b3 ? k4[i] : k4[i + 2];
            k2[i] = (b3 ? k4[i + 2] : k4[i]) + __shfl_xor_sync(0xffffffffu, give, 8);
        }
        float r = (b2 ? k2[1] : k2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? k2[0] : k2[1], 4);
        r += __shfl_xor_sync(0xffffffffu, r, 2);
        r += __shfl_xor_sync(0xffffffffu, r, 1);
        // lanes 4j .. 4j+3 now hold segment j; combine left to right
        for (int j = 0; j < n_seg; ++j) S += __shfl_sync(0xffffffffu, r, 4 * j);
        if constexpr (STATS) {
            if ((lane & 3) == 0 && (lane >> 2) < n_seg) a.partial[row * n_seg + (lane >> 2)] = r;
        }
    }
    __syncwarp();  // the scratch is rewritten by the next row

    return S;
}

// Statistic of a narrow row (32 * CPL chunks, CPL <= 4) whose segments are
// whole groups of lanes: lane l sums its CPL contiguous chunks l*CPL ..
// l*CPL + CPL - 1 (all in segment l / LPS, LPS = 32 / n_seg lanes per
// segment), visiting them in an order rotated with the lane so a warp's
// 16-byte shared-memory reads take the fewest wavefronts; then each segment
// is reduced over its lanes (a fixed butterfly) and the segments are added
// left to right.  Nothing is parked: every lane stays inside one segment.
// Returns S; `seg` receives the lane's segment total.
template <typename TA, int CPL>
__device__ __forceinline__ float narrow_statistic(const uint8_t *srow, int lane, int n_seg, float &seg) {
    constexpr int ROT = CPL == 4 ? 1 : 2;  // lanes that share a rotation step
    float2 cur = make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < CPL; ++u) {
        const int c = lane * CPL + ((u + (lane >> ROT)) & (CPL - 1));
        cur = __fadd2_rn(cur, chunk_sumsq<TA>(*reinterpret_cast<const uint4 *>(srow + c * 16)));
    }
    float r = cur.x + cur.y;
    const int lps = 32 / n_seg;
    for (int off = 1; off < lps; off <<= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
    seg = r;
    float tot[kFastMaxSeg];
#pragma unroll
    for (int j = 0; j < kFastMaxSeg; ++j) tot[j] = __shfl_sync(0xffffffffu, r, (j * lps) & 31);
    float S = 0.f;
#pragma unroll
    for (int j = 0; j < kFastMaxSeg; ++j)
        if (j < n_seg) S += tot[j];
    return S;
}

// One row held in shared memory, processed by one warp.  `part` is the warp's
// [8][32] scratch for lane partials; `wsm` the job's fp32 weights.  NARROW:
// the launch has narrow rows (the narrow statistic is compiled in; launches
// without them keep the wide path alone, and its register budget).
template <typename TA, bool STATS, bool NARROW>
__device__ __forceinline__ void process_row(const Args &a, const Job &J, const uint8_t *srow, const float4 *wsm,
                                            int64_t row, int lane, float *part) {
    const int nchunks = J.nchunks;
    float S;
    if (NARROW && J.narrow_cpl != 0) {
        const int n_seg = a.n_seg;
        float seg;
        if (J.narrow_cpl == 1) S = narrow_statistic<TA, 1>(srow, lane, n_seg, seg);
        else if (J.narrow_cpl == 2) S = narrow_statistic<TA, 2>(srow, lane, n_seg, seg);
        else S = narrow_statistic<TA, 4>(srow, lane, n_seg, seg);
        if constexpr (STATS) {
            const int lps = 32 / n_seg;
            if ((lane & (lps - 1)) == 0) a.partial[row * n_seg + lane / lps] = seg;
        }
    } else {
        S = row_statistic<TA, STATS>(a, J, srow, row, lane, part);
    }

    // ---- apply
    if constexpr (!STATS) {
        constexpr int G = 32 * kUnroll;  // chunks per group
        const float inv = rsqrtf(S / (float)J.d + a.eps);
        const float2 inv2 = make_float2(inv, inv);
        uint8_t *yr = J.y + row * J.ldo_bytes;
        int c1 = 0;
        if (nchunks >= G) {
            uint4 vn[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) vn[u] = *reinterpret_cast<const uint4 *>(srow + (u * 32 + lane) * 16);
            for (; c1 + G <= nchunks; c1 += G) {
                uint4 v[kUnroll];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) v[u] = vn[u];
                if (c1 + 2 * G <= nchunks) {
#pragma unroll
                    for (int u = 0; u < kUnroll; ++u)
                        vn[u] = *reinterpret_cast<const uint4 *>(srow + (c1 + G + u * 32 + lane) * 16);
                }
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) apply_chunk<TA>(v[u], c1 + u * 32 + lane, inv2, wsm, nchunks, yr);
            }
        }
        for (; c1 < nchunks; c1 += 32) {
            const int c = c1 + lane;
            if (c < nchunks) apply_chunk<TA>(*reinterpret_cast<const uint4 *>(srow + c * 16), c, inv2, wsm, nchunks, yr);
        }
    }
}

// Issues the bulk copies of one tile into a stage (one lane).
__device__ __forceinline__ void issue_tile(const Args &a, int64_t tile, int64_t nt0, uint8_t *stage_ptr,
                                           uint64_t *bar) {
    const int which = tile >= nt0 ? 1 : 0;
    const Job J = pick(a, which);
    const int64_t row0 = (tile - (which ? nt0 : 0)) * J.rows_per_tile;
    const int64_t left = J.rows - row0;
    const int nrows = left < J.rows_per_tile ? (int)left : J.rows_per_tile;
    const uint32_t fb = smem_u32(bar);
    mbar_arrive_expect_tx(fb, (uint32_t)(nrows * J.row_bytes));
    const uint32_t dst = smem_u32(stage_ptr);
    for (int r = 0; r < nrows; ++r)
        bulk_g2s(dst + r * J.row_bytes, J.x + (row0 + r) * J.ld_bytes, (uint32_t)J.row_bytes, fb);
}

template <typename TA, typename TW, bool STATS, bool NARROW>
__global__ void __launch_bounds__(kMaxThreads, 1) rownorm_staged_kernel(const Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int W = a.warps, SB = a.stage_bytes;
    const int spw = a.stages / W;
    uint8_t *wbase = smem + (size_t)a.stages * SB;
    uint64_t *full = reinterpret_cast<uint64_t *>(wbase + a.w_bytes);
    float *scratch = reinterpret_cast<float *>(full + a.stages);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // Programmatic dependent launch: the next kernel on the stream may be
    // scheduled now (its blocks land on SMs as this grid's blocks exit), and
    // this grid touches no global memory until the previous grid has finished
    // and its writes are visible (a no-op when launched without the attribute).
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) {
        for (int s = 0; s < a.stages; ++s) mbar_init(smem_u32(&full[s]), 1);  // issuing lane + bytes
        mbar_init_fence();
    }
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // The first batch of weight loads goes out before the tile copies, so it
    // does not queue behind them in the memory system; the weights are
    // widened and stored while the copies stream in.
    constexpr int E = Chunk<TA>::E;
    constexpr int WB = 4;  // weight chunks per thread per batch
    float wf[2][WB][E];
    if constexpr (!STATS) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            if (i < a.njobs) {
                const Job J = pick(a, i);
                const TW *w = static_cast<const TW *>(J.w);
#pragma unroll
                for (int u = 0; u < WB; ++u) {
                    const int c = u * (int)blockDim.x + (int)threadIdx.x;
                    if (c < J.nchunks) load_weights_batched<TW, E>(w + (int64_t)c * E, wf[i][u]);
                }
            }
        }
    }

    // Warp w handles this block's tiles w, w + W, w + 2W, ... (k-th: w + k W)
    // and owns stages w*spw .. w*spw + spw - 1; tile k lives in stage
    // w*spw + k % spw.  The warp refills a stage itself as soon as it has
    // read it, so no other warp's progress delays its copies.  (Claiming
    // tiles dynamically from a block-wide counter measured slower: the fixed
    // dealing keeps the whole grid streaming through memory in order.)
    const int64_t nt0 = a.job[0].ntiles;
    const int64_t step = (int64_t)W * gridDim.x;
    const int64_t first = blockIdx.x + (int64_t)warp * gridDim.x;
    float *part = scratch + warp * kFastMaxSeg * 32;
    int64_t issued = 0;  // tiles of this warp whose copies were issued
    if (lane == 0) {
        for (int j = 0; j < spw; ++j) {
            const int64_t tile = first + j * step;
            if (tile >= a.total_tiles) break;
            // (testing only) an injected fault: the copies are never issued, so
            // this stage's wait cannot complete and must give up on its own
            if (!(j == 0 && a.fault_warp == (int)blockIdx.x * W + warp))
                issue_tile(a, tile, nt0, smem + (size_t)(warp * spw + j) * SB, &full[warp * spw + j]);
            ++issued;
        }
    }
    issued = __shfl_sync(0xffffffffu, issued, 0);

    if constexpr (!STATS) {
        // weights of both jobs as fp32 in shared memory, chunk halves de-interleaved
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            if (i >= a.njobs) break;
            const Job J = pick(a, i);
            const TW *w = static_cast<const TW *>(J.w);
            float4 *dst = reinterpret_cast<float4 *>(wbase + J.w_offset);
            for (int c0 = 0; c0 < J.nchunks; c0 += WB * (int)blockDim.x) {
                float f[WB][E];
#pragma unroll
                for (int u = 0; u < WB; ++u) {
                    const int c = c0 + u * (int)blockDim.x + (int)threadIdx.x;
                    if (c < J.nchunks) {
                        if (c0 == 0) {
#pragma unroll
                            for (int e = 0; e < E; ++e) f[u][e] = wf[i][u][e];  // loaded above
                        } else {
                            load_weights_batched<TW, E>(w + (int64_t)c * E, f[u]);
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < WB; ++u) {
                    const int c = c0 + u * (int)blockDim.x + (int)threadIdx.x;
                    if (c < J.nchunks) {
#pragma unroll
                        for (int h = 0; h < E / 4; ++h)
                            dst[h * J.nchunks + c] =
                                make_float4(f[u][4 * h], f[u][4 * h + 1], f[u][4 * h + 2], f[u][4 * h + 3]);
                    }
                }
            }
        }
        __syncthreads();
    }

    int64_t k = 0;
    for (int64_t tile = first; tile < a.total_tiles; tile += step, ++k) {
        const int slot = (int)(k % spw);
        const int stage = warp * spw + slot;
        const uint32_t par = (uint32_t)(k / spw) & 1u;
        if (!mbar_wait(smem_u32(&full[stage]), par, &g_norm_error, a.wait_ns)) break;
        const int which = tile >= nt0 ? 1 : 0;
        const Job J = pick(a, which);
        const int64_t row0 = (tile - (which ? nt0 : 0)) * J.rows_per_tile;
        const int64_t left = J.rows - row0;
        const int nrows = left < J.rows_per_tile ? (int)left : J.rows_per_tile;
        const uint8_t *sbase = smem + (size_t)stage * SB;
        const float4 *wsm = reinterpret_cast<const float4 *>(wbase + J.w_offset);
        for (int r = 0; r < nrows; ++r)
            process_row<TA, STATS, NARROW>(a, J, sbase + r * J.row_bytes, wsm, row0 + r, lane, part);
        __syncwarp();
        // refill this stage with the warp's tile k + spw
        const int64_t next = tile + spw * step;
        if (next < a.total_tiles) {
            if (lane == 0) {
                // the generic-proxy reads of this stage precede the async-proxy writes
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                issue_tile(a, next, nt0, smem + (size_t)stage * SB, &full[stage]);
            }
            ++issued;
        }
    }
    // drain: copies this warp issued but did not consume (only after a failed
    // wait) must land before the block exits
    for (; k < issued; ++k)
        mbar_wait(smem_u32(&full[warp * spw + (int)(k % spw)]), (uint32_t)(k / spw) & 1u, &g_norm_error, a.wait_ns);
}

}  // namespace staged

// ---------------------------------------------------------------------------
// Element-wise kernel for any alignment, width and n_seg <= QKN_MAX_SEG: one
// row per 256-thread block; each segment is reduced over the block in turn.
// The row is read a second time (from L2) for the apply step.
constexpr int kScalarBlock = 256;

template <typename TA, typename TW, bool STATS>
__global__ void __launch_bounds__(kScalarBlock) rownorm_scalar_kernel(const RowArgs a) {
    __shared__ float warp_part[kScalarBlock / 32];
    __shared__ float seg_total[QKN_MAX_SEG];

    int64_t b = blockIdx.x;
    const int which = (b >= a.job[0].rows) ? 1 : 0;
    if (which) b -= a.job[0].rows;
    const RowJob J = pick_job(a, which);
    const TA *x = reinterpret_cast<const TA *>(J.x + b * J.ld_bytes);
    const int d = J.d, n_seg = a.n_seg, seg_len = d / n_seg;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    for (int j = 0; j < n_seg; ++j) {
        float s = 0.f;
        for (int i = threadIdx.x; i < seg_len; i += kScalarBlock) {
            const float f = to_f32<TA>(x[j * seg_len + i]);
            s = fmaf(f, f, s);
        }
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) warp_part[warp] = s;
        __syncthreads();
        if (threadIdx.x == 0) {
            float tot = 0.f;
            for (int w2 = 0; w2 < kScalarBlock / 32; ++w2) tot += warp_part[w2];
            seg_total[j] = tot;
        }
        __syncthreads();
    }

    if constexpr (STATS) {
        for (int j = threadIdx.x; j < n_seg; j += kScalarBlock) a.partial[b * n_seg + j] = seg_total[j];
    } else {
        float S = 0.f;
        for (int j = 0; j < n_seg; ++j) S += seg_total[j];
        const float inv = rsqrtf(S / (float)d + a.eps);
        TA *y = reinterpret_cast<TA *>(J.y + b * J.ldo_bytes);
        const TW *w = static_cast<const TW *>(J.w);
        for (int i = threadIdx.x; i < d; i += kScalarBlock)
            y[i] = from_f32<TA>((to_f32<TA>(x[i]) * inv) * to_f32<TW>(w[i]));
    }
}

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

// Ring geometry for the staged kernel: stage = the widest row (rounded up to
// 16 bytes); as many consumer warps (at most kMaxWarps) as allow two stages
// per warp next to the fp32 weights within the shared-memory limit.  Returns
// false when even 2 warps x 2 stages do not fit (the register kernel runs).
bool staged_geometry(int64_t max_row_bytes, int64_t w_bytes, int *warps, int *spw, int *stage_bytes) {
    const int64_t sb = (max_row_bytes + 15) / 16 * 16;
    for (int w = staged::kMaxWarps; w >= 2; --w) {
        const int64_t fixed = w_bytes + w * kFastMaxSeg * 32 * 4 + 8 * w * staged::kMaxStagesPerWarp;
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
template <typename TA, typename TW, bool STATS, bool NARROW>
qkn_status launch_staged_kernel(const staged::Args &a, int grid, int smem, cudaStream_t s) {
    // the attribute is a cap: set once per device to the whole budget the
    // geometry ever asks for
    static std::atomic<bool> attr_set[64];
    int dev = 0;
    cudaGetDevice(&dev);
    const bool known = dev >= 0 && dev < 64;
    if (!known || !attr_set[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(staged::rownorm_staged_kernel<TA, TW, STATS, NARROW>,
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
    const cudaError_t e = cudaLaunchKernelEx(&cfg, staged::rownorm_staged_kernel<TA, TW, STATS, NARROW>, a);
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
        // narrow rows of 32, 64 or 128 chunks whose segments are whole power-of-two lane groups
        J.narrow_cpl = 0;
        if (J.nchunks % 32 == 0 && J.nchunks <= 128) {
            const int cpl = J.nchunks / 32, lps = 32 / n_seg;
            if (lps * n_seg == 32 && (lps & (lps - 1)) == 0 && J.seg_chunks == cpl * lps) J.narrow_cpl = cpl;
        }
        J.ntiles = (rows + J.rows_per_tile - 1) / J.rows_per_tile;
        a.total_tiles += J.ntiles;
    }
    const int smem = staged::smem_bytes(a.warps, a.stages, a.stage_bytes, a.w_bytes);
    const int64_t grid = a.total_tiles < sm_count() ? a.total_tiles : sm_count();
    bool narrow = false;
    for (int i = 0; i < njobs; ++i) narrow = narrow || a.job[i].narrow_cpl != 0;
    if (narrow) return launch_staged_kernel<TA, TW, STATS, true>(a, (int)grid, smem, s);
    return launch_staged_kernel<TA, TW, STATS, false>(a, (int)grid, smem, s);
}

template <typename TA, typename TW, bool STATS>
qkn_status dispatch(const Tensor2 *ts, int njobs, int64_t rows, int n_seg, float eps,
                    float *partial, cudaStream_t s) {
    constexpr int E = Chunk<TA>::E;
    RowArgs a{};
    a.n_seg = n_seg;
    a.eps = eps;
    a.partial = partial;

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

    if (vec) {
        int64_t max_row_bytes = 0;
        for (int i = 0; i < njobs; ++i)
            if (ts[i].d * (int64_t)sizeof(TA) > max_row_bytes) max_row_bytes = ts[i].d * (int64_t)sizeof(TA);
        int64_t w_bytes = 0;
        for (int i = 0; i < njobs && !STATS; ++i) w_bytes += ts[i].d * 4;
        int warps = 0, spw = 0, sb = 0;
        if (staged_geometry(max_row_bytes, w_bytes, &warps, &spw, &sb))
            return launch_staged<TA, TW, STATS>(ts, njobs, rows, n_seg, eps, partial, warps, spw, sb, s);
    }

    if (vec) {
        const int cpt = kVecCfgs[cfg].cpt, block = kVecCfgs[cfg].block;
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
        if (cfg == 0) return launch_vec<TA, TW, 8, 256, STATS>(a, njobs, s);
        return launch_vec<TA, TW, 8, 1024, STATS>(a, njobs, s);
    }

    // chunked rows with more than 8 segments, or wider than one CTA's
    // registers hold: spread each row over the CTAs of a cluster
    if (chunked) {
        const int64_t need = (max_chunks + cl::kMaxChunksPerCta - 1) / cl::kMaxChunksPerCta;
        if (need <= cl::kMaxCluster) {
            int C = 1;
            while (C < need) C <<= 1;
            return launch_cluster<TA, TW, STATS>(ts, njobs, rows, n_seg, eps, partial, C, s);
        }
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

qkn_status check_seg(int n_seg) {
    if (n_seg < 1 || n_seg > QKN_MAX_SEG)
        return fail(QKN_ERR_SHAPE, "n_seg=%d outside [1, %d]", n_seg, QKN_MAX_SEG);
    return QKN_OK;
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

// ---------------------------------------------------------------------------
// Apply step of tensor-parallel QK-Norm (SwiftQK, abstract): a shard holding
// d of the row's d_full elements normalises its slice once the n_part scalar
// partial sums of the row (one per shard or segment) have been gathered:
//   S = ((p_0 + p_1) + ...) + p_{n_part-1},   y_i = (x_i * rsqrt(S / d_full + eps)) * w_i
// One warp per row; 16-byte accesses when the row layout allows.
namespace qkn {
namespace {

template <typename TA, typename TW, bool VEC>
__global__ void __launch_bounds__(256) apply_partials_kernel(const uint8_t *__restrict__ x, uint8_t *__restrict__ y,
                                                             const TW *__restrict__ w, const float *__restrict__ part,
                                                             int64_t rows, int d, int64_t ld_bytes,
                                                             int64_t ldo_bytes, int n_part, int64_t p_row,
                                                             int64_t p_part, float d_full, float eps) {
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;  // whole warp leaves together
    float S = 0.f;
    for (int j = 0; j < n_part; ++j) S += __ldg(part + row * p_row + j * p_part);
    const float inv = rsqrtf(S / d_full + eps);
    const uint8_t *xr = x + row * ld_bytes;
    uint8_t *yr = y + row * ldo_bytes;
    if constexpr (VEC) {
        constexpr int E = Chunk<TA>::E;
        const int nchunks = d / E;
        for (int c0 = 0; c0 < nchunks; c0 += 32 * 4) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = c0 + u * 32 + lane;
                v[u] = c < nchunks ? ld_stream(xr + (int64_t)c * 16) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c < nchunks) {
                    float f[E], wf[E];
                    Chunk<TA>::unpack(v[u], f);
                    load_weights_batched<TW, E>(w + (int64_t)c * E, wf);
#pragma unroll
                    for (int e = 0; e < E; ++e) f[e] = (f[e] * inv) * wf[e];
                    st_stream_batched(yr + (int64_t)c * 16, Chunk<TA>::pack(f));
                }
            }
        }
    } else {
        const TA *xe = reinterpret_cast<const TA *>(xr);
        TA *ye = reinterpret_cast<TA *>(yr);
        for (int i = lane; i < d; i += 32) ye[i] = from_f32<TA>((to_f32<TA>(xe[i]) * inv) * to_f32<TW>(w[i]));
    }
}

template <typename TA, typename TW>
qkn_status launch_apply(const void *x, const void *w, void *y, int64_t rows, int64_t d, int64_t ld, int64_t ldo,
                        const float *part, int n_part, int64_t p_row, int64_t p_part, int64_t d_full, float eps,
                        cudaStream_t s) {
    constexpr int E = Chunk<TA>::E;
    const size_t es = sizeof(TA);
    const uintptr_t walign = (E * sizeof(TW)) < 16 ? E * sizeof(TW) : 16;
    const bool vec = aligned(x, 16) && aligned(y, 16) && (ld * es) % 16 == 0 && (ldo * es) % 16 == 0 &&
                     d % E == 0 && aligned(w, walign);
    const int64_t blocks = (rows + 7) / 8;
    if (blocks > 0x7fffffffLL) return fail(QKN_ERR_SHAPE, "rmsnorm_apply_partials: too many rows");
    const uint8_t *xb = static_cast<const uint8_t *>(x);
    uint8_t *yb = static_cast<uint8_t *>(y);
    const TW *wt = static_cast<const TW *>(w);
    if (vec)
        apply_partials_kernel<TA, TW, true><<<(unsigned)blocks, 256, 0, s>>>(
            xb, yb, wt, part, rows, (int)d, ld * (int64_t)es, ldo * (int64_t)es, n_part, p_row, p_part, (float)d_full, eps);
    else
        apply_partials_kernel<TA, TW, false><<<(unsigned)blocks, 256, 0, s>>>(
            xb, yb, wt, part, rows, (int)d, ld * (int64_t)es, ldo * (int64_t)es, n_part, p_row, p_part, (float)d_full, eps);
    return check_launch("apply_partials_kernel launch");
}

}  // namespace
}  // namespace qkn

extern "C" QKN_API qkn_status rmsnorm_apply_partials(const void *x, const void *w, void *y, int64_t rows, int64_t d,
                                                     int64_t ld, int64_t ld_out, const float *partial, int n_part,
                                                     int64_t part_row_stride, int64_t part_stride, int64_t d_full,
                                                     qkn_dtype act, qkn_dtype wdt, float eps, void *stream) {
    using namespace qkn;
    if (!valid_dtype(act) || !valid_dtype(wdt))
        return fail(QKN_ERR_DTYPE, "rmsnorm_apply_partials: unknown dtype (act=%d, wdt=%d)", (int)act, (int)wdt);
    if (rows < 0 || d < 1 || d > 0x7fffffffLL || ld < d || ld_out < d || d_full < d || d_full > (1LL << 24))
        return fail(QKN_ERR_SHAPE, "rmsnorm_apply_partials: bad sizes rows=%lld d=%lld d_full=%lld", (long long)rows,
                    (long long)d, (long long)d_full);
    if (n_part < 1 || n_part > 4096 || part_row_stride < 0 || part_stride < 0)
        return fail(QKN_ERR_SHAPE, "rmsnorm_apply_partials: bad partial layout (n_part=%d)", n_part);
    if (!(eps >= 0.f) || isinf(eps)) return fail(QKN_ERR_EPS, "rmsnorm_apply_partials: eps must be finite and >= 0");
    if (rows == 0) return QKN_OK;
    if (x == nullptr || w == nullptr || y == nullptr || partial == nullptr)
        return fail(QKN_ERR_NULL, "rmsnorm_apply_partials: x, w, y and partial are required");
    if (!aligned(x, dtype_size(act)) || !aligned(y, dtype_size(act)) || !aligned(w, dtype_size(wdt)) ||
        !aligned(partial, 4))
        return fail(QKN_ERR_ALIGN, "rmsnorm_apply_partials: pointers must be aligned to their element size");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (act == QKN_BF16) {
        if (wdt == QKN_BF16)
            return launch_apply<__nv_bfloat16, __nv_bfloat16>(x, w, y, rows, d, ld, ld_out, partial, n_part,
                                                              part_row_stride, part_stride, d_full, eps, s);
        return launch_apply<__nv_bfloat16, float>(x, w, y, rows, d, ld, ld_out, partial, n_part, part_row_stride,
                                                  part_stride, d_full, eps, s);
    }
    if (wdt == QKN_BF16)
        return launch_apply<float, __nv_bfloat16>(x, w, y, rows, d, ld, ld_out, partial, n_part, part_row_stride,
                                                  part_stride, d_full, eps, s);
    return launch_apply<float, float>(x, w, y, rows, d, ld, ld_out, partial, n_part, part_row_stride, part_stride,
                                      d_full, eps, s);
}

extern "C" QKN_API qkn_status qkn_testing_arm_wait_fault(uint64_t wait_ns) {
    if (wait_ns == 0 || wait_ns > qkn::kWaitTimeoutNs)
        return qkn::fail(QKN_ERR_SHAPE, "qkn_testing_arm_wait_fault: wait_ns must be in (0, 2e9]");
    qkn::t_fault_wait_ns = wait_ns;
    return QKN_OK;
}

// ---------------------------------------------------------------------------
// Host-buffer form of qknorm_fused: the rows stream through a device
// workspace in chunks, on three streams that take chunks in turn, so the
// upload of one chunk, the kernel of another and the download of a third
// overlap (the link is full duplex).  Each stream owns a third of the
// workspace and handles every third chunk in order, which makes buffer reuse
// safe by stream order.  The streams start after the work already on the
// caller's stream and the caller's stream waits for them at the end, so the
// call is asynchronous like the others.
namespace qkn {
namespace {

constexpr int kHostStreams = 3;

struct HostPipe {
    bool ready = false;
    cudaStream_t s[kHostStreams];
    cudaEvent_t start, done[kHostStreams];
};

std::mutex g_pipe_mu;
HostPipe g_pipes[64];

qkn_status host_pipe(HostPipe **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "qknorm_fused_host: cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(QKN_ERR_UNSUPPORTED, "qknorm_fused_host: device %d", dev);
    std::lock_guard<std::mutex> lock(g_pipe_mu);
    HostPipe &p = g_pipes[dev];
    if (!p.ready) {
        for (int i = 0; i < kHostStreams; ++i) {
            if ((e = cudaStreamCreateWithFlags(&p.s[i], cudaStreamNonBlocking)) != cudaSuccess)
                return cuda_fail(e, "qknorm_fused_host: stream");
            if ((e = cudaEventCreateWithFlags(&p.done[i], cudaEventDisableTiming)) != cudaSuccess)
                return cuda_fail(e, "qknorm_fused_host: event");
        }
        if ((e = cudaEventCreateWithFlags(&p.start, cudaEventDisableTiming)) != cudaSuccess)
            return cuda_fail(e, "qknorm_fused_host: event");
        p.ready = true;
    }
    *out = &p;
    return QKN_OK;
}

}  // namespace
}  // namespace qkn

extern "C" QKN_API qkn_status qknorm_fused_host(const void *q, const void *k, const void *wq, const void *wk,
                                                void *q_out, void *k_out, int64_t T, int64_t dq, int64_t dk,
                                                qkn_dtype act, qkn_dtype wdt, float eps, int n_seg,
                                                void *workspace, size_t workspace_bytes, void *stream) {
    using namespace qkn;
    if (!valid_dtype(act) || !valid_dtype(wdt))
        return fail(QKN_ERR_DTYPE, "qknorm_fused_host: unknown dtype (act=%d, wdt=%d)", (int)act, (int)wdt);
    const bool has_k = dk > 0;
    if (T < 0 || dq < 1 || dk < 0 || dq > 0x7fffffffLL || dk > 0x7fffffffLL)
        return fail(QKN_ERR_SHAPE, "qknorm_fused_host: bad sizes T=%lld dq=%lld dk=%lld", (long long)T,
                    (long long)dq, (long long)dk);
    if (qkn_status st = check_seg(n_seg)) return st;
    if (dq % n_seg != 0 || dk % n_seg != 0)
        return fail(QKN_ERR_SHAPE, "qknorm_fused_host: dq / dk not multiples of n_seg=%d", n_seg);
    if (!(eps >= 0.f) || isinf(eps)) return fail(QKN_ERR_EPS, "qknorm_fused_host: eps must be finite and >= 0");
    if (T == 0) return QKN_OK;
    if (q == nullptr || wq == nullptr || q_out == nullptr || workspace == nullptr ||
        (has_k && (k == nullptr || wk == nullptr || k_out == nullptr)))
        return fail(QKN_ERR_NULL, "qknorm_fused_host: a required pointer is NULL");
    const int64_t es = (int64_t)dtype_size(act);
    const int64_t row_bytes = (dq + dk) * es;
    // every chunk buffer starts 256-byte aligned: q rows, then k rows
    const int64_t per_stream = (int64_t)(workspace_bytes / kHostStreams) / 256 * 256;
    int64_t chunk = per_stream / row_bytes;
    while (chunk > 0 && ((chunk * dq * es + 255) / 256 * 256 + chunk * dk * es) > per_stream) --chunk;
    if (chunk < 1)
        return fail(QKN_ERR_SHAPE, "qknorm_fused_host: workspace of %zu bytes is too small for 3 x one row (%lld B)",
                    workspace_bytes, (long long)row_bytes);
    if (!aligned(workspace, 256)) return fail(QKN_ERR_ALIGN, "qknorm_fused_host: workspace must be 256-byte aligned");
    HostPipe *p = nullptr;
    if (qkn_status st = host_pipe(&p)) return st;
    cudaStream_t caller = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaEventRecord(p->start, caller);
    for (int i = 0; i < kHostStreams && e == cudaSuccess; ++i) e = cudaStreamWaitEvent(p->s[i], p->start, 0);
    if (e != cudaSuccess) return cuda_fail(e, "qknorm_fused_host: ordering after the caller's stream");
    const uint8_t *qh = static_cast<const uint8_t *>(q), *kh = static_cast<const uint8_t *>(k);
    uint8_t *qo = static_cast<uint8_t *>(q_out), *ko = static_cast<uint8_t *>(k_out);
    const int64_t q_off = 0, k_off = (chunk * dq * es + 255) / 256 * 256;
    int c = 0;
    for (int64_t r0 = 0; r0 < T; r0 += chunk, ++c) {
        const int64_t n = (T - r0) < chunk ? (T - r0) : chunk;
        const int i = c % kHostStreams;
        cudaStream_t s = p->s[i];
        uint8_t *buf = static_cast<uint8_t *>(workspace) + (int64_t)i * per_stream;
        uint8_t *qd = buf + q_off, *kd = buf + k_off;
        e = cudaMemcpyAsync(qd, qh + r0 * dq * es, (size_t)(n * dq * es), cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess && has_k)
            e = cudaMemcpyAsync(kd, kh + r0 * dk * es, (size_t)(n * dk * es), cudaMemcpyHostToDevice, s);
        if (e != cudaSuccess) return cuda_fail(e, "qknorm_fused_host: upload");
        if (qkn_status st = qknorm_fused(qd, has_k ? kd : nullptr, wq, has_k ? wk : nullptr, nullptr, nullptr, n, dq,
                                         dk, dq, dk, dq, dk, act, wdt, eps, n_seg, s))
            return st;
        e = cudaMemcpyAsync(qo + r0 * dq * es, qd, (size_t)(n * dq * es), cudaMemcpyDeviceToHost, s);
        if (e == cudaSuccess && has_k)
            e = cudaMemcpyAsync(ko + r0 * dk * es, kd, (size_t)(n * dk * es), cudaMemcpyDeviceToHost, s);
        if (e != cudaSuccess) return cuda_fail(e, "qknorm_fused_host: download");
    }
    for (int i = 0; i < kHostStreams && e == cudaSuccess; ++i) {
        e = cudaEventRecord(p->done[i], p->s[i]);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(caller, p->done[i], 0);
    }
    if (e != cudaSuccess) return cuda_fail(e, "qknorm_fused_host: ordering before the caller's stream");
    return QKN_OK;
}
