// Staged row kernel: rows fed to shared memory by bulk copies, persistent.
//
// Included by qknorm.cu only: the kernels are instantiated by its dispatch
// and share its device error word g_norm_error (one translation unit).
#pragma once

#include "qkn_common.cuh"
#include "qkn_sync.cuh"
#include "rownorm_register.cuh"

namespace qkn {

// ---------------------------------------------------------------------------
// Staged kernel (rows up to ~40 KiB): persistent, one block per SM.  Launches
// whose widest row is at most 4 KiB take the register kernels instead
// (qknorm.cu's dispatch).
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
// 4j .. 4j+3 hold segment j; the segments are combined left to right.  With
// more than eight segments (up to 64) each segment has its own slot, lane j
// adds slot j's 32 lane sums in lane order, and the segments are again
// combined left to right.
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
    int reg_tpr_log2;      // >= 0: rows of at most 256 chunks and 8 segments, in the register
                           // kernels' arithmetic with 2^reg_tpr_log2 lanes per row; -1 otherwise
    float inv_seg_chunks;  // 1 / seg_chunks (the register kernels' segment index)
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
    int scratch_floats;  // per warp: segment slots x their lane stride
};

// Segment slots of a warp's scratch: 8 x 32 floats for up to 8 segments; for
// more, one slot per segment padded to 33 floats, so that lane j reading
// slot j's 32 entries in turn touches a different bank from every other lane.
constexpr int kManySegStride = 33;
inline int scratch_floats(int n_seg) {
    return n_seg <= kFastMaxSeg ? kFastMaxSeg * 32 : n_seg * kManySegStride;
}

// Shared memory: [ring][fp32 weights][full bars][W x scratch_floats scratch]
inline int smem_bytes(int warps, int stages, int stage_bytes, int w_bytes, int scratch_per_warp) {
    return stages * stage_bytes + w_bytes + stages * 8 + warps * scratch_per_warp * 4;
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
    J.reg_tpr_log2 = which ? j1.reg_tpr_log2 : j0.reg_tpr_log2;
    J.inv_seg_chunks = which ? j1.inv_seg_chunks : j0.inv_seg_chunks;
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
template <int STRIDE = 32>
__device__ __forceinline__ void accumulate(float2 sq, int c, float2 &cur, int &cur_seg, int &next_bound,
                                           int seg_chunks, float *part, int lane) {
    while (c >= next_bound) {
        part[cur_seg * STRIDE + lane] = cur.x + cur.y;
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

// Up to 8 segments: reduces the warp's parked segment sums (scratch [8][32])
// by recursive halving over the lanes (lanes 4j .. 4j+3 end with segment j),
// adds the segments left to right and returns S; STATS stores the segment
// sums.
template <bool STATS>
__device__ __forceinline__ float finish_statistic(const Args &a, float *part, int64_t row, int lane) {
    const int n_seg = a.n_seg;
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

// More than 8 segments (up to 64): the lane sums were parked one slot per
// segment (stride 33); lane j adds slot j's 32 entries in lane order (and
// slot j + 32's), then the segments are added left to right.  Returns S;
// STATS stores the segment sums.
template <bool STATS>
__device__ __forceinline__ float finish_many(const Args &a, const float *part, int64_t row, int lane) {
    const int n_seg = a.n_seg;
    __syncwarp();
    float r0 = 0.f, r1 = 0.f;
    if (lane < n_seg) {
        const float *p = part + lane * kManySegStride;
#pragma unroll 8
        for (int i = 0; i < 32; ++i) r0 += p[i];
    }
    if (lane + 32 < n_seg) {
        const float *p = part + (lane + 32) * kManySegStride;
#pragma unroll 8
        for (int i = 0; i < 32; ++i) r1 += p[i];
    }
    if constexpr (STATS) {
        if (lane < n_seg) a.partial[row * n_seg + lane] = r0;
        if (lane + 32 < n_seg) a.partial[row * n_seg + lane + 32] = r1;
    }
    float S = 0.f;
    const int lo = n_seg < 32 ? n_seg : 32;
    for (int j = 0; j < lo; ++j) S += __shfl_sync(0xffffffffu, r0, j);
    for (int j = 32; j < n_seg; ++j) S += __shfl_sync(0xffffffffu, r1, j - 32);
    __syncwarp();  // the scratch is rewritten by the next row
    return S;
}

// Statistic of one row held in shared memory, by one warp (any width): lane
// l adds its chunks l, l + 32, ... in order into a running pair sum that is
// parked in the warp's scratch `part` (slot [segment][lane]) whenever a
// segment ends; the slots are then reduced (finish_statistic or
// finish_many) and the segments added left to right.  Returns S.
template <typename TA, bool STATS, bool MANY = false>
__device__ __forceinline__ float row_statistic(const Args &a, const Job &J, const uint8_t *srow, int64_t row,
                                               int lane, float *part) {
    constexpr int STRIDE = MANY ? kManySegStride : 32;
    const int nchunks = J.nchunks;
    const int sc = J.seg_chunks;
    if constexpr (MANY) {
        // with 32 or more chunks per segment every lane has a chunk in every
        // segment, so every slot is written below; otherwise clear them first
        if (sc < 32)
            for (int j = 0; j < a.n_seg; ++j) part[j * STRIDE + lane] = 0.f;
    } else {
#pragma unroll
        for (int j = 0; j < kFastMaxSeg; ++j) part[j * 32 + lane] = 0.f;
    }
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
                    accumulate<STRIDE>(sq[u], c0 + u * 32 + lane, cur, cur_seg, next_bound, sc, part, lane);
            }
        }
    }
    for (; c0 < nchunks; c0 += 32) {
        const int c = c0 + lane;
        if (c < nchunks)
            accumulate<STRIDE>(chunk_sumsq<TA>(*reinterpret_cast<const uint4 *>(srow + c * 16)), c, cur, cur_seg,
                               next_bound, sc, part, lane);
    }
    part[cur_seg * STRIDE + lane] = cur.x + cur.y;
    if constexpr (MANY) return finish_many<STATS>(a, part, row, lane);
    else return finish_statistic<STATS>(a, part, row, lane);
}

// Kernel flavours, chosen per launch from the rows' shapes so that each
// keeps only the register budget of the paths it can take.
constexpr int kFlavorGeneric = 0;  // any row, up to 8 segments
constexpr int kFlavorManySeg = 1;  // 9 .. 64 segments
constexpr int kFlavorRegRows = 2;  // up to 8 segments; some rows in the register kernels' arithmetic

// One row held in shared memory, processed by one warp.  `part` is the warp's
// [8][32] scratch for lane partials; `wsm` the job's fp32 weights.  FLAVOR
// selects which statistic paths are compiled in (kFlavor*).
template <typename TA, bool STATS, int FLAVOR>
__device__ __forceinline__ void process_row(const Args &a, const Job &J, const uint8_t *srow, const float4 *wsm,
                                            int64_t row, int lane, float *part) {
    const int nchunks = J.nchunks;
    const float S = row_statistic<TA, STATS, FLAVOR == kFlavorManySeg>(a, J, srow, row, lane, part);

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

// Rows of at most 256 chunks (4 KiB) with up to 8 segments, which the
// register kernels normalise when they are launched on their own, in those
// kernels' arithmetic: lane l of the warp takes row l / tpr of a group of
// 32 / tpr rows of the stage and, as thread t = l % tpr of that row, its
// chunks t, t + tpr, ... (at most CPT of them).  The chunk sums and their
// segments (segment_sums), the reduction of each segment over the row's
// lanes, the left-to-right combine and (x * inv) * w with one rounding are
// those of stream::process_group, so such a row comes out bit for bit as it
// does without a wider job beside it.  The register kernels reduce each
// segment by a butterfly over the row's lanes; with 8 or more lanes per row
// the same additions are done here by recursive halving (halve_segments),
// with far fewer shuffles.
template <typename TA, bool STATS>
__device__ __forceinline__ void process_rows_reg(const Args &a, const Job &J, const uint8_t *sbase,
                                                 const float4 *wsm, int64_t row0, int nrows, int lane) {
    constexpr int CPT = stream::CPT;
    const int tpr_log2 = J.reg_tpr_log2, tpr = 1 << tpr_log2;
    const int rloc = lane >> tpr_log2, t = lane & (tpr - 1);
    const int rpw = 32 >> tpr_log2;  // rows per warp pass
    const int nchunks = J.nchunks, n_seg = a.n_seg;
    RowJob R{};  // the fields segment_sums reads
    R.seg_chunks = J.seg_chunks;
    R.tpr_log2 = tpr_log2;
    R.inv_seg_chunks = J.inv_seg_chunks;
    for (int r0 = 0; r0 < nrows; r0 += rpw) {
        const int r = r0 + rloc;
        const bool active = r < nrows;
        const uint8_t *srow = sbase + (size_t)(active ? r : 0) * J.row_bytes;
        uint4 v[CPT];
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int c = i * tpr + t;
            if (active && c < nchunks) v[i] = *reinterpret_cast<const uint4 *>(srow + c * 16);
            else v[i] = make_uint4(0u, 0u, 0u, 0u);
        }
        float acc[kFastMaxSeg];
        segment_sums<TA, CPT, true>(v, t, tpr, R, acc);
        const int64_t row = row0 + r;
        float S = 0.f;
        if (tpr >= 8) {
            int seg;
            const float h1 = halve_segments(acc, t, tpr, seg);
            if constexpr (STATS) {
                if (active && (t & ((tpr >> 3) - 1)) == 0 && seg < n_seg) a.partial[row * n_seg + seg] = h1;
            } else {
                const int rbase = lane & ~(tpr - 1);
#pragma unroll
                for (int j = 0; j < kFastMaxSeg; ++j) {
                    const float sj = __shfl_sync(0xffffffffu, h1, segment_lane(rbase, tpr, j));
                    if (j < n_seg) S += sj;
                }
            }
        } else {
#pragma unroll
            for (int j = 0; j < kFastMaxSeg; ++j) {
                if (j < n_seg) {
                    for (int off = tpr >> 1; off > 0; off >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
                }
            }
            if constexpr (STATS) {
                if (active && t == 0) {
#pragma unroll
                    for (int j = 0; j < kFastMaxSeg; ++j)
                        if (j < n_seg) a.partial[row * n_seg + j] = acc[j];
                }
            } else {
#pragma unroll
                for (int j = 0; j < kFastMaxSeg; ++j)
                    if (j < n_seg) S += acc[j];
            }
        }
        if constexpr (!STATS) {
            const float inv = rsqrtf(S / (float)J.d + a.eps);
            const float2 inv2 = make_float2(inv, inv);
            uint8_t *yr = J.y + (active ? row : row0) * J.ldo_bytes;
#pragma unroll
            for (int i = 0; i < CPT; ++i) {
                const int c = i * tpr + t;
                if (active && c < nchunks) apply_chunk<TA>(v[i], c, inv2, wsm, nchunks, yr);
            }
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

template <typename TA, typename TW, bool STATS, int FLAVOR>
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
    float *part = scratch + warp * a.scratch_floats;
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
        if (FLAVOR == kFlavorRegRows && J.reg_tpr_log2 >= 0) {
            process_rows_reg<TA, STATS>(a, J, sbase, wsm, row0, nrows, lane);
        } else {
            for (int r = 0; r < nrows; ++r)
                process_row<TA, STATS, FLAVOR>(a, J, sbase + r * J.row_bytes, wsm, row0 + r, lane, part);
        }
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

// Statistics alone (rmsnorm_partial_stats on rows the staged kernel would
// take).  Without an apply pass a row is read once, so
// the staging ring buys nothing: one warp per row reads it straight from
// global memory through the same row_statistic (the same summation order,
// hence bit for bit the partials qknorm_fused forms), with four 8-warp blocks
// per SM for the loads in flight.  Measured on B200 against the staged form:
// 65536 x 4096 bf16 125 -> 105 us, 16384 x 5120 44.5 -> 41.8 us.
// With more than 8 segments (MANY) the warps' slots live in dynamic shared
// memory (a.scratch_floats per warp) and the many-segment statistic runs.
template <typename TA, bool MANY>
__global__ void __launch_bounds__(256, 4) rowstats_direct_kernel(const Args a) {
    __shared__ float scratch[8][kFastMaxSeg * 32];
    extern __shared__ float many_scratch[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *part = MANY ? many_scratch + warp * a.scratch_floats : scratch[warp];
    const Job J = a.job[0];
    const int64_t nw = (int64_t)gridDim.x * 8;
    for (int64_t row = (int64_t)blockIdx.x * 8 + warp; row < J.rows; row += nw)
        row_statistic<TA, true, MANY>(a, J, J.x + row * J.ld_bytes, row, lane, part);
}

}  // namespace staged

}  // namespace qkn
