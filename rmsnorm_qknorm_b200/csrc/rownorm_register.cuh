// Register-resident row kernels: the vectorised kernel (a row in the registers
// of a group of threads) and the element-wise kernel for any alignment.
//
// Included by qknorm.cu only: the kernels are instantiated by its dispatch
// and share its device error word g_norm_error (one translation unit).
#pragma once

#include "qkn_common.cuh"
#include "qkn_sync.cuh"

namespace qkn {

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

// Per-segment sums of squares of a thread's chunks v[i] (chunk i * tpr + t
// of its row): each chunk's sum s (a fused multiply-add chain over its
// elements from zero) is added into acc[(i * tpr + t) / seg_chunks], each
// accumulator taking its chunks in increasing i.  When a segment is q whole
// chunk slots (seg_chunks = q * tpr), slot i lies in segment i / q for every
// thread, so q = 1, 2, 4 and q >= CPT (then the row is one segment: its
// chunks fill at most tpr * CPT slots) add each sum straight into its
// accumulator; other widths compute the segment index per chunk and add
// the sum to every accumulator, zero to all but the chunk's own.  Adding zero
// leaves a non-negative sum's bits unchanged, so both forms give the same
// bits.  SLOTS = false compiles the per-chunk form alone: the normalising
// kernels keep it (measured on B200: the streaming kernel ran 4-17 % slower
// with both forms compiled in, while the statistics alone, bound by issue
// slots, ran 17-24 % faster with the slot form).
template <typename TA, int CPT, bool SLOTS>
__device__ __forceinline__ void segment_sums(const uint4 (&v)[CPT], int t, int tpr, const RowJob &J,
                                             float (&acc)[kFastMaxSeg]) {
    static_assert(CPT == kFastMaxSeg, "slot i's segment is i / q < CPT");
    constexpr int E = Chunk<TA>::E;
#pragma unroll
    for (int j = 0; j < kFastMaxSeg; ++j) acc[j] = 0.f;
    const int q = (J.seg_chunks & (tpr - 1)) == 0 ? J.seg_chunks >> J.tpr_log2 : 0;
    if (SLOTS && (q == 1 || q == 2 || q == 4 || q >= CPT)) {
        float sq[CPT];
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            float f[E];
            Chunk<TA>::unpack(v[i], f);
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) s = fmaf(f[e], f[e], s);
            sq[i] = s;
        }
        if (q == 1) {
#pragma unroll
            for (int i = 0; i < CPT; ++i) acc[i] += sq[i];
        } else if (q == 2) {
#pragma unroll
            for (int j = 0; j < CPT / 2; ++j) acc[j] = (acc[j] + sq[2 * j]) + sq[2 * j + 1];
        } else if (q == 4) {
#pragma unroll
            for (int j = 0; j < CPT / 4; ++j)
                acc[j] = (((acc[j] + sq[4 * j]) + sq[4 * j + 1]) + sq[4 * j + 2]) + sq[4 * j + 3];
        } else {
#pragma unroll
            for (int i = 0; i < CPT; ++i) acc[0] += sq[i];
        }
        return;
    }
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
}

// Reduction of the eight segment slots acc[] over the tpr >= 8 lanes of a
// row (lane t of the row, XOR partners within the warp), with the additions
// of the butterfly that reduces each slot over XOR offsets tpr/2, tpr/4,
// ..., 1, done by recursive halving: at the first three offsets each lane
// keeps half of its slots (the upper half when its offset bit is set) and
// adds the partner's copy of them; at the remaining offsets it adds the
// partner's single value.  Each slot is summed in the butterfly's tree (lane
// and partner form a + b and b + a, which are equal), with 4 + 2 + 1 + 1...
// shuffles instead of 8 per offset.  Returns the total of slot `seg`, the
// one this lane ends with: seg = (bit b-1 of t, bit b-2, bit b-3), b = log2 tpr.
__device__ __forceinline__ float halve_segments(const float (&acc)[kFastMaxSeg], int t, int tpr, int &seg) {
    const bool u4 = t & (tpr >> 1), u2 = t & (tpr >> 2), u1 = t & (tpr >> 3);
    float h4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        h4[i] = (u4 ? acc[i + 4] : acc[i]) + __shfl_xor_sync(0xffffffffu, u4 ? acc[i] : acc[i + 4], tpr >> 1);
    float h2[2];
#pragma unroll
    for (int i = 0; i < 2; ++i)
        h2[i] = (u2 ? h4[i + 2] : h4[i]) + __shfl_xor_sync(0xffffffffu, u2 ? h4[i] : h4[i + 2], tpr >> 2);
    float h1 = (u1 ? h2[1] : h2[0]) + __shfl_xor_sync(0xffffffffu, u1 ? h2[0] : h2[1], tpr >> 3);
    for (int off = tpr >> 4; off > 0; off >>= 1) h1 += __shfl_xor_sync(0xffffffffu, h1, off);
    seg = (u4 ? 4 : 0) | (u2 ? 2 : 0) | (u1 ? 1 : 0);
    return h1;
}

// The lowest lane of a row (whose lanes start at rbase) that holds segment j
// after halve_segments.
__device__ __forceinline__ int segment_lane(int rbase, int tpr, int j) {
    return rbase + ((j >> 2) & 1) * (tpr >> 1) + ((j >> 1) & 1) * (tpr >> 2) + (j & 1) * (tpr >> 3);
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
    segment_sums<TA, CPT, STATS>(v, t, tpr, J, acc);

    // 3. reduce each segment over the threads of the row (fixed tree)
    const int n_seg = a.n_seg;
    if (STATS && tpr >= 8 && tpr <= 32) {  // uniform per block: a block serves one job
        // the same tree by recursive halving; each segment's total is written
        // by the lowest lane of the row that holds it
        int seg;
        const float v = halve_segments(acc, t, tpr, seg);
        if (active && (t & ((tpr >> 3) - 1)) == 0 && seg < n_seg) a.partial[row * n_seg + seg] = v;
        return;
    }
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
// Streaming form of the vectorised kernel for narrow rows (at most 32 threads
// per row, CPT = 8): persistent 256-thread blocks walk the row groups
// (rows_per_cta rows of one job) and load the next group's chunks while they
// normalise the current one, so loads stay in flight between groups (the
// one-shot form loads, then computes and stores with nothing in flight).  A
// row's arithmetic -- chunk-to-thread mapping, per-thread order, butterfly
// over the row's lanes -- is the vectorised kernel's, so the results are bit
// for bit the same.  Warp-level only: the row's lanes are within one warp.
namespace stream {

constexpr int CPT = 8;
constexpr int BLOCK = 256;
// Many-segment statistic (9 to QKN_MAX_SEG segments): per warp, the chunk
// sums of its rows (32 x CPT slots, one padding float after every 32 so that
// lanes summing neighbouring segments read distinct banks) and the segment
// sums (at most 32 x CPT of them: a row of n_seg segments holds at least
// n_seg chunks).
constexpr int kChunkSlots = 32 * CPT + 32 * CPT / 32;
constexpr int kScratchPerWarp = kChunkSlots + 32 * CPT;

__device__ __forceinline__ int padded(int i) { return i + (i >> 5); }

template <typename TA>
__device__ __forceinline__ void load_group(const RowArgs &a, int64_t g, int64_t n0, uint4 (&v)[CPT]) {
    const int which = g >= n0 ? 1 : 0;
    const RowJob J = pick_job(a, which);
    const int64_t b = g - (which ? n0 : 0);
    const int tpr = 1 << J.tpr_log2;
    const int t = threadIdx.x & (tpr - 1);
    const int64_t row = b * J.rows_per_cta + (threadIdx.x >> J.tpr_log2);
    const bool active = row < J.rows;
    const uint8_t *xr = J.x + (active ? row : 0) * J.ld_bytes;
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = i * tpr + t;
        if (active && c < J.nchunks) v[i] = ld_stream(xr + (int64_t)c * 16);
        else v[i] = make_uint4(0u, 0u, 0u, 0u);
    }
}

// Normalises (or, STATS, writes the segment sums of) the rows of a group
// from the n_seg > 8 segment sums formed in shared memory: every thread
// parks the sum of squares of each of its chunks, lane k of the warp then
// adds the chunks of segment k % n_seg of row k / n_seg in chunk order (and
// k + 32, ...), and the row's statistic combines its segment sums left to
// right.  The order of every sum is fixed by the row width and n_seg alone.
template <typename TA, typename TW, bool STATS>
__device__ __forceinline__ void process_group_many(const RowArgs &a, const RowJob &J, int64_t b,
                                                   const uint4 (&v)[CPT], float *scratch) {
    constexpr int E = Chunk<TA>::E;
    const int lane = threadIdx.x & 31;
    const int tpr = 1 << J.tpr_log2;
    const int t = threadIdx.x & (tpr - 1);
    const int rloc = lane >> J.tpr_log2;           // row within the warp
    const int rpw = 32 >> J.tpr_log2;              // rows per warp
    const int cap = tpr * CPT;                     // chunk slots per row
    const int64_t row0 = b * J.rows_per_cta + (int64_t)(threadIdx.x >> 5) * rpw;  // the warp's first row
    const int64_t row = row0 + rloc;
    const bool active = row < J.rows;
    const int nchunks = J.nchunks, n_seg = a.n_seg, sc = J.seg_chunks;
    float *cs = scratch;                           // chunk sums, padded
    float *ss = scratch + kChunkSlots;             // segment sums [rpw][n_seg]
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = i * tpr + t;
        float f[E];
        Chunk<TA>::unpack(v[i], f);
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) s = fmaf(f[e], f[e], s);
        if (c < nchunks) cs[padded(rloc * cap + c)] = s;
    }
    __syncwarp();
    const int tasks = rpw * n_seg;
    for (int k = lane; k < tasks; k += 32) {
        const int r = k / n_seg, j = k - r * n_seg;
        const int base = r * cap + j * sc;
        float s = 0.f;
        for (int q = 0; q < sc; ++q) s += cs[padded(base + q)];
        ss[k] = s;
    }
    __syncwarp();
    if constexpr (STATS) {
        for (int k = lane; k < tasks; k += 32) {
            const int r = k / n_seg;
            if (row0 + r < J.rows) a.partial[(row0 + r) * n_seg + (k - r * n_seg)] = ss[k];
        }
    } else {
        float S = 0.f;
        if (t == 0)
            for (int j = 0; j < n_seg; ++j) S += ss[rloc * n_seg + j];
        S = __shfl_sync(0xffffffffu, S, rloc << J.tpr_log2);
        const float inv = rsqrtf(S / (float)J.d + a.eps);
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
    __syncwarp();  // the next group rewrites the scratch
}

template <typename TA, typename TW, bool STATS>
__device__ __forceinline__ void process_group(const RowArgs &a, int64_t g, int64_t n0, const uint4 (&v)[CPT]) {
    constexpr int E = Chunk<TA>::E;
    const int which = g >= n0 ? 1 : 0;
    const RowJob J = pick_job(a, which);
    const int64_t b = g - (which ? n0 : 0);
    const int tpr = 1 << J.tpr_log2;
    const int t = threadIdx.x & (tpr - 1);
    const int64_t row = b * J.rows_per_cta + (threadIdx.x >> J.tpr_log2);
    const bool active = row < J.rows;
    const int nchunks = J.nchunks;

    float acc[kFastMaxSeg];
    segment_sums<TA, CPT, false>(v, t, tpr, J, acc);
    const int n_seg = a.n_seg;
    // each segment reduced over the row's lanes; with 8 or more lanes by
    // recursive halving (the butterfly's additions, a quarter of the
    // shuffles), the segment totals then gathered left to right
    float S = 0.f;
    if (!STATS && tpr >= 8) {
        int seg;
        const float h = halve_segments(acc, t, tpr, seg);
        const int rbase = (threadIdx.x & 31) & ~(tpr - 1);
#pragma unroll
        for (int j = 0; j < kFastMaxSeg; ++j) {
            const float sj = __shfl_sync(0xffffffffu, h, segment_lane(rbase, tpr, j));
            if (j < n_seg) S += sj;
        }
    } else {
#pragma unroll
        for (int j = 0; j < kFastMaxSeg; ++j) {
            if (j < n_seg) {
                for (int off = tpr >> 1; off > 0; off >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
            }
        }
#pragma unroll
        for (int j = 0; j < kFastMaxSeg; ++j)
            if (j < n_seg) S += acc[j];
    }
    if constexpr (STATS) {
        if (active && t == 0) {
            float *p = a.partial + row * n_seg;
#pragma unroll
            for (int j = 0; j < kFastMaxSeg; ++j)
                if (j < n_seg) p[j] = acc[j];
        }
    } else {
        const float inv = rsqrtf(S / (float)J.d + a.eps);
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

}  // namespace stream

// MANY: n_seg of 9 to QKN_MAX_SEG (rows of at most 32 x CPT chunks).
template <typename TA, typename TW, bool STATS, bool MANY>
__global__ void __launch_bounds__(stream::BLOCK, 2) rownorm_vec_stream_kernel(const RowArgs a) {
    // Launched as the programmatic dependent of the previous launch on the
    // stream: let the next launch's blocks take SM slots as this grid's
    // blocks exit, and touch global memory only once the previous grid has
    // completed and its writes are visible.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t n0 = a.job[0].nblocks, total = n0 + a.job[1].nblocks;
    int64_t g = blockIdx.x;
    if (g >= total) return;  // the whole block: no block-level synchronisation below
    __shared__ float scratch[MANY ? stream::BLOCK / 32 * stream::kScratchPerWarp : 1];
    uint4 cur[stream::CPT], nxt[stream::CPT];
    stream::load_group<TA>(a, g, n0, cur);
    for (; g < total; g += gridDim.x) {
        const int64_t gn = g + gridDim.x;
        if (gn < total) stream::load_group<TA>(a, gn, n0, nxt);
        if constexpr (MANY) {
            const int which = g >= n0 ? 1 : 0;
            stream::process_group_many<TA, TW, STATS>(a, pick_job(a, which), g - (which ? n0 : 0), cur,
                                                      scratch + (threadIdx.x >> 5) * stream::kScratchPerWarp);
        } else {
            stream::process_group<TA, TW, STATS>(a, g, n0, cur);
        }
#pragma unroll
        for (int i = 0; i < stream::CPT; ++i) cur[i] = nxt[i];
    }
}

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

}  // namespace qkn
