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
#include <math.h>

#include "qkn_common.cuh"

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

// ---------------------------------------------------------------- host side

namespace {

struct Tensor2 {
    const void *x;
    void *y;
    const void *w;
    int64_t d, ld, ldo;
};

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

template <typename TA, typename TW, bool STATS>
qkn_status dispatch(const Tensor2 *ts, int njobs, int64_t rows, int n_seg, float eps,
                    float *partial, cudaStream_t s) {
    constexpr int E = Chunk<TA>::E;
    RowArgs a{};
    a.n_seg = n_seg;
    a.eps = eps;
    a.partial = partial;

    // vector path eligibility: 16-byte rows, whole chunks per segment
    bool vec = n_seg <= kFastMaxSeg;
    int64_t max_chunks = 0;
    for (int i = 0; i < njobs && vec; ++i) {
        const Tensor2 &t = ts[i];
        const size_t es = sizeof(TA);
        const uintptr_t walign = (E * sizeof(TW)) < 16 ? E * sizeof(TW) : 16;
        vec = aligned(t.x, 16) && (t.ld * es) % 16 == 0 && t.d % E == 0 &&
              (t.d / n_seg) % E == 0 &&
              (STATS || (aligned(t.w, walign) && aligned(t.y, 16) && (t.ldo * es) % 16 == 0));
        if (t.d / E > max_chunks) max_chunks = t.d / E;
    }
    if (max_chunks >= (1 << 22)) vec = false;

    int cfg = -1;
    if (vec) {
        for (int c = 0; c < kNumVecCfgs; ++c) {
            if (max_chunks <= (int64_t)kVecCfgs[c].cpt * kVecCfgs[c].block) { cfg = c; break; }
        }
        if (cfg < 0) vec = false;
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
