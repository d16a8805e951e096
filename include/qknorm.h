/*
 * qknorm.h -- C ABI of libqknorm.so: layerwise QK-Norm with segment-wise
 * scalar statistics, and the FlashNorm fold + deferred-normalisation
 * projection, as hand-written CUDA kernels for B200 (sm_100a).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every data pointer is a DEVICE pointer owned by the caller; the library
 *   keeps no pointer after the call returns.
 * - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *   stream).  Work is enqueued asynchronously on it; nothing synchronises.
 * - Arguments are validated on the host before anything is launched.  A
 *   failed validation returns a nonzero qkn_status, launches nothing, and
 *   leaves a message in qkn_last_error() (thread-local).
 * - QKN_ERR_CUDA reports an error returned by the CUDA runtime for this
 *   call's launches (cudaGetLastError right after them); errors raised later
 *   by the device surface at the caller's next synchronisation, as usual.
 * - Rows are independent; an empty problem (zero rows) is valid, launches
 *   nothing and accepts NULL data pointers (an empty tensor may have no
 *   storage).  NaN / Inf inputs propagate to the rows that contain them.
 * - Results are deterministic: the same inputs give bitwise-equal outputs on
 *   every call (fixed reduction orders, no atomics).
 */
#ifndef QKNORM_H
#define QKNORM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QKN_API __attribute__((visibility("default")))
#else
#define QKN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QKN_OK = 0,
    QKN_ERR_NULL = 1,        /* a required pointer is NULL */
    QKN_ERR_SHAPE = 2,       /* negative size, zero width, leading dimension < width,
                                width not a multiple of n_seg, n_seg out of range,
                                or a size rule of the entry point not met */
    QKN_ERR_DTYPE = 3,       /* unknown qkn_dtype or a combination not offered */
    QKN_ERR_EPS = 4,         /* eps negative, NaN or infinite */
    QKN_ERR_ALIGN = 5,       /* an alignment the entry point requires is not met */
    QKN_ERR_CUDA = 6,        /* the CUDA runtime reported an error for this call */
    QKN_ERR_TIMEOUT = 7,     /* a bounded device-side wait gave up */
    QKN_ERR_UNSUPPORTED = 8  /* well-formed request outside what this build implements */
} qkn_status;

typedef enum {
    QKN_F32 = 0,   /* IEEE binary32 */
    QKN_BF16 = 1   /* bfloat16 (1 sign, 8 exponent, 7 fraction bits) */
} qkn_dtype;

/* Largest number of segments (emulated tensor-parallel shards) per row. */
#define QKN_MAX_SEG 64

/*
 * qknorm_fused -- layerwise QK-Norm of the query and key rows (one launch for both
 * where they take compatible kernels, below).
 *
 * Defined by: "SwiftQK: Fast and Communication-Efficient Tensor Parallelism
 * for Query-Key Normalization", abstract -- QK-Norm is an
 * RMSNorm whose factor depends on each token's full q (resp. k) vector; under
 * tensor parallelism every shard contributes a scalar partial sum of squares
 * and only these scalars are combined.  Here the n_seg shards are emulated on
 * one GPU as n_seg contiguous equal segments of each row:
 *   S_j  = sum over segment j of x_i^2                       (fp32)
 *   S    = ((S_0 + S_1) + S_2) + ... + S_{n_seg-1}            (fixed order)
 *   inv  = 1 / sqrt(S / d + eps)
 *   y_i  = (x_i * inv) * w_i, rounded once to the activation dtype.
 *
 * q      [T][dq] activations, row pitch ldq elements (ldq >= dq)
 * k      [T][dk] activations, row pitch ldk; dk == 0 normalises q only (k, wk
 *        and k_out are then ignored)
 * wq, wk [dq], [dk] weights, dtype `wdt` (may differ from `act`)
 * q_out, k_out  outputs [T][d] with pitches ldq_out, ldk_out; pass q_out ==
 *        NULL (resp. k_out == NULL) to normalise in place, in which case the
 *        input pitch is used and the ld*_out argument is ignored
 * act    QKN_F32 or QKN_BF16 (inputs and outputs); statistics are always fp32
 * eps    >= 0 and finite; a zero row with eps == 0 gives NaN (0/0), not an error
 * n_seg  1 .. QKN_MAX_SEG; dq and dk must both be multiples of n_seg
 *
 * Alignment: any element-aligned pointers and pitches are accepted.  When
 * every row start is 16-byte aligned and each segment is a whole number of
 * 16-byte chunks, a vectorised kernel runs: rows of at most 4096 bytes held
 * in registers; wider rows staged through shared memory while they fit the
 * staging ring (about 40 KiB, any n_seg); wider still, spread over the CTAs
 * of a thread-block cluster that exchange only their per-segment partial
 * sums (rows up to 8 x 16384 bf16 / 8 x 8192 fp32 elements).  Otherwise a
 * slower element-wise kernel computes the same result.
 * Each of q and k takes the kernel that its own width, dtype, alignment and
 * n_seg select, never T.  One launch serves both when they select the same
 * kernel, or when one selects the register kernels and the other the staged
 * kernel with n_seg <= 8 (the staged kernel then keeps the register kernels'
 * arithmetic for the narrower rows); otherwise k's launch follows q's on
 * `stream`.  So the bits of a row do not depend on the tensor beside it.
 * The staged and streaming register kernels are launched as programmatic
 * dependents: they touch no global memory before the previous kernel on
 * `stream` finished.
 */
QKN_API qkn_status qknorm_fused(const void *q, const void *k,
                                const void *wq, const void *wk,
                                void *q_out, void *k_out,
                                int64_t T, int64_t dq, int64_t dk,
                                int64_t ldq, int64_t ldk,
                                int64_t ldq_out, int64_t ldk_out,
                                qkn_dtype act, qkn_dtype wdt,
                                float eps, int n_seg, void *stream);

/*
 * qknorm_fused_host -- qknorm_fused on rows held in HOST memory.
 *
 * Same computation as qknorm_fused (SwiftQK, abstract), for q [T][dq] and
 * k [T][dk] in host memory (contiguous rows; pinned memory lets the copies
 * run at full link speed).  The rows stream through `workspace` (device, at
 * least 3 x (dq + dk) x element size bytes, 256-byte aligned) in chunks on
 * three internal streams that take chunks in turn, so the upload of one
 * chunk, the kernel of another and the download of a third overlap.  Results
 * land in q_out / k_out (host, may equal q / k).  wq, wk are DEVICE pointers.
 * The work is ordered after what is already on `stream`, and `stream` waits
 * for it: the call returns before the copies finish, so the host buffers must
 * stay valid (and unread) until `stream` has been synchronised.  dk == 0
 * normalises q only.  The internal streams are created on the first call per
 * device and kept until exit.
 */
QKN_API qkn_status qknorm_fused_host(const void *q, const void *k,
                                     const void *wq, const void *wk,
                                     void *q_out, void *k_out,
                                     int64_t T, int64_t dq, int64_t dk,
                                     qkn_dtype act, qkn_dtype wdt, float eps, int n_seg,
                                     void *workspace, size_t workspace_bytes, void *stream);

/*
 * rmsnorm_partial_stats -- the per-shard scalar statistics on their own.
 *
 * Defined by: SwiftQK, abstract -- the scalar partial sums of squares that
 * the shards exchange instead of the full activation vectors.
 *   partial[r][j] = sum_{i in [j*d/n_seg, (j+1)*d/n_seg)} x[r][i]^2  (fp32)
 *
 * x        [rows][d], pitch ld >= d, dtype `act` (QKN_F32 or QKN_BF16)
 * partial  [rows][n_seg] fp32, contiguous, written completely
 * n_seg    1 .. QKN_MAX_SEG, d % n_seg == 0
 * The summation order inside a segment is fixed for a given row width and
 * n_seg, so repeated calls give bitwise-equal partials.  The rows take the
 * kernel (and summation order) qknorm_fused gives them, so these are bit
 * for bit the partials it combines for the same rows and n_seg, whatever
 * tensor shares its launch, and rmsnorm_apply_partials on them reproduces
 * qknorm_fused exactly (when qknorm_fused's weights and outputs are 16-byte
 * aligned, like x; with unaligned ones it takes the element-wise kernel).
 */
QKN_API qkn_status rmsnorm_partial_stats(const void *x, int64_t rows, int64_t d,
                                         int64_t ld, qkn_dtype act, int n_seg,
                                         float *partial, void *stream);

/*
 * flashnorm_inv_rms -- FlashNorm's row statistic on its own.
 *
 * Defined by: FlashNorm (Graef, arXiv 2024), abstract, item (ii): the scalar
 * 1/rms of each row, which the projection applies to its output:
 *   inv[m] = 1 / sqrt(sum_k x[m][k]^2 / K + eps)   (fp32 sums of the bf16 x)
 * This is the pass flashnorm_proj runs beside the projection when given
 * inv_rms_out; the values are bit for bit the ones it writes there.
 *
 * x    [M][K] bf16, contiguous, 16-byte aligned; K a multiple of 8
 * inv  [M] fp32, written completely
 * eps  >= 0 and finite
 */
QKN_API qkn_status flashnorm_inv_rms(const void *x, float *inv, int64_t M, int64_t K, float eps,
                                     void *stream);

/*
 * rmsnorm_apply_partials -- the apply step of tensor-parallel QK-Norm.
 *
 * Defined by: SwiftQK, abstract -- under tensor parallelism each shard holds
 * a slice of the row and only the shards' scalar sums of squares are
 * exchanged; every shard then normalises its own slice with the combined
 * statistic.  With the n_part partials of each row gathered (for example
 * rmsnorm_partial_stats on every shard plus an all-gather of the scalars):
 *   S      = ((p_0 + p_1) + p_2) + ... + p_{n_part-1}   (fixed order, fp32)
 *   y[r][i] = (x[r][i] * rsqrt(S / d_full + eps)) * w[i]
 *
 * x, y     [rows][d] this shard's slice, pitches ld, ld_out (y may equal x)
 * w        [d] this shard's slice of the weights
 * partial  fp32; the j-th partial of row r is
 *          partial[r * part_row_stride + j * part_stride]
 *          (rmsnorm_partial_stats output: strides n_seg, 1; an all-gathered
 *          [n_part][rows] array: strides 1, rows)
 * n_part   1 .. 4096;  d_full = width of the whole row (the mean's divisor),
 *          d <= d_full <= 2^24
 */
QKN_API qkn_status rmsnorm_apply_partials(const void *x, const void *w, void *y,
                                          int64_t rows, int64_t d, int64_t ld, int64_t ld_out,
                                          const float *partial, int n_part,
                                          int64_t part_row_stride, int64_t part_stride,
                                          int64_t d_full, qkn_dtype act, qkn_dtype wdt,
                                          float eps, void *stream);

/*
 * flashnorm_fold_weights -- fold the RMSNorm weights into the next linear
 * layer (offline).
 *
 * Defined by: FlashNorm (Graef, arXiv 2024), abstract, item (i): the
 * normalisation weights disappear into the following weight matrix,
 *   W'[k][n] = w[k] * W[k][n]   computed in fp32, rounded once to bf16.
 *
 * w         [K], dtype `wdt` (QKN_F32 or QKN_BF16)
 * W         [K][N] bf16, row-major (N contiguous)
 * W_folded  bf16 output, [K][N] row-major when out_k_major == 0, or the
 *           transposed [N][K] (K contiguous) when out_k_major == 1 -- the
 *           layout flashnorm_proj reads
 * W_folded must not overlap W.
 */
QKN_API qkn_status flashnorm_fold_weights(const void *w, const void *W, void *W_folded,
                                          int64_t K, int64_t N, qkn_dtype wdt,
                                          int out_k_major, void *stream);

/*
 * flashnorm_proj -- RMSNorm followed by a linear layer, computed as
 * FlashNorm's deferred normalisation: a bf16 tensor-core GEMM on the raw x
 * with the folded weights, the scalar 1/rms(x) applied in the epilogue.
 *
 * Defined by: FlashNorm, abstract, item (ii): the scalar RMS normalisation is
 * moved to the matmul output, so RMS and matmul can run in parallel.
 *   inv[m]  = 1 / sqrt(sum_k x[m][k]^2 / K + eps)               (fp32)
 *   y[m][n] = inv[m] * sum_k x[m][k] * W'[n][k]   fp32 accumulate, bf16 out
 *
 * x          [M][K] bf16, row-major (K contiguous)
 * W_folded   w_k_major = 1: [N][K] bf16 (K contiguous, out_k_major == 1 of
 *            the fold, the layout the tensor cores read); w_k_major = 0:
 *            [K][N] bf16 (row-major, out_k_major == 0), copied K-major into a
 *            stream-ordered temporary first (an extra pass over W')
 * y          [M][N] bf16, row-major
 * inv_rms    optional [M] fp32 precomputed 1/rms (then used as given)
 * inv_rms_out optional [M] fp32; when inv_rms is NULL and this is given, a
 *            row-statistics pass writes each row's 1/rms here and the
 *            projection reads it (the faster form: the matmul keeps all of
 *            shared-memory bandwidth)
 * With both NULL the projection kernel computes each row's 1/rms itself from
 * the x tiles it streams for the matmul, in parallel with the tensor-core
 * work -- no extra pass and no workspace.
 * Sizes: M, N, K >= 1; K and N multiples of 8.  Pointers 16-byte aligned.
 * y must not overlap x or W_folded.  Nothing is allocated.
 */
QKN_API qkn_status flashnorm_proj(const void *x, const void *W_folded, void *y,
                                  int64_t M, int64_t N, int64_t K, int w_k_major,
                                  float eps, const float *inv_rms, float *inv_rms_out,
                                  void *stream);

/*
 * qkv_proj_qknorm -- RMSNorm, QKV projection and QK-Norm in one GEMM: the
 * normalised q and k are formed in the projection's epilogue and never
 * travel through HBM unnormalised.
 *
 * Defined by: FlashNorm, abstract (fold the input norm's weights into W',
 * apply the scalar 1/rms to the matmul output) and SwiftQK, abstract (the
 * QK-Norm factor depends on a token's full query / key vector; the pieces of
 * that vector held in different places contribute scalar partial sums of
 * squares, combined in a fixed order):
 *   u[m][n]              = r[m] * sum_k x[m][k] W'[n][k]      fp32 accumulate
 *   y[m][0:nq)           = RMSNorm(u[m][0:nq);  wq, eps_qk)
 *   y[m][nq:nq+nk)       = RMSNorm(u[m][nq:nq+nk); wk, eps_qk)
 *   y[m][nq+nk:nq+nk+nv) = u[m][nq+nk:nq+nk+nv)
 * with RMSNorm(v; w, e)_i = (v_i * 1/sqrt(mean(v^2) + e)) * w_i in fp32 and
 * one RNE rounding to bf16.  A row's q (k) statistic is the sum, in tile
 * order, of its per-256-column-tile partial sums, exchanged between the
 * CTAs of one kernel.
 *
 * r[m]: inv_rms given -> used as given; inv_rms NULL and inv_rms_out given
 * -> a statistics pass writes 1/sqrt(mean(x[m]^2) + eps) there first; both
 * NULL -> r = 1 (x used as it is, e.g. already normalised).
 *
 * x [M][K] bf16; W_folded [nq+nk+nv][K] bf16 (K contiguous, from
 * flashnorm_fold_weights with out_k_major = 1); y [M][nq+nk+nv] bf16; wq
 * [nq], wk [nk] of dtype wdt.  K, nq, nk, nv multiples of 8 (nv may be 0);
 * x, W_folded, y, wq, wk, workspace 16-byte aligned.  workspace: device
 * scratch of at least qkv_proj_qknorm_workspace_bytes(M, nq, nk, nv) bytes,
 * or NULL to allocate it stream-ordered inside the call.  The kernel is
 * launched cooperatively (all its CTAs resident at once); QKN_ERR_UNSUPPORTED
 * when nq or nk spans more 256-column tiles than the device has SMs.  A
 * device-side wait that gives up is reported by qkn_check_device.
 */
QKN_API qkn_status qkv_proj_qknorm(const void *x, const void *W_folded, void *y,
                                   int64_t M, int64_t K, int64_t nq, int64_t nk, int64_t nv,
                                   const void *wq, const void *wk, qkn_dtype wdt,
                                   float eps, float eps_qk,
                                   const float *inv_rms, float *inv_rms_out,
                                   void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of device workspace qkv_proj_qknorm needs (0 for invalid sizes). */
QKN_API size_t qkv_proj_qknorm_workspace_bytes(int64_t M, int64_t nq, int64_t nk, int64_t nv);

/*
 * qkv_norm_proj -- QKV projection with QKV-normalisation, pre-attention
 * RMSNorm eliminated.
 *
 * Defined by: FlashNorm, abstract -- by the scale invariance of RMS, an
 * RMSNorm followed by a linear layer followed by another RMSNorm allows the
 * first RMSNorm to be eliminated (models that normalise q, k and v).  With
 * the pre-attention norm's weights folded into W' (flashnorm_fold_weights),
 * its 1/rms(x) cancels in the per-row norms that follow:
 *   u       = x W'^T                         (no row scaling; bf16 out)
 *   y[:, 0:nq)          = RMSNorm(u_q; wq, eps)   with n_seg partials
 *   y[:, nq:nq+nk)      = RMSNorm(u_k; wk, eps)
 *   y[:, nq+nk:nq+nk+nv) = RMSNorm(u_v; wv, eps)  (when nv > 0)
 * Exact up to rounding when the eliminated norm's eps is 0; with eps > 0 the
 * two differ by the relative size of that eps next to the rows' mean square.
 *
 * x [M][K] bf16; W_folded [nq+nk+nv][K] bf16 (K contiguous); y [M][nq+nk+nv]
 * bf16; wq, wk, wv weights of dtype wdt.  K and nq+nk+nv multiples of 8;
 * nq, nk, nv multiples of n_seg; x, W_folded, y 16-byte aligned.  Three
 * launches (projection, q+k norm, v norm) on `stream`; nothing is allocated.
 */
QKN_API qkn_status qkv_norm_proj(const void *x, const void *W_folded, void *y,
                                 int64_t M, int64_t K, int64_t nq, int64_t nk, int64_t nv,
                                 const void *wq, const void *wk, const void *wv,
                                 qkn_dtype wdt, float eps, int n_seg, void *stream);

/*
 * flashnorm_proj_noalloc -- flashnorm_proj for callers that cannot allocate
 * device memory during the call.
 *
 * No counterpart in the pages: FlashNorm describes the computation, not how
 * its scratch is obtained.  This variant exists for callers that must not
 * call cudaMalloc (or any allocator) at call time -- runtimes that plan the
 * whole device memory up front and forbid allocations on the hot path,
 * callers under a framework whose allocator owns the device, real-time loops
 * that cannot absorb an allocator's latency.
 *
 * Same arguments and the same launches as flashnorm_proj with inv_rms ==
 * NULL and an inv_rms_out buffer, so the result is bit-identical to that
 * call: a row-statistics pass writes the 1/rms vector into a fixed 1 MiB
 * array compiled into the library (a file-scope __device__ variable, present
 * on every GPU that loads the library until the process exits), then the
 * projection reads it.  The call allocates nothing.
 *
 * Limits and caveats:
 * - M <= 262144 rows; larger M returns QKN_ERR_SHAPE before any launch.
 * - W_folded must be K-major (w_k_major = 1): a row-major W' would need a
 *   temporary copy, so w_k_major = 0 returns QKN_ERR_UNSUPPORTED.
 * - Every call on a GPU shares the one array: calls that overlap on the GPU
 *   (e.g. on two streams at once) race on it and must be serialised by the
 *   caller.  Each call writes the entries it reads, so the array's leftover
 *   contents from an earlier call never reach the result.
 * - The first call on a device (with that device current) looks up the
 *   array's device address with cudaGetSymbolAddress and caches it with the
 *   current CUDA context; make that first call before any stream capture.
 *   If the context changes (e.g. after cudaDeviceReset the module is loaded
 *   again, possibly elsewhere), the next call looks the address up again, so
 *   that call, too, belongs outside a stream capture.
 */
QKN_API qkn_status flashnorm_proj_noalloc(const void *x, const void *W_folded, void *y,
                                          int64_t M, int64_t N, int64_t K, int w_k_major,
                                          float eps, void *stream);

/*
 * qkn_check_device -- synchronises `stream`, then reads and clears the
 * current device's error word.  Returns QKN_ERR_TIMEOUT when a bounded
 * device-side wait of an earlier launch (the projection kernel's mbarrier
 * waits give up after 2 s) recorded a failure, QKN_ERR_CUDA when the
 * synchronisation itself failed, QKN_OK otherwise.  Not part of the page's
 * method: it is the host-visible end of the kernels' bounded waits.
 */
QKN_API qkn_status qkn_check_device(void *stream);

/*
 * qkn_testing_arm_wait_fault -- TESTING ONLY: exercises the bounded waits
 * without faulting the GPU.  Arms a one-shot fault for the next launch of the
 * staged norm kernel made from this host thread (qknorm_fused on rows it
 * handles, or rmsnorm_partial_stats with more than 8 segments on such rows;
 * with fewer the statistics read rows without a staging ring and the hook
 * stays armed): warp 0 of block 0 does not issue
 * the copies of its first tile, so its wait on that stage cannot complete;
 * every wait of that launch gives up after wait_ns (0 < wait_ns <= 2e9)
 * instead of 2 s, records the failure, drains and exits.  The launch's output
 * is then incomplete, and qkn_check_device reports QKN_ERR_TIMEOUT.
 */
QKN_API qkn_status qkn_testing_arm_wait_fault(uint64_t wait_ns);

/*
 * qkn_testing_arm_exchange_fault -- TESTING ONLY.  Arms, for this host
 * thread's next qkv_proj_qknorm call, a wait limit of wait_ns
 * (0 < wait_ns <= 2 s) and one epilogue warp that does not count itself in
 * after publishing its first partial sums, so the exchange waits of that row
 * block run out.  The kernel then records the
 * failure, stops waiting, and returns; qkn_check_device reports
 * QKN_ERR_TIMEOUT.  No GPU fault is involved.  QKN_ERR_SHAPE for a wait_ns
 * out of range.
 */
QKN_API qkn_status qkn_testing_arm_exchange_fault(uint64_t wait_ns);

/* Message describing the last nonzero status returned on this host thread. */
QKN_API const char *qkn_last_error(void);

/* Library version string, e.g. "qknorm 0.1.0 sm_100a". */
QKN_API const char *qkn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QKNORM_H */
