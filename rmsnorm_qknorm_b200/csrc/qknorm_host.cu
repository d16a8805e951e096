// Host-buffer form of qknorm_fused (streams rows through the GPU).
#include <math.h>

#include <mutex>

#include "qkn_common.cuh"

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
    // Chunk size: filling and draining the pipeline costs about one chunk each
    // way and every chunk a fixed overhead (its copies and events), so the best
    // chunk grows as the square root of the bytes moved: ~sqrt(bytes x 1.5 MB),
    // at least 16 MiB (below that one chunk beat three), at most what the
    // workspace holds; measured best near 56 MB for 2.1 GB and 17 MB for
    // 200 MB.  Which rows share a chunk never changes a row's result.
    {
        const double total = (double)T * (double)row_bytes;
        double target = sqrt(total * 1.5e6);
        if (target < 16.0 * 1024 * 1024) target = 16.0 * 1024 * 1024;
        int64_t rows_target = (int64_t)(target / (double)row_bytes);
        if (rows_target < 1) rows_target = 1;
        if (rows_target < chunk) chunk = rows_target;
    }
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
