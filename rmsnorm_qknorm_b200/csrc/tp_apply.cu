// Apply step of tensor-parallel QK-Norm (SwiftQK, abstract).
#include <math.h>

#include "qkn_common.cuh"

// ---------------------------------------------------------------------------
// Apply step of tensor-parallel QK-Norm (SwiftQK, abstract): a shard holding
// d of the row's d_full elements normalises its slice once the n_part scalar
// partial sums of the row (one per shard or segment) have been gathered:
//   S = ((p_0 + p_1) + ...) + p_{n_part-1},   y_i = (x_i * rsqrt(S / d_full + eps)) * w_i
// 16-byte accesses when the row layout allows, with 2^tpr_log2 threads per
// row (narrow rows share a warp, so a short row does not leave lanes idle);
// otherwise one warp per row, element by element.
namespace qkn {
namespace {

template <typename TA, typename TW, bool VEC>
__global__ void __launch_bounds__(256) apply_partials_kernel(const uint8_t *__restrict__ x, uint8_t *__restrict__ y,
                                                             const TW *__restrict__ w, const float *__restrict__ part,
                                                             int64_t rows, int d, int64_t ld_bytes,
                                                             int64_t ldo_bytes, int n_part, int64_t p_row,
                                                             int64_t p_part, float d_full, float eps, int tpr_log2) {
    const int tpr = 1 << tpr_log2;
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> tpr_log2) + (threadIdx.x >> tpr_log2);
    const int t = threadIdx.x & (tpr - 1);
    if (row >= rows) return;  // no collective operations below
    float S = 0.f;
    for (int j = 0; j < n_part; ++j) S += __ldg(part + row * p_row + j * p_part);
    const float inv = rsqrtf(S / d_full + eps);
    const uint8_t *xr = x + row * ld_bytes;
    uint8_t *yr = y + row * ldo_bytes;
    if constexpr (VEC) {
        constexpr int E = Chunk<TA>::E;
        const int nchunks = d / E;
        for (int c0 = 0; c0 < nchunks; c0 += tpr * 4) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = c0 + u * tpr + t;
                v[u] = c < nchunks ? ld_stream(xr + (int64_t)c * 16) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = c0 + u * tpr + t;
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
        for (int i = t; i < d; i += tpr) ye[i] = from_f32<TA>((to_f32<TA>(xe[i]) * inv) * to_f32<TW>(w[i]));
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
    // threads per row: enough for four chunks each, at most a warp
    int tpr_log2 = 5;
    if (vec) {
        const int64_t per4 = (d / E + 3) / 4;
        tpr_log2 = 0;
        while (tpr_log2 < 5 && (int64_t(1) << tpr_log2) < per4) ++tpr_log2;
    }
    const int64_t rows_per_block = 256 >> tpr_log2;
    const int64_t blocks = (rows + rows_per_block - 1) / rows_per_block;
    if (blocks > 0x7fffffffLL) return fail(QKN_ERR_SHAPE, "rmsnorm_apply_partials: too many rows");
    const uint8_t *xb = static_cast<const uint8_t *>(x);
    uint8_t *yb = static_cast<uint8_t *>(y);
    const TW *wt = static_cast<const TW *>(w);
    if (vec)
        apply_partials_kernel<TA, TW, true><<<(unsigned)blocks, 256, 0, s>>>(
            xb, yb, wt, part, rows, (int)d, ld * (int64_t)es, ldo * (int64_t)es, n_part, p_row, p_part, (float)d_full, eps, tpr_log2);
    else
        apply_partials_kernel<TA, TW, false><<<(unsigned)blocks, 256, 0, s>>>(
            xb, yb, wt, part, rows, (int)d, ld * (int64_t)es, ldo * (int64_t)es, n_part, p_row, p_part, (float)d_full, eps, tpr_log2);
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
