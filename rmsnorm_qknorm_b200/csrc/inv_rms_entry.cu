// FlashNorm's row statistic on its own (FlashNorm: Fast Normalization for
// Transformers, abstract, item (ii)): the scalar 1/rms of each row of x, the
// pass flashnorm_proj runs beside the projection when it is given a [M]
// workspace.  The kernel is the projection's own statistics pass.
#include <math.h>

#include "gemm_tc.cuh"
#include "qkn_common.cuh"

extern "C" QKN_API qkn_status flashnorm_inv_rms(const void *x, float *inv, int64_t M, int64_t K, float eps,
                                                void *stream) {
    using namespace qkn;
    if (M < 0 || K < 1 || M > 0x7fffffffLL || K > 0x7fffffffLL)
        return fail(QKN_ERR_SHAPE, "flashnorm_inv_rms: bad sizes M=%lld K=%lld", (long long)M, (long long)K);
    if (K % 8 != 0) return fail(QKN_ERR_SHAPE, "flashnorm_inv_rms: K=%lld must be a multiple of 8", (long long)K);
    if (!(eps >= 0.f) || isinf(eps)) return fail(QKN_ERR_EPS, "flashnorm_inv_rms: eps must be finite and >= 0");
    if (M == 0) return QKN_OK;
    if (x == nullptr || inv == nullptr) return fail(QKN_ERR_NULL, "flashnorm_inv_rms: x and inv are required");
    if (!aligned(x, 16) || !aligned(inv, 4))
        return fail(QKN_ERR_ALIGN, "flashnorm_inv_rms: x must be 16-byte aligned, inv 4-byte aligned");
    return launch_inv_rms(x, inv, M, K, eps, static_cast<cudaStream_t>(stream));
}
