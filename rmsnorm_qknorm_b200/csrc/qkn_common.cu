// Error reporting and device queries shared by every entry point.
#include <atomic>
#include <stdarg.h>
#include <stdio.h>

#include "qkn_common.cuh"

namespace qkn {

static thread_local char g_last_error[512] = "";

qkn_status fail(qkn_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return st;
}

qkn_status cuda_fail(cudaError_t e, const char *what) {
    return fail(QKN_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

qkn_status check_launch(const char *what) {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? QKN_OK : cuda_fail(e, what);
}

int sm_count() {
    static std::atomic<int> cached[64];  // per device; 0 until first asked
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

}  // namespace qkn

extern "C" QKN_API const char *qkn_last_error(void) { return qkn::g_last_error; }

extern "C" QKN_API const char *qkn_version(void) { return "qknorm 0.1.0 sm_100a"; }
