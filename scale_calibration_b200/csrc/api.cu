// Status strings, thread-local error detail, device queries.
#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "common.cuh"

namespace lh {

static thread_local char g_msg[512];

void clear_error() { g_msg[0] = 0; }

lh_status fail(lh_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return s;
}

lh_status cuda_status(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return LH_OK;
    return fail(LH_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

int sm_count() {
    static std::mutex mu;
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cache[dev] = n;
    }
    return cache[dev];
}

}  // namespace lh

extern "C" const char* lh_status_string(lh_status s) {
    switch (s) {
        case LH_OK: return "LH_OK";
        case LH_ERR_INVALID_ARG: return "LH_ERR_INVALID_ARG";
        case LH_ERR_UNSUPPORTED: return "LH_ERR_UNSUPPORTED";
        case LH_ERR_ALIGNMENT: return "LH_ERR_ALIGNMENT";
        case LH_ERR_WORKSPACE: return "LH_ERR_WORKSPACE";
        case LH_ERR_CUDA: return "LH_ERR_CUDA";
        case LH_ERR_TIMEOUT: return "LH_ERR_TIMEOUT";
    }
    return "LH_ERR_UNKNOWN";
}

extern "C" const char* lh_last_error_message(void) { return lh::g_msg; }
