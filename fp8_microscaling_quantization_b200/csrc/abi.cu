// abi.cu -- status strings, last-error reporting and device queries shared by
// every libbsq entry point.
#include <cstdarg>
#include <cstdio>

#include "host_util.h"

namespace bsq {

// ------------------------------------------------------------ host helpers --

static thread_local char g_last_error[512] = "";

bsq_status fail(bsq_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return s;
}

bsq_status check_launch(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(BSQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return BSQ_OK;
}

int sm_count() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

}  // namespace bsq

using namespace bsq;

BSQ_API const char* bsq_status_string(bsq_status s) {
    switch (s) {
        case BSQ_OK: return "ok";
        case BSQ_ERR_INVALID_ARG: return "invalid argument";
        case BSQ_ERR_UNSUPPORTED: return "unsupported";
        case BSQ_ERR_CUDA: return "CUDA error";
        case BSQ_ERR_DEVICE: return "device-reported error";
    }
    return "unknown status";
}

BSQ_API const char* bsq_last_error(void) { return g_last_error; }

BSQ_API int bsq_version(void) { return 1; }

