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

#ifdef BSQ_DEBUG
// each unit's collector (debug builds only), defined next to its kernels
cudaError_t bsq_dbg_take_flat(uint32_t*, uint32_t*);
cudaError_t bsq_dbg_take_nvfp4(uint32_t*, uint32_t*);
cudaError_t bsq_dbg_take_static(uint32_t*, uint32_t*);
cudaError_t bsq_dbg_take_kv(uint32_t*, uint32_t*);
cudaError_t bsq_dbg_take_cache(uint32_t*, uint32_t*);
cudaError_t bsq_dbg_take_gmm(uint32_t*, uint32_t*);

BSQ_API bsq_status bsq_debug_counters(uint32_t* count, uint32_t* first_code) {
    if (!count || !first_code) return fail(BSQ_ERR_INVALID_ARG, "bsq_debug_counters: null pointer");
    *count = 0;
    *first_code = 0;
    cudaError_t e = cudaDeviceSynchronize();
    cudaError_t (*take[])(uint32_t*, uint32_t*) = {bsq_dbg_take_flat, bsq_dbg_take_nvfp4, bsq_dbg_take_static,
                                                  bsq_dbg_take_kv, bsq_dbg_take_cache, bsq_dbg_take_gmm};
    for (auto f : take)
        if (e == cudaSuccess) e = f(count, first_code);
    if (e != cudaSuccess) return fail(BSQ_ERR_CUDA, "bsq_debug_counters: %s", cudaGetErrorString(e));
    return BSQ_OK;
}
#else
BSQ_API bsq_status bsq_debug_counters(uint32_t* count, uint32_t* first_code) {
    if (count) *count = 0;
    if (first_code) *first_code = 0;
    return fail(BSQ_ERR_UNSUPPORTED, "bsq_debug_counters: not a BSQ_DEBUG build");
}
#endif

