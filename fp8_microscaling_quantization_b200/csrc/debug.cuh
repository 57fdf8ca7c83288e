// debug.cuh -- index checks of the BSQ_DEBUG build of libbsq.
//
// Built with -DBSQ_DEBUG, every checked device access first tests its index
// against the extent the kernel was given.  A failing check skips the access
// (the kernel never traps), counts the failure in a device word of its
// translation unit and records the first failing check as (file id << 16) |
// source line.  bsq_debug_counters() collects and clears the words of all
// units.  Without BSQ_DEBUG a check is the constant true and costs nothing.
// Each .cu file defines BSQ_DBG_FILE (its file id) before including this.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace bsq {

#ifdef BSQ_DEBUG
static __device__ uint32_t g_dbg_count;
static __device__ uint32_t g_dbg_first;

__device__ __forceinline__ bool dbg_ok(bool cond, uint32_t code) {
    if (!cond && atomicAdd(&g_dbg_count, 1u) == 0u) g_dbg_first = code;
    return cond;
}

// Adds this unit's failure count to *count, records its first failing check
// in *first when *first is still 0, and clears the unit's words.
static inline cudaError_t dbg_take(uint32_t* count, uint32_t* first) {
    uint32_t c = 0, f = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&c, g_dbg_count, sizeof(c));
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&f, g_dbg_first, sizeof(f));
    if (e != cudaSuccess) return e;
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_dbg_count, &zero, sizeof(zero));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_dbg_first, &zero, sizeof(zero));
    *count += c;
    if (*first == 0 && c != 0) *first = f;
    return e;
}

#define BSQ_DOK(cond) ::bsq::dbg_ok((cond), ((uint32_t)(BSQ_DBG_FILE) << 16) | (uint32_t)__LINE__)
#else
#define BSQ_DOK(cond) (true)
#endif

}  // namespace bsq
