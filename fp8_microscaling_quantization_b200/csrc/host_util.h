// host_util.h -- host-side helpers shared by the libbsq translation units:
// status / last-error reporting, device properties, fast integer division.
#pragma once

#include <cstdint>
#include <cstdio>
#include <cuda_runtime.h>

#include "../../include/bsq.h"

#define BSQ_API extern "C" __attribute__((visibility("default")))

namespace bsq {

// Records a message for bsq_last_error() and returns the status.
bsq_status fail(bsq_status s, const char* fmt, ...);

// Checks cudaGetLastError() after a launch.
bsq_status check_launch(const char* what);

// Number of SMs of the current device (cached per device).
int sm_count();

// Division by a runtime-constant 32-bit divisor d >= 1 without a divide
// instruction (round-up multiplier, Granlund & Montgomery 1994):
//   s = ceil(log2 d),  m = floor(2**32 * (2**s - d) / d) + 1,
//   n / d = (umulhi(n, m) + n) >> s   for every 32-bit n.
struct FastDiv {
    uint32_t d, m, s;
};

inline FastDiv make_fastdiv(uint32_t d) {
    FastDiv f;
    f.d = d;
    f.s = 0;
    while ((uint64_t(1) << f.s) < d) ++f.s;
    f.m = (uint32_t)(((uint64_t(1) << 32) * ((uint64_t(1) << f.s) - d)) / d + 1);
    return f;
}

#ifdef __CUDACC__
__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
    return (uint32_t)(((uint64_t)__umulhi(n, f.m) + n) >> f.s);
}
#endif

}  // namespace bsq
