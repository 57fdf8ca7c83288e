// grouped_mm.cu -- fused-dequant grouped GEMM (placeholder until the tcgen05 kernel lands).
#include "host_util.h"

using namespace bsq;

BSQ_API bsq_status bsq_grouped_mm_fp4(bsq_format fmt, bsq_dir dir, const void* a, const uint8_t* packed,
                                      const uint8_t* scales, const float* row_scale, const int32_t* offs, int E,
                                      int64_t T, int64_t N, int64_t K, void* out, uint32_t* err,
                                      bsq_stream_t stream) {
    (void)fmt; (void)dir; (void)a; (void)packed; (void)scales; (void)row_scale; (void)offs; (void)E;
    (void)T; (void)N; (void)K; (void)out; (void)err; (void)stream;
    return fail(BSQ_ERR_UNSUPPORTED, "bsq_grouped_mm_fp4: not built yet");
}
