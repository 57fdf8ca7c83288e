// static.cu -- static two-level NVFP4 fake-quant (calibrated scales).
//
// ModelOpt tensor_quantizer page, StaticBlockScaleQuantizer: the block amax
// comes from calibration (an input, one fp32 per 16-element block) and one
// global amax A sets the second level:
//   per-tensor scale   pts = A / 6, floored at 1e-8          (_amax_to_scale)
//   floor              min_value = (2**-9 / 448) * pts        (_block_scale_from_amax)
//   block scale        sb = amax_b / 6, or min_value where amax_b / 6 <= min_value
//   e4m3 block scale   code = e4m3(sb * f), sq = e4m3(code) / f, f = 448 / pts
//                      (scaled_e4m3 maps pts to 448)
//   output             y = cast(e2m1(x / sq) * sq)              (_fake_quantize)
// binary32 throughout, every product and quotient rounded once, in this order.
// The straight-through backward is the identity (no kernel).
//
// One lane per 16-element block, two blocks in flight per lane; the e2m1
// codes of x / sq come from the division-free exact quotient rounding.
#include "common.cuh"

namespace bsq {

// (float)(2**-9 / 448): the smallest e4m3 subnormal over the e4m3 maximum,
// rounded to binary32 once from its binary64 value
constexpr float kStaticMinRatio = (float)(0.001953125 / 448.0);

template <typename T, int U>
__global__ void __launch_bounds__(kThreads) nv_static_fq_kernel(const T* __restrict__ x,
                                                                const float* __restrict__ block_amax,
                                                                const float* __restrict__ global_amax,
                                                                int64_t nblocks, T* y) {
    float pts = __fdiv_rn(__ldg(global_amax), 6.0f);
    if (pts <= 1e-8f) pts = 1e-8f;
    const float min_value = __fmul_rn(kStaticMinRatio, pts);
    const float f = __fdiv_rn(448.0f, pts);
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t base = (int64_t)blockIdx.x * kThreads + threadIdx.x; base < nblocks; base += U * stride) {
        float v[U][16], a[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t b = base + u * stride;
            if (b < nblocks) {
                load16(x + b * 16, v[u]);
                a[u] = __ldg(block_amax + b);
            } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) v[u][j] = 0.0f;
                a[u] = 0.0f;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t b = base + u * stride;
            if (b >= nblocks) continue;
            float sb = __fdiv_rn(a[u], 6.0f);
            if (sb <= min_value) sb = min_value;
            const uint32_t code = e4m3x2_encode_hw(__fmul_rn(sb, f), 0.0f) & 0xFFu;
            const float sq = __fdiv_rn(e4m3_decode(code), f);
            const uint32_t c0 = e2m1x8_of_quotient(v[u], sq), c1 = e2m1x8_of_quotient(v[u] + 8, sq);
            float o[16];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                o[j] = __fmul_rn(e2m1_decode((c0 >> (4 * j)) & 15u), sq);
                o[8 + j] = __fmul_rn(e2m1_decode((c1 >> (4 * j)) & 15u), sq);
            }
            store8(y + b * 16, o);
            store8(y + b * 16 + 8, o + 8);
        }
    }
}

}  // namespace bsq

using namespace bsq;

BSQ_API bsq_status bsq_fake_quantize_nvfp4_static(const void* x, bsq_dtype t, int64_t rows, int64_t K,
                                                  const float* block_amax, const float* global_amax, void* y,
                                                  bsq_stream_t stream) {
    const char* fn = "bsq_fake_quantize_nvfp4_static";
    BSQ_TRY(check_dtype(t));
    BSQ_TRY(check_matrix(fn, x, rows, K, 16));
    if (rows * K == 0) return BSQ_OK;
    if (!block_amax || !global_amax || !y) return fail(BSQ_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(block_amax, 4) || !aligned(global_amax, 4))
        return fail(BSQ_ERR_INVALID_ARG, "%s: misaligned pointer", fn);
    const size_t bytes = (size_t)(rows * K) * (t == BSQ_BF16 ? 2 : 4);
    const char* xb = (const char*)x;
    const char* yb = (const char*)y;
    if (xb != yb && xb < yb + bytes && yb < xb + bytes)
        return fail(BSQ_ERR_INVALID_ARG, "%s: x and y overlap without being the same buffer", fn);
    const int64_t nblocks = rows * K / 16;
    cudaStream_t st = (cudaStream_t)stream;
    if (t == BSQ_BF16)
        launch_fit<nv_static_fq_kernel<uint16_t, 2>>(nblocks, 2, st, (const uint16_t*)x, block_amax, global_amax,
                                                      nblocks, (uint16_t*)y);
    else
        launch_fit<nv_static_fq_kernel<float, 2>>(nblocks, 2, st, (const float*)x, block_amax, global_amax, nblocks,
                                                   (float*)y);
    return check_launch(fn);
}
