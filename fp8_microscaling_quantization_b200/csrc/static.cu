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
// A lane is 8 consecutive elements (one 16-byte load and store), so a warp
// instruction covers one contiguous span; the two lanes of a block each
// derive its scale.  Four chunks in flight per lane.  The physical scale of
// each of the 128 positive e4m3 codes (and its reciprocal) is tabulated per
// CTA, since f is fixed per launch; the e2m1 codes of x / sq come from the
// division-free exact quotient rounding, and decode back through the
// hardware e2m1 -> f16x2 conversion.
#define BSQ_DBG_FILE 3
#include "debug.cuh"
#include "common.cuh"

namespace bsq {

// (float)(2**-9 / 448): the smallest e4m3 subnormal over the e4m3 maximum,
// rounded to binary32 once from its binary64 value
constexpr float kStaticMinRatio = (float)(0.001953125 / 448.0);

template <typename T, int U>
__global__ void __launch_bounds__(kThreads) nv_static_fq_kernel(const T* __restrict__ x,
                                                                const float* __restrict__ block_amax,
                                                                const float* __restrict__ global_amax,
                                                                int64_t nchunks, T* y) {
    // the physical scale of every positive e4m3 code, and its reciprocal, for
    // this launch's global amax (one division per code, not per block)
    __shared__ float sq_of[128], rsq_of[128];
    float pts = __fdiv_rn(__ldg(global_amax), 6.0f);
    if (pts <= 1e-8f) pts = 1e-8f;
    const float min_value = __fmul_rn(kStaticMinRatio, pts);
    const float f = __fdiv_rn(448.0f, pts);
    for (int c = threadIdx.x; c < 128; c += kThreads) {
        const float sq = __fdiv_rn(e4m3_decode((uint32_t)c), f);
        sq_of[c] = sq;
        rsq_of[c] = __frcp_rn(sq);
    }
    __syncthreads();
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t base = (int64_t)blockIdx.x * kThreads + threadIdx.x; base < nchunks; base += U * stride) {
        float v[U][8], a[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t c = base + u * stride;
            if (c < nchunks && BSQ_DOK((c >> 1) < (nchunks + 1) / 2)) {
                load8(x + c * 8, v[u]);
                a[u] = __ldg(block_amax + (c >> 1));
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) v[u][j] = 0.0f;
                a[u] = 0.0f;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t c = base + u * stride;
            if (c >= nchunks) continue;
            // both lanes of a block derive the same scale from the same amax;
            // sb * f is positive and at most 448, so the code is in 1..126
            float sb = __fdiv_rn(a[u], 6.0f);
            if (sb <= min_value) sb = min_value;
            const uint32_t code = e4m3x2_encode_hw(__fmul_rn(sb, f), 0.0f) & 0x7Fu;
            const float sq = sq_of[code];
            const uint32_t pk = e2m1x8_of_quotient_r(v[u], sq, rsq_of[code]);
            float e[8], o[8];
            e2m1x8_decode_hw(pk, e);
#pragma unroll
            for (int j = 0; j < 8; ++j) o[j] = __fmul_rn(e[j], sq);
            store8(y + c * 8, o);
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
    const int64_t nchunks = rows * K / 8;
    cudaStream_t st = (cudaStream_t)stream;
    if (t == BSQ_BF16)
        launch_fit<nv_static_fq_kernel<uint16_t, 4>>(nchunks, 4, st, (const uint16_t*)x, block_amax, global_amax,
                                                      nchunks, (uint16_t*)y);
    else
        launch_fit<nv_static_fq_kernel<float, 4>>(nchunks, 4, st, (const float*)x, block_amax, global_amax, nchunks,
                                                   (float*)y);
    return check_launch(fn);
}

#ifdef BSQ_DEBUG
cudaError_t bsq_dbg_take_static(uint32_t* count, uint32_t* first) { return bsq::dbg_take(count, first); }
#endif
