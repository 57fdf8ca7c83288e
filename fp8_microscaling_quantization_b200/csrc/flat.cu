// flat.cu -- MXFP4, MXFP8 and FP8 (power-of-two) quantize, and dequantize for all formats.
//
// Work unit: a "chunk" of 8 consecutive elements (one 16-byte bf16 vector).
// A 16- or 32-column block spans 2 or 4 adjacent lanes of a warp, so the
// block amax is one or two warp shuffles.  Loads are 128-bit streaming
// loads; every warp store instruction writes one contiguous span.  Grids are
// multiples of the SM count with several chunks in flight per thread.
//
// Formulas: mxfp4 page quantize_mxfp4 / dequantize_mxfp4; nvfp4 page
// dequantize_nvfp4; deepseek_v41 quantization page quantize_cache ("fp8"),
// _power_of_two_ceiling; ModelOpt tensor_quantizer page, is_mxfp /
// _real_quantize (MXFP8: e4m3 elements, e8m0 scale per 32), with the MXFP4
// exponent rule carried over to e4m3 (2**(floor(log2(amax)) - 8)).
#include <cstdarg>
#include <cstring>
#include <mutex>

#define BSQ_DBG_FILE 1
#include "debug.cuh"
#include "common.cuh"
#include "tcgen05.cuh"

namespace bsq {

// ----------------------------------------------------------- MXFP4 / FP8 ----
// Flat block quantization (blocks never cross rows because K % block == 0).

template <typename T, int FMT /*0 = fp8, 1 = mxfp4, 3 = mxfp8*/, int BLOCK, int U>
__global__ void __launch_bounds__(kThreads) flat_quant_kernel(const T* __restrict__ x, int64_t nchunks,
                                                              uint8_t* __restrict__ codes,
                                                              uint8_t* __restrict__ scales) {
    constexpr int L = BLOCK / 8;
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t base = (int64_t)blockIdx.x * kThreads + (threadIdx.x & ~31); base < nchunks; base += U * stride) {
        Raw8<T> raw[U];  // every chunk's load in flight before any arithmetic
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t c = base + u * stride + lane;
            if (c < nchunks) raw[u].load(x + c * 8);
            else raw[u].zero();
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t c = base + u * stride + lane;
            float vu[8];
            raw[u].get(vu);
            const float amax_b = group_max<L>(amax8(vu));
            if (FMT == 1) {
                const int e = mx_exponent(amax_b);
                const float inv = exp2_int(-e);  // x * 2**-e == x / 2**e exactly
                float q[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) q[j] = vu[j] * inv;
                const uint32_t packed = e2m1x8_encode_hw(q);
                if (c < nchunks) {
                    reinterpret_cast<uint32_t*>(codes)[c] = packed;
                    if ((lane % L) == 0 && BSQ_DOK(c / L < nchunks / L)) scales[c / L] = (uint8_t)(e + 127);
                }
            } else if (FMT == 3) {
                // MXFP8: values above 448 saturate (cvt ... satfinite)
                const int e = mx8_exponent(amax_b);
                const float inv = exp2_int(-e);  // x * 2**-e == x / 2**e exactly
                uint2 w;
                w.x = e4m3x2_encode_hw(vu[0] * inv, vu[1] * inv) |
                      (e4m3x2_encode_hw(vu[2] * inv, vu[3] * inv) << 16);
                w.y = e4m3x2_encode_hw(vu[4] * inv, vu[5] * inv) |
                      (e4m3x2_encode_hw(vu[6] * inv, vu[7] * inv) << 16);
                if (c < nchunks) {
                    reinterpret_cast<uint2*>(codes)[c] = w;
                    if ((lane % L) == 0 && BSQ_DOK(c / L < nchunks / L)) scales[c / L] = (uint8_t)(e + 127);
                }
            } else {
                const uint32_t pb = pow2_scale_biased<8, 0x600000u>(amax_b);  // 448 = 1.75 * 2**8
                const float p = __uint_as_float(pb << 23);
                const float inv = __uint_as_float((254u - pb) << 23);  // 1 / p, exact
                uint2 w;
                w.x = e4m3x2_encode_hw(vu[0] * inv, vu[1] * inv) |
                      (e4m3x2_encode_hw(vu[2] * inv, vu[3] * inv) << 16);
                w.y = e4m3x2_encode_hw(vu[4] * inv, vu[5] * inv) |
                      (e4m3x2_encode_hw(vu[6] * inv, vu[7] * inv) << 16);
                if (c < nchunks) {
                    reinterpret_cast<uint2*>(codes)[c] = w;
                    if ((lane % L) == 0 && BSQ_DOK(c / L < nchunks / L)) scales[c / L] = (uint8_t)pb;
                }
            }
        }
    }
}

// Dequantize (all formats).  Item = the EPI consecutive output elements of
// one lane: 8 for bf16 output (one 16-byte store) and 4 for fp32 output (one
// 16-byte store), so consecutive lanes write consecutive 16-byte pieces and a
// warp store instruction covers one contiguous 512-byte span.  e2m1 and e4m3
// codes are decoded by the hardware conversions (exact).
//   FMT_MX : y = e2m1 * 2**(scale - 127)
//   FMT_NV : y = (e2m1 * e4m3(scale)) * g[row], row = block / bpr
//   FMT_FP8: y = e4m3 * 2**(scale - 127)
enum { FMT_FP8 = 0, FMT_MX = 1, FMT_NV = 2 };

template <int FMT, typename TOUT, int BLOCK, int U>
__global__ void __launch_bounds__(kThreads) dequant_kernel(const uint8_t* __restrict__ codes,
                                                           const uint8_t* __restrict__ scales,
                                                           const float* __restrict__ g, FastDiv bpr,
                                                           int64_t nitems, TOUT* __restrict__ y) {
    constexpr int EPI = (sizeof(TOUT) == 2) ? 8 : 4;         // elements per item
    constexpr int CB = (FMT == FMT_FP8) ? EPI : EPI / 2;     // code bytes per item
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t base = (int64_t)blockIdx.x * kThreads + threadIdx.x; base < nitems; base += U * stride) {
        uint32_t w0[U], w1[U], sc[U];
        float gr[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t it = base + u * stride;
            w0[u] = w1[u] = sc[u] = 0u;
            gr[u] = 0.0f;
            if (it < nitems) {
                if (CB == 2) w0[u] = __ldcs(reinterpret_cast<const unsigned short*>(codes) + it);
                else if (CB == 4) w0[u] = __ldcs(reinterpret_cast<const unsigned int*>(codes) + it);
                else {
                    const uint2 t = __ldcs(reinterpret_cast<const uint2*>(codes) + it);
                    w0[u] = t.x;
                    w1[u] = t.y;
                }
                const int64_t blk = (it * EPI) / BLOCK;
                if (BSQ_DOK(blk * BLOCK < nitems * EPI)) sc[u] = scales[blk];
                if (FMT == FMT_NV && BSQ_DOK((int64_t)fdiv((uint32_t)blk, bpr) * bpr.d * BLOCK < nitems * EPI))
                    gr[u] = g[fdiv((uint32_t)blk, bpr)];
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t it = base + u * stride;
            if (it >= nitems) continue;
            float v[8];
            if (FMT == FMT_FP8) {
                const float p = e8m0_decode(sc[u]);
#pragma unroll
                for (int i = 0; i < EPI / 2; ++i) {
                    const uint32_t word = (i < 2) ? w0[u] : w1[u];
                    const float2 d = mul_f32x2(e4m3x2_decode_hw((word >> (16 * (i & 1))) & 0xFFFFu), make_float2(p, p));
                    v[2 * i] = d.x;
                    v[2 * i + 1] = d.y;
                }
            } else if (FMT == FMT_MX) {
                const float s = e8m0_decode(sc[u]);
                // e2m1 * s is exact (a power of two); the decode gives code 8 as +0
                float e[8];
                e2m1x8_decode_hw(w0[u], e);  // fp32 output: the first EPI = 4 are used
                const float2 s2 = make_float2(s, s);
#pragma unroll
                for (int j = 0; j < EPI; j += 2) {
                    const float2 t = mul_f32x2(make_float2(e[j], e[j + 1]), s2);
                    v[j] = t.x;
                    v[j + 1] = t.y;
                }
            } else {
                // NVFP4: e2m1 * e4m3 is exact (6 significant bits), taken from
                // the f16 decodes, then one rounding by the row scale
                const uint32_t s2 = e4m3_to_f16x2(sc[u]);
                uint32_t e2[4];
                e2m1x8_to_f16x2(w0[u], e2);  // fp32 output: the first EPI = 4 are used
                const float2 g2 = make_float2(gr[u], gr[u]);
#pragma unroll
                for (int j = 0; j < EPI; j += 2) {
                    const float2 t = mul_f32x2(mul_f16_to_f32(e2[j / 2], s2), g2);
                    v[j] = t.x;
                    v[j + 1] = t.y;
                }
            }
            TOUT* dst = y + it * EPI;
            if (!BSQ_DOK(it < nitems)) continue;
            if (sizeof(TOUT) == 2) {
                store8(reinterpret_cast<uint16_t*>(dst), v);
            } else {
                __stcs(reinterpret_cast<float4*>(dst), make_float4(v[0], v[1], v[2], v[3]));
            }
        }
    }
}

}  // namespace bsq

using namespace bsq;

BSQ_API bsq_status bsq_dequantize_nvfp4(const uint8_t* packed, const uint8_t* scales_e4m3, const float* row_scale,
                                        int64_t rows, int64_t K, void* y, bsq_dtype yt, bsq_stream_t stream) {
    BSQ_TRY(check_dtype(yt));
    BSQ_TRY(check_matrix("bsq_dequantize_nvfp4", packed, rows, K, 16));
    if (rows * K == 0) return BSQ_OK;
    if (!scales_e4m3 || !row_scale || !y) return fail(BSQ_ERR_INVALID_ARG, "bsq_dequantize_nvfp4: null pointer");
    if (!aligned(packed, 4) || !aligned(y, 16)) return fail(BSQ_ERR_INVALID_ARG, "bsq_dequantize_nvfp4: misaligned pointer");
    const FastDiv bpr = make_fastdiv((uint32_t)(K / 16));
    cudaStream_t st = (cudaStream_t)stream;
    if (yt == BSQ_BF16) {
        const int64_t nitems = rows * K / 8;
        launch_fit<dequant_kernel<FMT_NV, uint16_t, 16, 4>>(nitems, 4, st, packed, scales_e4m3, row_scale, bpr, nitems,
                                                              (uint16_t*)y);
    } else {
        const int64_t nitems = rows * K / 4;
        launch_fit<dequant_kernel<FMT_NV, float, 16, 4>>(nitems, 4, st, packed, scales_e4m3, row_scale, bpr, nitems,
                                                           (float*)y);
    }
    return check_launch("bsq_dequantize_nvfp4");
}

BSQ_API bsq_status bsq_quantize_mxfp4(const void* x, bsq_dtype xt, int64_t rows, int64_t K, uint8_t* packed,
                                      uint8_t* scales_e8m0, bsq_stream_t stream) {
    BSQ_TRY(check_dtype(xt));
    BSQ_TRY(check_matrix("bsq_quantize_mxfp4", x, rows, K, 32));
    if (rows * K == 0) return BSQ_OK;
    if (!packed || !scales_e8m0) return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_mxfp4: null output");
    if (!aligned(x, 16) || !aligned(packed, 4)) return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_mxfp4: misaligned pointer");
    const int64_t nchunks = rows * K / 8;
    cudaStream_t st = (cudaStream_t)stream;
    if (xt == BSQ_BF16)
        launch_fit<flat_quant_kernel<uint16_t, 1, 32, 4>>(nchunks, 4, st, (const uint16_t*)x, nchunks, packed,
                                                            scales_e8m0);
    else
        launch_fit<flat_quant_kernel<float, 1, 32, 4>>(nchunks, 4, st, (const float*)x, nchunks, packed, scales_e8m0);
    return check_launch("bsq_quantize_mxfp4");
}

BSQ_API bsq_status bsq_dequantize_mxfp4(const uint8_t* packed, const uint8_t* scales_e8m0, int64_t rows, int64_t K,
                                        void* y, bsq_dtype yt, bsq_stream_t stream) {
    BSQ_TRY(check_dtype(yt));
    BSQ_TRY(check_matrix("bsq_dequantize_mxfp4", packed, rows, K, 32));
    if (rows * K == 0) return BSQ_OK;
    if (!scales_e8m0 || !y) return fail(BSQ_ERR_INVALID_ARG, "bsq_dequantize_mxfp4: null pointer");
    if (!aligned(packed, 4) || !aligned(y, 16)) return fail(BSQ_ERR_INVALID_ARG, "bsq_dequantize_mxfp4: misaligned pointer");
    cudaStream_t st = (cudaStream_t)stream;
    const FastDiv none = make_fastdiv(1);
    if (yt == BSQ_BF16) {
        const int64_t nitems = rows * K / 8;
        launch_fit<dequant_kernel<FMT_MX, uint16_t, 32, 4>>(nitems, 4, st, packed, scales_e8m0, (const float*)nullptr,
                                                              none, nitems, (uint16_t*)y);
    } else {
        const int64_t nitems = rows * K / 4;
        launch_fit<dequant_kernel<FMT_MX, float, 32, 4>>(nitems, 4, st, packed, scales_e8m0, (const float*)nullptr, none,
                                                           nitems, (float*)y);
    }
    return check_launch("bsq_dequantize_mxfp4");
}

BSQ_API bsq_status bsq_quantize_mxfp8(const void* x, bsq_dtype xt, int64_t rows, int64_t K, uint8_t* codes_e4m3,
                                      uint8_t* scales_e8m0, bsq_stream_t stream) {
    BSQ_TRY(check_dtype(xt));
    BSQ_TRY(check_matrix("bsq_quantize_mxfp8", x, rows, K, 32));
    if (rows * K == 0) return BSQ_OK;
    if (!codes_e4m3 || !scales_e8m0) return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_mxfp8: null output");
    if (!aligned(x, 16) || !aligned(codes_e4m3, 8))
        return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_mxfp8: misaligned pointer");
    const int64_t nchunks = rows * K / 8;
    cudaStream_t st = (cudaStream_t)stream;
    if (xt == BSQ_BF16)
        launch_fit<flat_quant_kernel<uint16_t, 3, 32, 4>>(nchunks, 4, st, (const uint16_t*)x, nchunks, codes_e4m3,
                                                            scales_e8m0);
    else
        launch_fit<flat_quant_kernel<float, 3, 32, 4>>(nchunks, 4, st, (const float*)x, nchunks, codes_e4m3,
                                                         scales_e8m0);
    return check_launch("bsq_quantize_mxfp8");
}

// MXFP8 dequantize is the e4m3 * 2**(scale - 127) decode of the FP8 stored
// form with 32-element blocks.
BSQ_API bsq_status bsq_dequantize_mxfp8(const uint8_t* codes_e4m3, const uint8_t* scales_e8m0, int64_t rows,
                                        int64_t K, void* y, bsq_dtype yt, bsq_stream_t stream) {
    BSQ_TRY(check_dtype(yt));
    BSQ_TRY(check_matrix("bsq_dequantize_mxfp8", codes_e4m3, rows, K, 32));
    if (rows * K == 0) return BSQ_OK;
    if (!scales_e8m0 || !y) return fail(BSQ_ERR_INVALID_ARG, "bsq_dequantize_mxfp8: null pointer");
    if (!aligned(codes_e4m3, 8) || !aligned(y, 16))
        return fail(BSQ_ERR_INVALID_ARG, "bsq_dequantize_mxfp8: misaligned pointer");
    cudaStream_t st = (cudaStream_t)stream;
    const FastDiv none = make_fastdiv(1);
    const float* nog = nullptr;
    if (yt == BSQ_BF16) {
        const int64_t nb = rows * K / 8;
        launch_fit<dequant_kernel<FMT_FP8, uint16_t, 32, 4>>(nb, 4, st, codes_e4m3, scales_e8m0, nog, none, nb,
                                                               (uint16_t*)y);
    } else {
        const int64_t nf = rows * K / 4;
        launch_fit<dequant_kernel<FMT_FP8, float, 32, 4>>(nf, 4, st, codes_e4m3, scales_e8m0, nog, none, nf,
                                                            (float*)y);
    }
    return check_launch("bsq_dequantize_mxfp8");
}

BSQ_API bsq_status bsq_quantize_fp8(const void* x, bsq_dtype xt, int64_t rows, int64_t K, int block,
                                    uint8_t* codes_e4m3, uint8_t* scales_e8m0, bsq_stream_t stream) {
    BSQ_TRY(check_dtype(xt));
    if (block != 16 && block != 32) return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_fp8: block must be 16 or 32");
    BSQ_TRY(check_matrix("bsq_quantize_fp8", x, rows, K, block));
    if (rows * K == 0) return BSQ_OK;
    if (!codes_e4m3 || !scales_e8m0) return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_fp8: null output");
    if (!aligned(x, 16) || !aligned(codes_e4m3, 8)) return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_fp8: misaligned pointer");
    const int64_t nchunks = rows * K / 8;
    cudaStream_t st = (cudaStream_t)stream;
    if (xt == BSQ_BF16) {
        const uint16_t* xb = (const uint16_t*)x;
        if (block == 32) launch_fit<flat_quant_kernel<uint16_t, 0, 32, 4>>(nchunks, 4, st, xb, nchunks, codes_e4m3, scales_e8m0);
        else launch_fit<flat_quant_kernel<uint16_t, 0, 16, 4>>(nchunks, 4, st, xb, nchunks, codes_e4m3, scales_e8m0);
    } else {
        const float* xf = (const float*)x;
        if (block == 32) launch_fit<flat_quant_kernel<float, 0, 32, 4>>(nchunks, 4, st, xf, nchunks, codes_e4m3, scales_e8m0);
        else launch_fit<flat_quant_kernel<float, 0, 16, 4>>(nchunks, 4, st, xf, nchunks, codes_e4m3, scales_e8m0);
    }
    return check_launch("bsq_quantize_fp8");
}

BSQ_API bsq_status bsq_dequantize_fp8(const uint8_t* codes_e4m3, const uint8_t* scales_e8m0, int64_t rows, int64_t K,
                                      int block, void* y, bsq_dtype yt, bsq_stream_t stream) {
    BSQ_TRY(check_dtype(yt));
    if (block != 16 && block != 32) return fail(BSQ_ERR_INVALID_ARG, "bsq_dequantize_fp8: block must be 16 or 32");
    BSQ_TRY(check_matrix("bsq_dequantize_fp8", codes_e4m3, rows, K, block));
    if (rows * K == 0) return BSQ_OK;
    if (!scales_e8m0 || !y) return fail(BSQ_ERR_INVALID_ARG, "bsq_dequantize_fp8: null pointer");
    if (!aligned(codes_e4m3, 8) || !aligned(y, 16)) return fail(BSQ_ERR_INVALID_ARG, "bsq_dequantize_fp8: misaligned pointer");
    cudaStream_t st = (cudaStream_t)stream;
    const FastDiv none = make_fastdiv(1);
    const int64_t nb = rows * K / 8, nf = rows * K / 4;
    if (yt == BSQ_BF16) {
        const float* nog = nullptr;
        if (block == 32) launch_fit<dequant_kernel<FMT_FP8, uint16_t, 32, 4>>(nb, 4, st, codes_e4m3, scales_e8m0, nog, none, nb, (uint16_t*)y);
        else launch_fit<dequant_kernel<FMT_FP8, uint16_t, 16, 4>>(nb, 4, st, codes_e4m3, scales_e8m0, nog, none, nb, (uint16_t*)y);
    } else {
        const float* nog = nullptr;
        if (block == 32) launch_fit<dequant_kernel<FMT_FP8, float, 32, 4>>(nf, 4, st, codes_e4m3, scales_e8m0, nog, none, nf, (float*)y);
        else launch_fit<dequant_kernel<FMT_FP8, float, 16, 4>>(nf, 4, st, codes_e4m3, scales_e8m0, nog, none, nf, (float*)y);
    }
    return check_launch("bsq_dequantize_fp8");
}

#ifdef BSQ_DEBUG
cudaError_t bsq_dbg_take_flat(uint32_t* count, uint32_t* first) { return bsq::dbg_take(count, first); }
#endif
