// kv_cache.cu -- dequantize a list-of-blocks NVFP4 KV cache into one
// contiguous [1, blocks * block_tokens, heads, 128] tensor.
//
// NeMo AutoModel model-filter page, dequantize_kv_cache: block b of the cache
// is a quantized tensor of block_tokens * heads rows of 128 values (row =
// token-in-block * heads + head) with e2m1 codes, one e4m3 scale per 16 values
// and one amax; its global scale is amax / (6 * 448) and its rows dequantize
// as dequantize_nvfp4 does, (e2m1 * e4m3) * g in binary32, one final rounding
// to the output dtype.  Block b fills output tokens [b * block_tokens,
// (b + 1) * block_tokens), so the output of block b is one contiguous range.
//
// One fused launch for every block.  The work is cut into units of
// kThreads * kKvUnroll consecutive items (an item is 8 outputs, one 16-byte
// bf16 store, or 4 fp32 outputs) that never straddle two cache blocks; a CTA
// takes units in turn and each thread handles kKvUnroll items kThreads apart,
// so a warp's loads and stores are contiguous.  A unit's block pointers and
// amax are the same address for every thread of the CTA, and they are loaded
// while the previous unit runs, so the codes of a unit are requested without
// first waiting for a pointer.  e2m1 codes are decoded by the hardware
// e2m1 -> f16x2 conversion.
#define BSQ_DBG_FILE 4
#include "debug.cuh"
#include "common.cuh"

namespace bsq {

constexpr int kKvUnroll = 8;  // items per thread per unit

// The block pointers sit in device memory where the host cannot check them:
// word loads go through these, which fall back to byte loads when a pointer
// is not aligned for the word (a sliced tensor can start anywhere).
__device__ __forceinline__ uint32_t ld_codes(const uint8_t* p, uint32_t o, int bytes) {
    const uint8_t* q = p + (size_t)o * bytes;
    if ((reinterpret_cast<uintptr_t>(q) & (uintptr_t)(bytes - 1)) == 0)
        return (bytes == 4) ? __ldcs(reinterpret_cast<const unsigned int*>(q))
                            : (uint32_t)__ldcs(reinterpret_cast<const unsigned short*>(q));
    uint32_t w = 0;
    for (int i = 0; i < bytes; ++i) w |= (uint32_t)q[i] << (8 * i);
    return w;
}

__device__ __forceinline__ float ld_f32_any(const float* p) {
    if ((reinterpret_cast<uintptr_t>(p) & 3u) == 0) return __ldg(p);
    const uint8_t* q = reinterpret_cast<const uint8_t*>(p);
    return __uint_as_float((uint32_t)q[0] | ((uint32_t)q[1] << 8) | ((uint32_t)q[2] << 16) | ((uint32_t)q[3] << 24));
}

template <typename TOUT, int U>
__global__ void __launch_bounds__(kThreads) kv_dequant_kernel(const uint8_t* const* __restrict__ values,
                                                              const uint8_t* const* __restrict__ scales,
                                                              const float* const* __restrict__ amax,
                                                              FastDiv units_per_block, uint32_t items_per_block,
                                                              int64_t nunits, TOUT* __restrict__ y) {
    constexpr int EPI = (sizeof(TOUT) == 2) ? 8 : 4;  // outputs per item
    constexpr int UNIT = kThreads * U;                // items per unit
    int64_t unit = blockIdx.x;
    if (unit >= nunits) return;
    uint32_t b = fdiv((uint32_t)unit, units_per_block);
    const uint8_t* vb = values[b];
    const uint8_t* sb = scales[b];
    float a = ld_f32_any(amax[b]);
    for (; unit < nunits; unit += gridDim.x) {
        const uint32_t c = (uint32_t)unit - b * units_per_block.d;
        const float g = __fdiv_rn(a, 2688.0f);
        // the next unit's block pointers and amax, loaded while this unit runs
        const int64_t nxt = unit + gridDim.x;
        uint32_t nb = b;
        const uint8_t* nvb = vb;
        const uint8_t* nsb = sb;
        float na = a;
        if (nxt < nunits) {
            nb = fdiv((uint32_t)nxt, units_per_block);
            if (nb != b && BSQ_DOK((int64_t)nb * units_per_block.d < nunits)) {
                nvb = values[nb];
                nsb = scales[nb];
                na = ld_f32_any(amax[nb]);
            }
        }
        const uint32_t o0 = c * UNIT + threadIdx.x;  // item within the block
        uint32_t w[U], sc[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t o = o0 + u * kThreads;
            w[u] = sc[u] = 0u;
            if (o < items_per_block && BSQ_DOK(((o * EPI) >> 4) < items_per_block * EPI / 16)) {
                w[u] = ld_codes(vb, o, EPI / 2);
                // element o * EPI of the block: scale byte (o * EPI) / 16 of
                // the row-major [rows, 8] scales
                sc[u] = sb[(o * EPI) >> 4];
            }
        }
        TOUT* yb = y + (int64_t)b * items_per_block * EPI;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t o = o0 + u * kThreads;
            if (o >= items_per_block) continue;
            const uint32_t s2 = e4m3_to_f16x2(sc[u]);
            uint32_t e2[4];
            float v[8];
            e2m1x8_to_f16x2(w[u], e2);  // fp32 output: only the first 4 are used
            // e2m1 * s first (exact, from the f16 decodes), then one rounding by g
#pragma unroll
            for (int i = 0; i < EPI; i += 2) {
                const float2 t = mul_f32x2(mul_f16_to_f32(e2[i / 2], s2), make_float2(g, g));
                v[i] = t.x;
                v[i + 1] = t.y;
            }
            TOUT* dst = yb + (int64_t)o * EPI;
            if (!BSQ_DOK((int64_t)b * units_per_block.d < nunits && o < items_per_block)) continue;
            if (sizeof(TOUT) == 2) {
                uint4 o4;
                o4.x = pack_bf16x2(v[0], v[1]);
                o4.y = pack_bf16x2(v[2], v[3]);
                o4.z = pack_bf16x2(v[4], v[5]);
                o4.w = pack_bf16x2(v[6], v[7]);
                __stcs(reinterpret_cast<uint4*>(dst), o4);
            } else {
                __stcs(reinterpret_cast<float4*>(dst), make_float4(v[0], v[1], v[2], v[3]));
            }
        }
        b = nb;
        vb = nvb;
        sb = nsb;
        a = na;
    }
}

}  // namespace bsq

using namespace bsq;

BSQ_API bsq_status bsq_dequantize_kv_cache_nvfp4(const uint8_t* const* values, const uint8_t* const* scales,
                                                 const float* const* amax, int64_t nblocks, int64_t block_tokens,
                                                 int64_t heads, void* y, bsq_dtype yt, bsq_stream_t stream) {
    const char* fn = "bsq_dequantize_kv_cache_nvfp4";
    BSQ_TRY(check_dtype(yt));
    if (nblocks < 0 || block_tokens < 0 || heads < 0) return fail(BSQ_ERR_INVALID_ARG, "%s: negative size", fn);
    if (nblocks == 0 || block_tokens == 0 || heads == 0) return BSQ_OK;
    if (!values || !scales || !amax || !y) return fail(BSQ_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (!aligned(values, 8) || !aligned(scales, 8) || !aligned(amax, 8) || !aligned(y, 16))
        return fail(BSQ_ERR_INVALID_ARG, "%s: misaligned pointer", fn);
    const int epi = (yt == BSQ_BF16) ? 8 : 4;
    const int64_t items_per_block = block_tokens * heads * 128 / epi;
    const int64_t nitems = nblocks * items_per_block;
    if (items_per_block * epi > 0xFFFFFFFFll || nitems > 0xFFFFFFFFll)
        return fail(BSQ_ERR_UNSUPPORTED, "%s: more than 2**32 outputs per block or items in all", fn);
    constexpr int kUnit = kThreads * kKvUnroll;
    const int64_t upb = (items_per_block + kUnit - 1) / kUnit;  // units per cache block
    const int64_t nunits = nblocks * upb;
    const FastDiv fupb = make_fastdiv((uint32_t)upb);
    const uint32_t ipb = (uint32_t)items_per_block;
    cudaStream_t st = (cudaStream_t)stream;
    if (yt == BSQ_BF16)
        launch_fit_ctas<kv_dequant_kernel<uint16_t, kKvUnroll>>(nunits, st, values, scales, amax, fupb, ipb, nunits,
                                                                (uint16_t*)y);
    else
        launch_fit_ctas<kv_dequant_kernel<float, kKvUnroll>>(nunits, st, values, scales, amax, fupb, ipb, nunits,
                                                             (float*)y);
    return check_launch(fn);
}

#ifdef BSQ_DEBUG
cudaError_t bsq_dbg_take_kv(uint32_t* count, uint32_t* first) { return bsq::dbg_take(count, first); }
#endif
