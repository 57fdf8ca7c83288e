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
// One fused launch for every block: an item is 8 outputs (bf16, one 16-byte
// store) or 4 (fp32), consecutive lanes take consecutive items, and each warp
// walks a run of 32 * U items.  The block of an item comes from a
// constant-divisor multiply; a lane loads the block's pointers and global
// scale only when its item enters another block, so the load pipe carries
// little beyond the codes, the scale bytes and the stores.  e2m1 codes are
// decoded by the hardware e2m1 -> f16x2 conversion.
#include "common.cuh"

namespace bsq {

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
                                                              FastDiv items_per_block, int64_t nitems,
                                                              TOUT* __restrict__ y) {
    constexpr int EPI = (sizeof(TOUT) == 2) ? 8 : 4;  // outputs per item
    constexpr int RUN = 32 * U;                       // items of one warp's run
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
    // the block's pointers and global scale, reloaded only when a lane's item
    // moves into another block (a run lies in one block unless it straddles
    // a boundary)
    uint32_t cur = 0xFFFFFFFFu;
    const uint8_t* vb = nullptr;
    const uint8_t* sb = nullptr;
    float g = 0.0f;
    for (int64_t run = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); run * RUN < nitems;
         run += warps) {
        uint32_t w[U], sc[U];
        float gr[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t it = run * RUN + u * 32 + lane;  // consecutive lanes, consecutive items
            w[u] = sc[u] = 0u;
            gr[u] = 0.0f;
            if (it < nitems) {
                const uint32_t b = fdiv((uint32_t)it, items_per_block);
                if (b != cur) {
                    cur = b;
                    vb = values[b];
                    sb = scales[b];
                    g = __fdiv_rn(ld_f32_any(amax[b]), 2688.0f);
                }
                const uint32_t o = (uint32_t)it - b * items_per_block.d;  // item within the block
                w[u] = ld_codes(vb, o, EPI / 2);
                // element o * EPI of the block: row (o * EPI) / 128, scale column ((o * EPI) % 128) / 16,
                // i.e. scale byte (o * EPI) / 16 of the row-major [rows, 8] scales
                sc[u] = sb[(o * EPI) >> 4];
                gr[u] = g;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t it = run * RUN + u * 32 + lane;
            if (it >= nitems) continue;
            const float s = e4m3_decode(sc[u]);
            float e[8], v[8];
            e2m1x8_decode_hw(w[u], e);  // fp32 output: only the first 4 are used
            // e2m1 * s first (exact), then one rounding by g
#pragma unroll
            for (int i = 0; i < EPI; ++i) v[i] = __fmul_rn(__fmul_rn(e[i], s), gr[u]);
            TOUT* dst = y + it * EPI;
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
    if (items_per_block > 0x7FFFFFFF || nitems > 0xFFFFFFFFll)
        return fail(BSQ_ERR_UNSUPPORTED, "%s: more than 2**32 output items", fn);
    const FastDiv ipb = make_fastdiv((uint32_t)items_per_block);
    cudaStream_t st = (cudaStream_t)stream;
    if (yt == BSQ_BF16)
        launch_fit<kv_dequant_kernel<uint16_t, 8>>(nitems, 8, st, values, scales, amax, ipb, nitems, (uint16_t*)y);
    else
        launch_fit<kv_dequant_kernel<float, 8>>(nitems, 8, st, values, scales, amax, ipb, nitems, (float*)y);
    return check_launch(fn);
}
