// cache.cu -- quantize_cache fake-quant and its straight-through backward.
//
// Formulas: deepseek_v41 quantization page quantize_cache /
// _CacheQuantization.forward / .backward: quantize then dequantize each group
// of `block` channels in binary32, one final rounding to the input dtype; a
// final partial group is zero-padded.
#include <cstdarg>
#include <cstring>
#include <mutex>

#define BSQ_DBG_FILE 5
#include "debug.cuh"
#include "common.cuh"
#include "tcgen05.cuh"

namespace bsq {

// ------------------------------------------------------- quantize_cache ----
// Per-CTA tables of the NVFP4 path (unused by the other formats).
struct NvTables {
    float inv[128];
    NvBound bounds[8];
};
__device__ __forceinline__ void fill_nv_tables(NvTables* t) {
    fill_inv_e4m3(t->inv);
    fill_nv_bounds(t->bounds);
}

template <int FMT, int L>
__device__ __forceinline__ void cache_chunk(const float v[8], float g, float rg, const NvTables* tab, float out[8]);

// S lanes per row (S a power of two, 2 <= S <= 32; 32/S rows per warp); lane
// i of a row walks the chunks i, i + S, ...  of the zero-padded row, so the
// L lanes of a block are adjacent.  VEC: rows are 16-byte aligned and C % 8 == 0.

template <typename T, int FMT, int BLOCK, int S, bool VEC>
__global__ void __launch_bounds__(kThreads) cache_kernel(const T* __restrict__ x, T* __restrict__ y, int64_t rows,
                                                         int64_t C) {
    constexpr int L = BLOCK / 8;
    constexpr int RPW = 32 / S;  // rows per warp
    __shared__ NvTables tab;
    if (FMT == BSQ_NVFP4) {
        fill_nv_tables(&tab);
        __syncthreads();
    }
    const int lane = threadIdx.x & 31;
    const int sl = lane % S;
    const int64_t nb = (C + BLOCK - 1) / BLOCK;
    const int64_t cpr = nb * L;  // chunks in the padded row
    const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
    const int64_t wid = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    for (int64_t r0 = wid * RPW; r0 < rows; r0 += warps * RPW) {
        const int64_t r = r0 + lane / S;
        const bool row_ok = r < rows;
        const T* xr = x + (row_ok ? r : 0) * C;
        T* yr = y + (row_ok ? r : 0) * C;
        float g = 0.0f, rg = 0.0f;
        if (FMT == BSQ_NVFP4) {
            float m = 0.0f;
            for (int64_t c0 = 0; c0 < cpr; c0 += S) {
                const int64_t c = c0 + sl;
                float v[8];
                const int64_t n = C - c * 8;
                if (row_ok && c < cpr && n > 0) {
                    if (VEC && n >= 8) load8(xr + c * 8, v);
                    else load_n(xr + c * 8, (int)(n < 8 ? n : 8), v);
                    m = fmaxf(m, amax8(v));
                }
            }
            m = (S == 32) ? warp_max_nonneg(m) : group_max<S>(m);
            g = __fdiv_rn(m, kNvGlobalDiv);
            rg = nv_recip_or_zero(g);
        }
        for (int64_t c0 = 0; c0 < cpr; c0 += S) {
            const int64_t c = c0 + sl;
            const int64_t n = C - c * 8;
            float v[8];
            if (row_ok && c < cpr && n > 0) {
                if (VEC && n >= 8) load8(xr + c * 8, v);
                else load_n(xr + c * 8, (int)(n < 8 ? n : 8), v);
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j] = 0.0f;
            }
            float out[8];
            cache_chunk<FMT, L>(v, g, rg, &tab, out);
            if (row_ok && c < cpr && n > 0) {
                if (BSQ_DOK(r < rows && c * 8 < C)) {
                    if (VEC && n >= 8) store8(yr + c * 8, out);
                    else store_n(yr + c * 8, (int)(n < 8 ? n : 8), out);
                }
            }
        }
    }
}

// Fake-quant of one 8-element chunk in registers (the block's lanes are
// adjacent; g is the row scale for NVFP4, rg = nv_recip_or_zero(g)).  The
// power-of-two scales come from the bits of the block amax (pow2_scale_biased)
// and the NVFP4 codes from the brackets and the fma settling of straddled
// elements, all without a division; the dequantized value is one
// multiply by the positive scale, folded with +0.0 into an fma so that code 8
// (-0.0 from the hardware decode) gives the table's +0.0.
template <int FMT, int L>
__device__ __forceinline__ void cache_chunk(const float v[8], float g, float rg, const NvTables* tab, float out[8]) {
    const float amax_b = group_max<L>(amax8(v));
    const float2 zero2 = make_float2(0.0f, 0.0f);
    if (FMT == BSQ_FP8) {
        const uint32_t pb = pow2_scale_biased<8, 0x600000u>(amax_b);  // 448 = 1.75 * 2**8
        const float p = __uint_as_float(pb << 23), inv = __uint_as_float((254u - pb) << 23);
        const float2 inv2 = make_float2(inv, inv), p2 = make_float2(p, p);
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            const float2 q = mul_f32x2(make_float2(v[j], v[j + 1]), inv2);  // exact: inv is a power of two
            const float2 o = mul_f32x2(e4m3x2_decode_hw(e4m3x2_encode_hw(q.x, q.y)), p2);
            out[j] = o.x;
            out[j + 1] = o.y;
        }
    } else if (FMT == BSQ_MXFP4) {
        const uint32_t pb = pow2_scale_biased<2, 0x400000u>(amax_b);  // 6 = 1.5 * 2**2
        const float p = __uint_as_float(pb << 23), inv = __uint_as_float((254u - pb) << 23);
        const float2 inv2 = make_float2(inv, inv), p2 = make_float2(p, p);
        float q[8], e[8];
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            const float2 t = mul_f32x2(make_float2(v[j], v[j + 1]), inv2);
            q[j] = t.x;
            q[j + 1] = t.y;
        }
        e2m1x8_decode_raw(e2m1x8_encode_hw(q), e);
#pragma unroll
        for (int j = 0; j < 8; j += 2) {  // exact product, +0.0 for code 8
            const float2 o = fma_f32x2(make_float2(e[j], e[j + 1]), p2, zero2);
            out[j] = o.x;
            out[j + 1] = o.y;
        }
    } else {
        if (g == 0.0f) {
#pragma unroll
            for (int j = 0; j < 8; ++j) out[j] = 0.0f;
        } else {
            const uint32_t sc = nv_scale_code(amax_b, g, rg);
            const float s = e4m3x2_decode_hw(sc).x;
            uint32_t codes;
            const float r = __fmul_rn(tab->inv[sc], rg);
            if (r >= 2.3509887e-38f && r <= 4.2535296e37f) {
                const float2 rlo = make_float2(__fmul_rn(r, 0.99999952f), __fmul_rn(r, 0.99999952f));
                const float2 rhi = make_float2(__fmul_rn(r, 1.00000048f), __fmul_rn(r, 1.00000048f));
                float lo[8], hi[8];
#pragma unroll
                for (int j = 0; j < 8; j += 2) {
                    const float2 a = mul_f32x2(make_float2(v[j], v[j + 1]), rlo);
                    const float2 b = mul_f32x2(make_float2(v[j], v[j + 1]), rhi);
                    lo[j] = a.x; lo[j + 1] = a.y;
                    hi[j] = b.x; hi[j + 1] = b.y;
                }
                codes = e2m1x8_encode_hw(lo);
                const uint32_t diff = codes ^ e2m1x8_encode_hw(hi);
                if (diff) codes = nv_settle_straddles_regs(codes, diff, v, __fmul_rn(s, g), tab->bounds);
            } else {
                codes = e2m1x8_of_quotient(v, __fmul_rn(s, g));
            }
            float e[8];
            e2m1x8_decode_raw(codes, e);
            // (e2m1 * s) is exact, then one rounding by g (+0.0 for code 8)
            const float2 s2 = make_float2(s, s), g2 = make_float2(g, g);
#pragma unroll
            for (int j = 0; j < 8; j += 2) {
                const float2 o = fma_f32x2(mul_f32x2(make_float2(e[j], e[j + 1]), s2), g2, zero2);
                out[j] = o.x;
                out[j + 1] = o.y;
            }
        }
    }
}

// FP8 / MXFP4 fake-quant when every row is a whole number of blocks and
// 16-byte aligned: the blocks tile the flat tensor, so this is a flat stream
// with U chunks in flight per lane.  Bounded to 32 registers so that 8 CTAs
// fit on an SM: the tensors of this path are 8-70 MB, and at that size more
// resident warps (more loads in flight at the start) beat more chunks per
// lane.
template <typename T, int FMT, int BLOCK, int U>
__global__ void __launch_bounds__(kThreads, 8) cache_flat_kernel(const T* __restrict__ x, T* __restrict__ y,
                                                              int64_t nchunks) {
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
            float v[8], out[8];
            raw[u].get(v);
            cache_chunk<FMT, L>(v, 0.0f, 0.0f, nullptr, out);
            if (c < nchunks && BSQ_DOK(c * 8 + 8 <= nchunks * 8)) store8(y + c * 8, out);
        }
    }
}

// Row-resident fake-quant: S lanes per row, every lane loads its (at most
// NCH) chunks of the zero-padded row before any arithmetic; NVFP4 reduces
// the row amax over the S lanes.  Handles partial groups and ragged C.
// With 16-byte rows (VEC) the first row's words are requested before the
// per-CTA tables are filled, and (when the double buffer is small) the next
// row's words before the current row is coded, so a warp's rows do not each
// wait for a DRAM round trip.
template <typename T, int FMT, int BLOCK, int S, bool VEC, int NCH>
__global__ void __launch_bounds__(kThreads) cache_row_kernel(const T* __restrict__ x, T* __restrict__ y,
                                                             int64_t rows, int64_t C) {
    constexpr int L = BLOCK / 8;
    constexpr int RPW = 32 / S;
    constexpr bool PF = VEC && NCH * sizeof(T) <= 4;  // prefetch the next row (at most 16 registers of words)
    __shared__ NvTables tab;
    const int lane = threadIdx.x & 31;
    const int sl = lane % S;
    const int64_t cpr = ((C + BLOCK - 1) / BLOCK) * L;
    const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
    const int64_t wid = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    const int64_t step = warps * RPW;
    // the words of this lane's chunks of the row starting at r0 (zeros past
    // the row, the padding and the last row)
    auto load_row = [&](Raw8<T>* w, int64_t r0) {
        const int64_t r = r0 + lane / S;
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            const int64_t c = sl + (int64_t)i * S;
            if (r < rows && c < cpr && C - c * 8 > 0) w[i].load_cs(x + r * C + c * 8);
            else w[i].zero();
        }
    };
    Raw8<T> cur[NCH], nxt[NCH];
    const int64_t first = wid * RPW;
    if (VEC) load_row(cur, first);
    if (FMT == BSQ_NVFP4) {
        fill_nv_tables(&tab);
        __syncthreads();
    }
    for (int64_t r0 = first; r0 < rows; r0 += step) {
        if (PF && r0 + step < rows) load_row(nxt, r0 + step);
        if (VEC && !PF && r0 != first) load_row(cur, r0);
        const int64_t r = r0 + lane / S;
        const bool row_ok = r < rows;
        const T* xr = x + (row_ok ? r : 0) * C;
        T* yr = y + (row_ok ? r : 0) * C;
        float v[NCH][8];
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            if (VEC) {
                cur[i].get(v[i]);  // zeros where nothing was loaded
            } else {
                const int64_t c = sl + (int64_t)i * S;
                const int64_t n = C - c * 8;
                if (row_ok && c < cpr && n > 0) {
                    load_n(xr + c * 8, (int)(n < 8 ? n : 8), v[i]);
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) v[i][j] = 0.0f;
                }
            }
            m = fmaxf(m, amax8(v[i]));
        }
        float g = 0.0f, rg = 0.0f;
        if (FMT == BSQ_NVFP4) {
            g = __fdiv_rn(S == 32 ? warp_max_nonneg(m) : group_max<S>(m), kNvGlobalDiv);
            rg = nv_recip_or_zero(g);
        }
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            if (i * S >= cpr) break;  // uniform across the warp
            const int64_t c = sl + (int64_t)i * S;
            const int64_t n = C - c * 8;
            float out[8];
            cache_chunk<FMT, L>(v[i], g, rg, &tab, out);
            if (row_ok && c < cpr && n > 0) {
                if (BSQ_DOK(r < rows && c * 8 < C)) {
                    if (VEC && n >= 8) store8(yr + c * 8, out);
                    else store_n(yr + c * 8, (int)(n < 8 ? n : 8), out);
                }
            }
        }
        if (PF) {
#pragma unroll
            for (int i = 0; i < NCH; ++i) cur[i] = nxt[i];
        }
    }
}

}  // namespace bsq

using namespace bsq;

template <typename T, int FMT, int BLOCK, bool VEC, int S>
static void launch_cache_rows(const T* x, T* y, int64_t rows, int64_t C, int nch, cudaStream_t st) {
    const int64_t rpw = 32 / S;
    const int64_t warps = (rows + rpw - 1) / rpw;
    const int64_t ctas = (warps + kThreads / 32 - 1) / (kThreads / 32);
    if (nch <= 1) launch_fit_ctas<cache_row_kernel<T, FMT, BLOCK, S, VEC, 1>>(ctas, st, x, y, rows, C);
    else if (nch <= 2) launch_fit_ctas<cache_row_kernel<T, FMT, BLOCK, S, VEC, 2>>(ctas, st, x, y, rows, C);
    else if (nch <= 3) launch_fit_ctas<cache_row_kernel<T, FMT, BLOCK, S, VEC, 3>>(ctas, st, x, y, rows, C);
    else if (nch <= 4) launch_fit_ctas<cache_row_kernel<T, FMT, BLOCK, S, VEC, 4>>(ctas, st, x, y, rows, C);
    else launch_fit_ctas<cache_kernel<T, FMT, BLOCK, S, VEC>>(ctas, st, x, y, rows, C);
}

template <typename T, int FMT, int BLOCK, bool VEC>
static void launch_cache_s(const T* x, T* y, int64_t rows, int64_t C, cudaStream_t st) {
    const int64_t cpr = ((C + BLOCK - 1) / BLOCK) * (BLOCK / 8);
    if (FMT != BSQ_NVFP4 && VEC && C % BLOCK == 0) {
        const int64_t nchunks = rows * C / 8;
        launch_fit<cache_flat_kernel<T, FMT, BLOCK, 2>>(nchunks, 2, st, x, y, nchunks);
        return;
    }
    int S = 2;
    while (S < 32 && S < cpr) S <<= 1;
    if (S < BLOCK / 8) S = BLOCK / 8;
    const int nch = (int)((cpr + S - 1) / S);
    switch (S) {
        case 2: launch_cache_rows<T, FMT, BLOCK, VEC, 2>(x, y, rows, C, nch, st); break;
        case 4: launch_cache_rows<T, FMT, BLOCK, VEC, 4>(x, y, rows, C, nch, st); break;
        case 8: launch_cache_rows<T, FMT, BLOCK, VEC, 8>(x, y, rows, C, nch, st); break;
        case 16: launch_cache_rows<T, FMT, BLOCK, VEC, 16>(x, y, rows, C, nch, st); break;
        default: launch_cache_rows<T, FMT, BLOCK, VEC, 32>(x, y, rows, C, nch, st); break;
    }
}

template <typename T, int FMT>
static void launch_cache_b(int block, const T* x, T* y, int64_t rows, int64_t C, bool vec, cudaStream_t st) {
    if (block == 16) {
        if (vec) launch_cache_s<T, FMT, 16, true>(x, y, rows, C, st);
        else launch_cache_s<T, FMT, 16, false>(x, y, rows, C, st);
    } else {
        if (vec) launch_cache_s<T, FMT, 32, true>(x, y, rows, C, st);
        else launch_cache_s<T, FMT, 32, false>(x, y, rows, C, st);
    }
}

template <typename T>
static void launch_cache(bsq_format fmt, int block, const T* x, T* y, int64_t rows, int64_t C, bool vec,
                         cudaStream_t st) {
    if (fmt == BSQ_FP8) launch_cache_b<T, BSQ_FP8>(block, x, y, rows, C, vec, st);
    else if (fmt == BSQ_MXFP4) launch_cache_b<T, BSQ_MXFP4>(block, x, y, rows, C, vec, st);
    else launch_cache_b<T, BSQ_NVFP4>(block, x, y, rows, C, vec, st);
}

BSQ_API bsq_status bsq_quantize_cache(bsq_format fmt, int block, const void* x, void* y, bsq_dtype t, int64_t rows,
                                      int64_t C, bsq_stream_t stream) {
    BSQ_TRY(check_dtype(t));
    if (fmt != BSQ_FP8 && fmt != BSQ_MXFP4 && fmt != BSQ_NVFP4)
        return fail(BSQ_ERR_UNSUPPORTED, "bsq_quantize_cache: format %d not supported", (int)fmt);
    if (block != 16 && block != 32) return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_cache: block must be 16 or 32");
    if (rows < 0 || C < 0) return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_cache: negative size");
    if (rows * C == 0) return BSQ_OK;
    if (!x || !y) return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_cache: null pointer");
    const size_t es = (t == BSQ_BF16) ? 2 : 4;
    const char* xb = (const char*)x;
    const char* yb = (const char*)y;
    const size_t bytes = (size_t)(rows * C) * es;
    if (xb < yb + bytes && yb < xb + bytes) return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_cache: x and y overlap");
    const bool vec = aligned(x, 16) && aligned(y, 16) && ((C * (int64_t)es) % 16 == 0) && (C % 8 == 0);
    cudaStream_t st = (cudaStream_t)stream;
    if (t == BSQ_BF16) launch_cache(fmt, block, (const uint16_t*)x, (uint16_t*)y, rows, C, vec, st);
    else launch_cache(fmt, block, (const float*)x, (float*)y, rows, C, vec, st);
    return check_launch("bsq_quantize_cache");
}

BSQ_API bsq_status bsq_quantize_cache_backward(const void* grad_out, void* grad_in, bsq_dtype t, int64_t n_elems,
                                               bsq_stream_t stream) {
    BSQ_TRY(check_dtype(t));
    if (n_elems < 0) return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_cache_backward: negative size");
    if (n_elems == 0 || grad_in == grad_out) return BSQ_OK;
    if (!grad_out || !grad_in) return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_cache_backward: null pointer");
    const size_t bytes = (size_t)n_elems * (t == BSQ_BF16 ? 2 : 4);
    cudaError_t e = cudaMemcpyAsync(grad_in, grad_out, bytes, cudaMemcpyDeviceToDevice, (cudaStream_t)stream);
    if (e != cudaSuccess) return fail(BSQ_ERR_CUDA, "bsq_quantize_cache_backward: %s", cudaGetErrorString(e));
    return BSQ_OK;
}

#ifdef BSQ_DEBUG
cudaError_t bsq_dbg_take_cache(uint32_t* count, uint32_t* first) { return bsq::dbg_take(count, first); }
#endif
