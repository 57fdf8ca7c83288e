// nvfp4.cu -- NVFP4 quantize: per-row scale, given row scales, ModelOpt tensor scale.
//
// Formulas: nvfp4 page quantize_nvfp4 / quantize_nvfp4_modelopt (ModelOpt
// convention global = amax / (6 * 448), block_scale = e4m3(amax_b / 6 /
// global) floored at 2**-9, code = round_to_e2m1(w / (block_scale *
// global))).  One lane per 16-element block; the e4m3 scale and the e2m1
// codes are bit-exact with mostly no division (see common.cuh).
#include <cstdarg>
#include <cstring>
#include <mutex>

#define BSQ_DBG_FILE 2
#include "debug.cuh"
#include "common.cuh"
#include "tcgen05.cuh"

namespace bsq {

// One CTA per row for the per-row amax rule.
constexpr int kRowThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kRowThreads) nv_rowamax_quant_kernel(const T* __restrict__ x, int64_t rows, int64_t K,
                                                                    uint8_t* __restrict__ packed,
                                                                    uint8_t* __restrict__ scales,
                                                                    float* __restrict__ g_out) {
    // One CTA per row (grid-stride).  Pass 1 streams the row from HBM with
    // plain cached loads (four blocks in flight per thread) and reduces its
    // amax; pass 2 reads the same row again -- it is still in L2, only the
    // rows of the CTAs in flight (a few tens of MB) are live -- and quantizes
    // one 16-element block per thread.
    __shared__ float red[32];
    const int64_t bpr = K / 16;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const T* xr = x + r * K;
        float m = 0.0f;
        for (int64_t b0 = 0; b0 < bpr; b0 += 4 * kRowThreads) {
            float v[4][16];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t blk = b0 + u * kRowThreads + threadIdx.x;
                if (blk < bpr) load16(xr + blk * 16, v[u]);
                else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[u][j] = 0.0f;
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) m = fmaxf(m, fmaxf(amax8(v[u]), amax8(v[u] + 8)));
        }
        const float g = __fdiv_rn(block_reduce_max(m, red), kNvGlobalDiv);
        if (threadIdx.x == 0) g_out[r] = g;
        const float rg = nv_recip_or_zero(g);
        for (int64_t blk = threadIdx.x; blk < bpr; blk += kRowThreads) {
            float v[16];
            load16(xr + blk * 16, v);
            uint32_t sb;
            const uint2 pk = nv_quant_block(v, g, rg, &sb);
            if (BSQ_DOK(r < rows && blk < bpr)) {
                reinterpret_cast<uint2*>(packed + r * (K / 2))[blk] = pk;
                scales[r * bpr + blk] = (uint8_t)sb;
            }
        }
    }
}

// Row amax for rows too long to keep in registers: pass 1 of the per-row rule.
template <typename T>
__global__ void __launch_bounds__(kThreads) row_amax_kernel(const T* __restrict__ x, int64_t rows, int64_t K,
                                                            float* __restrict__ g_out) {
    __shared__ float red[32];
    const int64_t cpr = K / 8;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        float m = 0.0f;
        for (int64_t c = threadIdx.x; c < cpr; c += kThreads) {
            float v[8];
            load8(x + r * K + c * 8, v);
            m = fmaxf(m, amax8(v));
        }
        const float amax = block_reduce_max(m, red);
        if (threadIdx.x == 0) g_out[r] = __fdiv_rn(amax, kNvGlobalDiv);
    }
}

// Tensor amax, pass 1 of the ModelOpt layout: one partial maximum per CTA.
template <typename T, int U>
__global__ void __launch_bounds__(kThreads) amax_partial_kernel(const T* __restrict__ x, int64_t nchunks,
                                                                float* __restrict__ partial) {
    __shared__ float red[32];
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    float m = 0.0f;
    for (int64_t base = (int64_t)blockIdx.x * kThreads + threadIdx.x; base < nchunks; base += U * stride) {
        float v[U][8];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t c = base + u * stride;
            if (c < nchunks) load8(x + c * 8, v[u]);
            else {
#pragma unroll
                for (int j = 0; j < 8; ++j) v[u][j] = 0.0f;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) m = fmaxf(m, amax8(v[u]));
    }
    const float r = block_reduce_max(m, red);
    if (threadIdx.x == 0) partial[blockIdx.x] = r;
}

// Flat NVFP4 quantization with a known row scale, one lane per 16-element
// block: MODE 0 = per-row scales given in g_in (copied to g_out), MODE 1 =
// tensor scale from the partial maxima (reduced by every CTA; CTA 0 publishes
// it), MODE 2 = per-row scales computed by row_amax_kernel into g_out.
template <typename T, int MODE, int U>
__global__ void __launch_bounds__(kThreads) nv_flat_quant_kernel(const T* __restrict__ x, int64_t nblocks, FastDiv bpr,
                                                                 const float* __restrict__ g_in,
                                                                 const float* __restrict__ partial, int npartial,
                                                                 uint8_t* __restrict__ packed,
                                                                 uint8_t* __restrict__ scales,
                                                                 float* __restrict__ g_out) {
    __shared__ float red[32];
    float g_tensor = 0.0f, rg_tensor = 0.0f;
    if (MODE == 1) {
        float m = 0.0f;
        for (int i = threadIdx.x; i < npartial; i += kThreads) m = fmaxf(m, partial[i]);
        g_tensor = __fdiv_rn(block_reduce_max(m, red), kNvGlobalDiv);
        rg_tensor = nv_recip_or_zero(g_tensor);
        if (blockIdx.x == 0 && threadIdx.x == 0) g_out[0] = g_tensor;
    }
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t base = (int64_t)blockIdx.x * kThreads + threadIdx.x; base < nblocks; base += U * stride) {
        float v[U][16];
        float g[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t b = base + u * stride;
            g[u] = g_tensor;
            if (b < nblocks) {
                load16(x + b * 16, v[u]);
                if (MODE != 1) g[u] = (MODE == 0 ? g_in : g_out)[fdiv((uint32_t)b, bpr)];
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t b = base + u * stride;
            if (b >= nblocks) continue;
            uint32_t sb;
            const float rg = (MODE == 1) ? rg_tensor : nv_recip_or_zero(g[u]);
            const uint2 pk = nv_quant_block(v[u], g[u], rg, &sb);
            if (!BSQ_DOK(b < nblocks)) continue;
            reinterpret_cast<uint2*>(packed)[b] = pk;
            scales[b] = (uint8_t)sb;
            if (MODE == 0) {
                const uint32_t row = fdiv((uint32_t)b, bpr);
                if ((uint32_t)b == row * bpr.d && BSQ_DOK((int64_t)row * bpr.d < nblocks)) g_out[row] = g[u];
            }
        }
    }
}

// ------------------------------------------- rows staged in shared memory
//
// One CTA per row (persistent over the rows blockIdx.x + i * gridDim.x).
// Thread t owns the 16-element blocks t, t + nt, ... (at most kStgMaxBpt) of
// every row: it copies them into shared memory itself with cp.async, S - 1
// rows ahead, so the HBM stream runs while earlier rows are computed, and it
// reads back only its own blocks, so stages are reused without waiting for
// the other threads.  A first sweep takes the blocks' amaxes; MODE 2 reduces
// the row amax across the CTA (the kernel's only per-row barrier; per-warp
// slots alternate by row parity).  A second sweep forms the codes without a
// division:
//  - bf16 rows: every quotient correctly rounded by one fma correction
//    (nv_block_codes_bf16), the same work for every element, so the warp
//    never diverges on the data;
//  - fp32 rows: the bracket codes, and an element whose brackets disagree
//    settled in place by an exact fma test (nv_block_codes_fast).  With a
//    scale tied to the data (a row or tensor amax / 2688) a few percent of
//    the blocks hold such an element (one with the same significand as the
//    amax, for instance).
// MODE 0 takes g from g_in, MODE 1 the tensor scale from the partial maxima,
// MODE 2 the row's own amax / 2688.  NT is the launch's maximum thread count,
// MINB the CTAs per SM the register budget is sized for.
constexpr int kStgMaxThreads = 512, kStgMaxBpt = 4;
// blocks per thread the launch plan aims for (at most kStgMaxBpt)
#ifndef BSQ_STG_BPT
#define BSQ_STG_BPT 4
#endif
static_assert(BSQ_STG_BPT >= 1 && BSQ_STG_BPT <= kStgMaxBpt, "blocks per thread of the staged kernel");

template <typename T, int MODE, int S, int NT, int MINB>
__global__ void __launch_bounds__(NT, MINB)
    nv_row_staged_kernel(const T* __restrict__ x, int64_t rows, int K, const float* __restrict__ g_in,
                         const float* __restrict__ partial, int npartial, uint8_t* __restrict__ packed,
                         uint8_t* __restrict__ scales, float* __restrict__ g_out) {
    extern __shared__ __align__(128) uint8_t stage_mem[];
    __shared__ float red[2][NT / 32];
    __shared__ float inv_tab[128];
    __shared__ NvBound bounds[8];
    constexpr int kCopies = (int)sizeof(T);  // 16-byte copies per block: 2 (bf16) or 4 (fp32)
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
    const int bpr = K / 16;
    const uint32_t stage_bytes = ((uint32_t)K * (uint32_t)sizeof(T) + 127u) & ~127u;
    constexpr bool kBf16 = sizeof(T) == 2;  // bf16: correctly rounded quotients; fp32: brackets
    if (!kBf16) {
        fill_inv_e4m3(inv_tab);
        fill_nv_bounds(bounds);
    }
    float g_t = 0.0f, rg_t = 0.0f;
    if (MODE == 1) {
        float m = 0.0f;
        for (int i = tid; i < npartial; i += nt) m = fmaxf(m, partial[i]);
        m = warp_max_nonneg(m);
        if (lane == 0) red[0][warp] = m;
    }
    __syncthreads();
    if (MODE == 1) {
        const float m = warp_max_nonneg(lane < nw ? red[0][lane] : 0.0f);
        g_t = __fdiv_rn(m, kNvGlobalDiv);
        rg_t = nv_recip_or_zero(g_t);
        if (blockIdx.x == 0 && tid == 0) g_out[0] = g_t;
        __syncthreads();  // red[0] is reused by the rows below
    }
    const int64_t first = blockIdx.x, step = gridDim.x;
    const int64_t my_rows = (first < rows) ? (rows - 1 - first) / step + 1 : 0;
    // this thread's blocks: byte offsets within a row (32-bit), and how many
    constexpr uint32_t kBlkBytes = 16u * (uint32_t)sizeof(T);
    const uint32_t smem0 = (uint32_t)__cvta_generic_to_shared(stage_mem);
    const int myb = (bpr > tid) ? min(kStgMaxBpt, (bpr - 1 - tid) / nt + 1) : 0;
    auto issue = [&](int64_t i) {
        if (i < my_rows) {
            const uint8_t* src = reinterpret_cast<const uint8_t*>(x + (first + i * step) * (int64_t)K);
            const uint32_t dst = smem0 + (uint32_t)(i % S) * stage_bytes;
#pragma unroll
            for (int j = 0; j < kStgMaxBpt; ++j) {
                if (j < myb) {
                    const uint32_t off = (uint32_t)(tid + j * nt) * kBlkBytes;
#pragma unroll
                    for (int c = 0; c < kCopies; ++c)
                        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + off + 16u * c),
                                     "l"(src + off + 16u * c)
                                     : "memory");
                }
            }
        }
        cp_async_commit();  // one group per row, empty past the last row
    };
#pragma unroll
    for (int i = 0; i < S - 1; ++i) issue(i);
    for (int64_t i = 0; i < my_rows; ++i) {
        const int64_t r = first + i * step;
        issue(i + S - 1);        // into the stage of row i - 1, which this thread has finished
        cp_async_wait<S - 1>();  // this thread's copies of row i have landed
        const uint32_t xs = smem0 + (uint32_t)(i % S) * stage_bytes;  // shared address of row i
        float am[kStgMaxBpt];
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < kStgMaxBpt; ++j) {
            am[j] = 0.0f;
            if (j < myb) {
                Raw16<T> raw;
                raw.load_smem(xs + (uint32_t)(tid + j * nt) * kBlkBytes);
                am[j] = raw.amax();
                m = fmaxf(m, am[j]);
            }
        }
        float g;
        if (MODE == 2) {
            m = warp_max_nonneg(m);
            if (lane == 0) red[i & 1][warp] = m;
            __syncthreads();
            const float mm = warp_max_nonneg(lane < nw ? red[i & 1][lane] : 0.0f);
            g = __fdiv_rn(mm, kNvGlobalDiv);
        } else if (MODE == 0) {
            g = BSQ_DOK(r < rows) ? g_in[r] : 0.0f;
        } else {
            g = g_t;
        }
        if (MODE != 1 && tid == 0 && BSQ_DOK(r < rows)) g_out[r] = g;
        const float rg = (MODE == 1) ? rg_t : nv_recip_or_zero(g);
        uint8_t* prow = packed + r * (int64_t)(K / 2);
        uint8_t* srow = scales + r * (int64_t)bpr;
        uint32_t redo_self = 0u;
#pragma unroll
        for (int j = 0; j < kStgMaxBpt; ++j) {
            if (j < myb && BSQ_DOK(tid + j * nt < bpr && (uint32_t)(tid + j * nt + 1) * kBlkBytes <= stage_bytes)) {
                const int b = tid + j * nt;
                const uint32_t blk = xs + (uint32_t)b * kBlkBytes;
                uint32_t sb = 0u;
                uint2 pk = make_uint2(0u, 0u);
                if (g != 0.0f) {
                    Raw16<T> raw;
                    raw.load_smem(blk);
                    sb = nv_scale_code(am[j], g, rg);
                    bool ok;
                    if constexpr (kBf16) ok = nv_block_codes_bf16(raw, am[j], sb, g, &pk);
                    else ok = nv_block_codes_fast<T>(raw, blk, sb, g, rg, inv_tab, bounds, &pk);
                    if (!ok) redo_self |= 1u << j;
                }
                reinterpret_cast<uint2*>(prow)[b] = pk;
                srow[b] = (uint8_t)sb;
            }
        }
        while (redo_self) {  // r out of range (g near the ends of the binary32 range)
            const int j = __ffs(redo_self) - 1;
            redo_self &= redo_self - 1u;
            const int b = tid + j * nt;
            Raw16<T> raw;
            raw.load_smem(xs + (uint32_t)b * kBlkBytes);
            reinterpret_cast<uint2*>(prow)[b] = nv_block_codes_slow<T>(raw, g, nv_scale_code(am[j], g, rg));
        }
    }
    cp_async_wait<0>();
}

}  // namespace bsq

using namespace bsq;

// Staged-row launch plan for rows of K elements of T: threads per CTA (a
// multiple of 32, at most kStgMaxBpt blocks each), stages of the ring and the
// register-budget variant: up to 384 threads run three CTAs of two stages per
// SM (56 registers a thread) when their stages fit, otherwise two CTAs of
// three (or two) stages (64 registers).  nt = 0: the row does not fit.
struct StagedPlan {
    int nt = 0, stages = 0;
    bool three = false;
    size_t smem = 0;
};

template <typename T>
static StagedPlan staged_plan(int64_t K) {
    StagedPlan p;
    const int64_t bpr = K / 16;
    const int64_t row_bytes = K * (int64_t)sizeof(T);
    if (bpr < 1 || bpr > (int64_t)kStgMaxThreads * kStgMaxBpt || row_bytes > 100 * 1024) return p;
    const int64_t stage_bytes = (row_bytes + 127) / 128 * 128;
    // as many blocks per thread as allowed (the per-row work of a thread is
    // shared by more blocks), but at least 64 threads
    const int bpt = (int)std::max<int64_t>(1, std::min<int64_t>(BSQ_STG_BPT, bpr / 64));
    const int64_t per = (bpr + bpt - 1) / bpt;
    p.nt = (int)((per + 31) / 32 * 32);
    if (p.nt > kStgMaxThreads) return StagedPlan();
    // per CTA: the stages, under 1 KiB of static shared memory and 1 KiB the
    // hardware reserves, against the 228 KiB of an SM
    if (p.nt <= 384 && 3 * (2 * stage_bytes + 4 * 1024) <= 228 * 1024) {
        p.three = true;
        p.stages = 2;
    } else {
        p.stages = (3 * stage_bytes <= 110 * 1024) ? 3 : 2;
    }
    p.smem = (size_t)(p.stages * stage_bytes);
    return p;
}

template <typename T, int MODE, int S, int NT, int MINB>
static bsq_status launch_staged_v(const StagedPlan& p, const T* x, int64_t rows, int64_t K, const float* g_in,
                                  const float* partial, int npartial, uint8_t* packed, uint8_t* scales, float* g_out,
                                  cudaStream_t st, const char* fn) {
    static std::mutex mu;
    static size_t opted[64] = {0};
    auto kern = nv_row_staged_kernel<T, MODE, S, NT, MINB>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (opted[dev] < p.smem) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
            if (e != cudaSuccess) return fail(BSQ_ERR_CUDA, "%s: shared-memory opt-in failed (%s)", fn, cudaGetErrorString(e));
            opted[dev] = p.smem;
        }
    }
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, p.nt, p.smem) != cudaSuccess || per_sm < 1) {
        cudaGetLastError();
        per_sm = 1;
    }
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(rows, (int64_t)sm_count() * per_sm));
    kern<<<grid, p.nt, p.smem, st>>>(x, rows, (int)K, g_in, partial, npartial, packed, scales, g_out);
    return check_launch(fn);
}

template <typename T, int MODE>
static bsq_status launch_staged(const StagedPlan& p, const T* x, int64_t rows, int64_t K, const float* g_in,
                                const float* partial, int npartial, uint8_t* packed, uint8_t* scales, float* g_out,
                                cudaStream_t st, const char* fn) {
    if (p.three)
        return launch_staged_v<T, MODE, 2, 384, 3>(p, x, rows, K, g_in, partial, npartial, packed, scales, g_out, st, fn);
    if (p.stages == 3)
        return launch_staged_v<T, MODE, 3, kStgMaxThreads, 2>(p, x, rows, K, g_in, partial, npartial, packed, scales,
                                                               g_out, st, fn);
    return launch_staged_v<T, MODE, 2, kStgMaxThreads, 2>(p, x, rows, K, g_in, partial, npartial, packed, scales,
                                                           g_out, st, fn);
}

// Second pass of the ModelOpt layout: quantize with the tensor scale reduced
// from the P partial maxima (staged rows where they fit, else flat blocks).
template <typename T>
static bsq_status launch_tensor_quant(const T* x, int64_t rows, int64_t K, const float* partial, int P,
                                      uint8_t* packed, uint8_t* scales, float* tensor_scale_out, cudaStream_t st,
                                      const char* fn) {
    const StagedPlan sp = staged_plan<T>(K);
    if (sp.nt) return launch_staged<T, 1>(sp, x, rows, K, nullptr, partial, P, packed, scales, tensor_scale_out, st, fn);
    const int64_t nblocks = rows * (K / 16);
    launch_fit<nv_flat_quant_kernel<T, 1, 2>>(nblocks, 2, st, x, nblocks, make_fastdiv((uint32_t)(K / 16)),
                                              (const float*)nullptr, partial, P, packed, scales, tensor_scale_out);
    return check_launch(fn);
}

template <typename T>
static bsq_status launch_nv_rowamax(const T* x, int64_t rows, int64_t K, uint8_t* packed, uint8_t* scales,
                                    float* g_out, cudaStream_t st) {
    const int64_t cpr = K / 8;
    const StagedPlan sp = staged_plan<T>(K);
    if (sp.nt) return launch_staged<T, 2>(sp, x, rows, K, nullptr, nullptr, 0, packed, scales, g_out, st,
                                          "bsq_quantize_nvfp4");
    if (K <= 65536) {
        static_assert(kRowThreads == kThreads, "row kernel launched with the common block size");
        launch_fit_ctas<nv_rowamax_quant_kernel<T>>(rows, st, x, rows, K, packed, scales, g_out);
        return check_launch("bsq_quantize_nvfp4");
    }
    // long rows: amax pass, then the flat pass with the computed row scales
    launch_fit_ctas<row_amax_kernel<T>>(rows, st, x, rows, K, g_out);
    BSQ_TRY(check_launch("bsq_quantize_nvfp4"));
    (void)cpr;
    const int64_t nblocks = rows * (K / 16);
    const float* none = nullptr;
    launch_fit<nv_flat_quant_kernel<T, 2, 2>>(nblocks, 2, st, x, nblocks, make_fastdiv((uint32_t)(K / 16)), none, none,
                                              0, packed, scales, g_out);
    return check_launch("bsq_quantize_nvfp4");
}

BSQ_API bsq_status bsq_quantize_nvfp4(const void* x, bsq_dtype xt, int64_t rows, int64_t K,
                                      const float* row_scale_in, uint8_t* packed, uint8_t* scales_e4m3,
                                      float* row_scale_out, bsq_stream_t stream) {
    BSQ_TRY(check_dtype(xt));
    BSQ_TRY(check_matrix("bsq_quantize_nvfp4", x, rows, K, 16));
    if (rows * K == 0) return BSQ_OK;
    if (!packed || !scales_e4m3 || !row_scale_out) return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_nvfp4: null output");
    if (!aligned(x, 16) || !aligned(packed, 8)) return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_nvfp4: misaligned pointer");
    cudaStream_t st = (cudaStream_t)stream;
    if (row_scale_in) {
        if (xt == BSQ_BF16) {
            const StagedPlan sp = staged_plan<uint16_t>(K);
            if (sp.nt)
                return launch_staged<uint16_t, 0>(sp, (const uint16_t*)x, rows, K, row_scale_in, nullptr, 0, packed,
                                                  scales_e4m3, row_scale_out, st, "bsq_quantize_nvfp4");
        } else {
            const StagedPlan sp = staged_plan<float>(K);
            if (sp.nt)
                return launch_staged<float, 0>(sp, (const float*)x, rows, K, row_scale_in, nullptr, 0, packed,
                                               scales_e4m3, row_scale_out, st, "bsq_quantize_nvfp4");
        }
        const int64_t nblocks = rows * (K / 16);
        const FastDiv bpr = make_fastdiv((uint32_t)(K / 16));
        if (xt == BSQ_BF16)
            launch_fit<nv_flat_quant_kernel<uint16_t, 0, 2>>(nblocks, 2, st, (const uint16_t*)x, nblocks, bpr, row_scale_in,
                                                             (const float*)nullptr, 0, packed, scales_e4m3, row_scale_out);
        else
            launch_fit<nv_flat_quant_kernel<float, 0, 2>>(nblocks, 2, st, (const float*)x, nblocks, bpr, row_scale_in,
                                                          (const float*)nullptr, 0, packed, scales_e4m3, row_scale_out);
        return check_launch("bsq_quantize_nvfp4");
    }
    if (xt == BSQ_BF16) return launch_nv_rowamax((const uint16_t*)x, rows, K, packed, scales_e4m3, row_scale_out, st);
    return launch_nv_rowamax((const float*)x, rows, K, packed, scales_e4m3, row_scale_out, st);
}

static int tensor_partials(int64_t rows, int64_t K) {
    const int64_t nchunks = rows * (K / 8);
    return grid_for(nchunks, 4);
}

BSQ_API size_t bsq_nvfp4_tensor_scratch_bytes(int64_t rows, int64_t K) {
    if (rows <= 0 || K <= 0) return 16;
    return (size_t)((tensor_partials(rows, K) * sizeof(float) + 15) / 16 * 16);
}

BSQ_API bsq_status bsq_quantize_nvfp4_tensor(const void* x, bsq_dtype xt, int64_t rows, int64_t K, uint8_t* packed,
                                             uint8_t* scales_e4m3, float* tensor_scale_out, void* scratch,
                                             size_t scratch_bytes, bsq_stream_t stream) {
    BSQ_TRY(check_dtype(xt));
    BSQ_TRY(check_matrix("bsq_quantize_nvfp4_tensor", x, rows, K, 16));
    if (!tensor_scale_out) return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_nvfp4_tensor: null tensor scale");
    cudaStream_t st = (cudaStream_t)stream;
    if (rows * K == 0) {
        if (cudaMemsetAsync(tensor_scale_out, 0, sizeof(float), st) != cudaSuccess)
            return check_launch("bsq_quantize_nvfp4_tensor");
        return BSQ_OK;
    }
    if (!packed || !scales_e4m3 || !scratch) return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_nvfp4_tensor: null pointer");
    if (!aligned(x, 16) || !aligned(packed, 8) || !aligned(scratch, 16))
        return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_nvfp4_tensor: misaligned pointer");
    const int P = tensor_partials(rows, K);
    if (scratch_bytes < (size_t)P * sizeof(float))
        return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_nvfp4_tensor: scratch of %zu bytes, need %zu", scratch_bytes,
                    (size_t)P * sizeof(float));
    const int64_t nchunks = rows * (K / 8);
    float* partial = (float*)scratch;
    if (xt == BSQ_BF16) {
        amax_partial_kernel<uint16_t, 4><<<P, kThreads, 0, st>>>((const uint16_t*)x, nchunks, partial);
        BSQ_TRY(check_launch("bsq_quantize_nvfp4_tensor"));
        return launch_tensor_quant((const uint16_t*)x, rows, K, partial, P, packed, scales_e4m3, tensor_scale_out, st,
                                   "bsq_quantize_nvfp4_tensor");
    }
    amax_partial_kernel<float, 4><<<P, kThreads, 0, st>>>((const float*)x, nchunks, partial);
    BSQ_TRY(check_launch("bsq_quantize_nvfp4_tensor"));
    return launch_tensor_quant((const float*)x, rows, K, partial, P, packed, scales_e4m3, tensor_scale_out, st,
                               "bsq_quantize_nvfp4_tensor");
}

// ----------------------------------------------- no-allocation variant ----
// Some callers cannot hand the library a scratch buffer: a serving engine that
// reserves all device memory up front and forbids allocations afterwards, or a
// plain C caller with no device allocator of its own.  For them the per-tensor
// NVFP4 quantization can keep its per-CTA partial maxima in this file-scope
// device array instead.  Every GPU that loads the library holds these 16 KiB
// until the process exits.  The partial maxima are fully written by the first
// pass before the second pass reads them, so nothing needs clearing between
// calls.
constexpr int kNoAllocMaxPartials = 4096;
static __device__ __align__(256) float g_noalloc_partials[kNoAllocMaxPartials];

// Device address of g_noalloc_partials, looked up once per device with that
// device current (in host code the array's name is only a host-side handle).
// The address is cached for the life of the process; a device reset, which
// tears down the context the module was loaded in, leaves it stale.
static float* noalloc_partials_ptr(bsq_status* st) {
    static std::mutex mu;
    static float* ptrs[64] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) {
        *st = fail(BSQ_ERR_CUDA, "bsq_quantize_nvfp4_tensor_noalloc: no current device (%s)",
                   cudaGetErrorString(e));
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (ptrs[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_partials);
        if (e != cudaSuccess || p == nullptr) {
            *st = fail(BSQ_ERR_CUDA, "bsq_quantize_nvfp4_tensor_noalloc: cudaGetSymbolAddress failed (%s)",
                       cudaGetErrorString(e));
            return nullptr;
        }
        ptrs[dev] = (float*)p;
    }
    *st = BSQ_OK;
    return ptrs[dev];
}

BSQ_API bsq_status bsq_quantize_nvfp4_tensor_noalloc(const void* x, bsq_dtype xt, int64_t rows, int64_t K,
                                                     uint8_t* packed, uint8_t* scales_e4m3, float* tensor_scale_out,
                                                     bsq_stream_t stream) {
    BSQ_TRY(check_dtype(xt));
    BSQ_TRY(check_matrix("bsq_quantize_nvfp4_tensor_noalloc", x, rows, K, 16));
    if (!tensor_scale_out) return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_nvfp4_tensor_noalloc: null tensor scale");
    cudaStream_t st = (cudaStream_t)stream;
    if (rows * K == 0) {
        if (cudaMemsetAsync(tensor_scale_out, 0, sizeof(float), st) != cudaSuccess)
            return check_launch("bsq_quantize_nvfp4_tensor_noalloc");
        return BSQ_OK;
    }
    if (!packed || !scales_e4m3) return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_nvfp4_tensor_noalloc: null pointer");
    if (!aligned(x, 16) || !aligned(packed, 8))
        return fail(BSQ_ERR_INVALID_ARG, "bsq_quantize_nvfp4_tensor_noalloc: misaligned pointer");
    const int P = tensor_partials(rows, K);
    if (P > kNoAllocMaxPartials)
        return fail(BSQ_ERR_UNSUPPORTED,
                    "bsq_quantize_nvfp4_tensor_noalloc: needs %d partial maxima, the built-in scratch holds %d",
                    P, kNoAllocMaxPartials);
    bsq_status status;
    float* partial = noalloc_partials_ptr(&status);
    if (!partial) return status;
    const int64_t nchunks = rows * (K / 8);
    if (xt == BSQ_BF16) {
        amax_partial_kernel<uint16_t, 4><<<P, kThreads, 0, st>>>((const uint16_t*)x, nchunks, partial);
        BSQ_TRY(check_launch("bsq_quantize_nvfp4_tensor_noalloc"));
        return launch_tensor_quant((const uint16_t*)x, rows, K, partial, P, packed, scales_e4m3, tensor_scale_out, st,
                                   "bsq_quantize_nvfp4_tensor_noalloc");
    }
    amax_partial_kernel<float, 4><<<P, kThreads, 0, st>>>((const float*)x, nchunks, partial);
    BSQ_TRY(check_launch("bsq_quantize_nvfp4_tensor_noalloc"));
    return launch_tensor_quant((const float*)x, rows, K, partial, P, packed, scales_e4m3, tensor_scale_out, st,
                               "bsq_quantize_nvfp4_tensor_noalloc");
}

#ifdef BSQ_DEBUG
cudaError_t bsq_dbg_take_nvfp4(uint32_t* count, uint32_t* first) { return bsq::dbg_take(count, first); }
#endif
