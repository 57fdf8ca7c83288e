// quant.cu -- HBM-bound block quantize / dequantize kernels for sm_100a and
// their C-ABI entry points (NVFP4, MXFP4, FP8 power-of-two, cache fake-quant,
// straight-through backward).
//
// Work unit: a "chunk" of 8 consecutive elements (one 16-byte bf16 vector).
// A 16- or 32-column block spans 2 or 4 adjacent lanes of a warp, so the
// block amax is two or three warp shuffles.  Loads are 128-bit, streaming
// (ld.global.cs); stores are coalesced 4/8/16-byte vectors.  Every grid is a
// multiple of the SM count (grid-stride loops, several chunks in flight per
// thread) so HBM, not issue, is the limiter.
//
// Formulas (NeMo AutoModel API pages):
//   nvfp4 page quantize_nvfp4 / quantize_nvfp4_modelopt / dequantize_nvfp4
//   mxfp4 page quantize_mxfp4 / dequantize_mxfp4
//   deepseek_v41 quantization page quantize_cache / _power_of_two_ceiling /
//   _CacheQuantization.backward
#include <algorithm>
#include <cstdarg>
#include <cstring>
#include <mutex>

#include "formats.cuh"
#include "host_util.h"
#include "tcgen05.cuh"

namespace bsq {

// ------------------------------------------------------------ host helpers --

static thread_local char g_last_error[512] = "";

bsq_status fail(bsq_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return s;
}

bsq_status check_launch(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(BSQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return BSQ_OK;
}

int sm_count() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

static inline bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

// ---------------------------------------------------------- device helpers --

constexpr int kThreads = 256;
constexpr float kE2M1Max = 6.0f;       // nvfp4 page E2M1_MAX
constexpr float kE4M3Max = 448.0f;     // nvfp4 page E4M3_MAX
constexpr float kE4M3MinSub = 0.001953125f;  // nvfp4 page E4M3_MIN_SUBNORMAL = 2**-9
constexpr float kF32MinNormal = 1.17549435e-38f;  // 2**-126
constexpr float kNvGlobalDiv = 2688.0f;  // 6 * 448

template <typename T> struct Elem;
template <> struct Elem<uint16_t> { static constexpr int kBytes = 2; };
template <> struct Elem<float> { static constexpr int kBytes = 4; };

// 8 consecutive elements starting at p (16-byte aligned for bf16, 32 for fp32).
__device__ __forceinline__ void load8(const uint16_t* p, float v[8]) {
    uint4 w = __ldcs(reinterpret_cast<const uint4*>(p));
    v[0] = bf16_lo(w.x); v[1] = bf16_hi(w.x); v[2] = bf16_lo(w.y); v[3] = bf16_hi(w.y);
    v[4] = bf16_lo(w.z); v[5] = bf16_hi(w.z); v[6] = bf16_lo(w.w); v[7] = bf16_hi(w.w);
}
__device__ __forceinline__ void load8(const float* p, float v[8]) {
    float4 a = __ldcs(reinterpret_cast<const float4*>(p));
    float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
// Up to n (< 8) elements with scalar loads, zero fill (ragged rows).
__device__ __forceinline__ void load_n(const uint16_t* p, int n, float v[8]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = (j < n) ? __uint_as_float((uint32_t)p[j] << 16) : 0.0f;
}
__device__ __forceinline__ void load_n(const float* p, int n, float v[8]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = (j < n) ? p[j] : 0.0f;
}

__device__ __forceinline__ void store8(uint16_t* p, const float v[8]) {
    uint4 w;
    w.x = pack_bf16x2(v[0], v[1]); w.y = pack_bf16x2(v[2], v[3]);
    w.z = pack_bf16x2(v[4], v[5]); w.w = pack_bf16x2(v[6], v[7]);
    __stcs(reinterpret_cast<uint4*>(p), w);
}
__device__ __forceinline__ void store8(float* p, const float v[8]) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
    __stcs(reinterpret_cast<float4*>(p) + 1, make_float4(v[4], v[5], v[6], v[7]));
}
__device__ __forceinline__ void store_n(uint16_t* p, int n, const float v[8]) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
        if (j < n) {
            __nv_bfloat16 h = __float2bfloat16_rn(v[j]);
            p[j] = *reinterpret_cast<uint16_t*>(&h);
        }
}
__device__ __forceinline__ void store_n(float* p, int n, const float v[8]) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
        if (j < n) p[j] = v[j];
}

__device__ __forceinline__ float amax8(const float v[8]) {
    float m = fabsf(v[0]);
#pragma unroll
    for (int j = 1; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
    return m;
}

// Max over the `L` adjacent lanes that share a block (L = 1, 2, 4, ...).
template <int L>
__device__ __forceinline__ float group_max(float m) {
#pragma unroll
    for (int o = 1; o < L; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    return m;
}

__device__ __forceinline__ float block_reduce_max(float m, float* smem /* >= 32 floats */) {
    m = group_max<32>(m);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();  // smem may still be read from a previous use
    if (lane == 0) smem[warp] = m;
    __syncthreads();
    float r = 0.0f;
    const int nw = (blockDim.x + 31) >> 5;
    for (int w = 0; w < nw; ++w) r = fmaxf(r, smem[w]);
    return r;
}

// MXFP4 block exponent: floor(log2(amax)) - 2, zero block -> -127, clamped.
__device__ __forceinline__ int mx_exponent(float amax_b) {
    int e = (amax_b == 0.0f) ? -127 : floor_log2_exact(amax_b) - 2;
    return max(-127, min(127, e));
}

// Power-of-two block scale pow2ceil(max(amax / fmt_max, 2**-126)).
__device__ __forceinline__ float pow2_scale(float amax_b, float fmt_max) {
    float a = __fdiv_rn(amax_b, fmt_max);
    if (a < kF32MinNormal) a = kF32MinNormal;
    return pow2_ceil_normal(a);
}

// NVFP4 block scale byte: e4m3(max((amax_b / 6) / g, 2**-9)).
__device__ __forceinline__ uint32_t nv_scale_byte(float amax_b, float g) {
    float t = __fdiv_rn(__fdiv_rn(amax_b, kE2M1Max), g);
    t = fmaxf(t, kE4M3MinSub);
    return e4m3_encode_sw(t);
}

// ----------------------------------------------------------- MXFP4 / FP8 ----
// Flat block quantization (blocks never cross rows because K % block == 0).

template <typename T, int FMT /*0 = fp8, 1 = mxfp4*/, int BLOCK, int U>
__global__ void __launch_bounds__(kThreads) flat_quant_kernel(const T* __restrict__ x, int64_t nchunks,
                                                              uint8_t* __restrict__ codes,
                                                              uint8_t* __restrict__ scales) {
    constexpr int L = BLOCK / 8;
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t base = (int64_t)blockIdx.x * kThreads + (threadIdx.x & ~31); base < nchunks; base += U * stride) {
        float v[U][8];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t c = base + u * stride + lane;
            if (c < nchunks) load8(x + c * 8, v[u]);
            else {
#pragma unroll
                for (int j = 0; j < 8; ++j) v[u][j] = 0.0f;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t c = base + u * stride + lane;
            const float amax_b = group_max<L>(amax8(v[u]));
            if (FMT == 1) {
                const int e = mx_exponent(amax_b);
                const float inv = exp2_int(-e);  // x * 2**-e == x / 2**e exactly
                float q[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) q[j] = v[u][j] * inv;
                const uint32_t packed = e2m1x8_encode_hw(q);
                if (c < nchunks) {
                    reinterpret_cast<uint32_t*>(codes)[c] = packed;
                    if ((lane % L) == 0) scales[c / L] = (uint8_t)(e + 127);
                }
            } else {
                const float p = pow2_scale(amax_b, kE4M3Max);
                const float inv = exp2_int(127 - f32_biased_exp(p));  // 1 / p, exact
                uint2 w;
                w.x = e4m3x2_encode_hw(v[u][0] * inv, v[u][1] * inv) |
                      (e4m3x2_encode_hw(v[u][2] * inv, v[u][3] * inv) << 16);
                w.y = e4m3x2_encode_hw(v[u][4] * inv, v[u][5] * inv) |
                      (e4m3x2_encode_hw(v[u][6] * inv, v[u][7] * inv) << 16);
                if (c < nchunks) {
                    reinterpret_cast<uint2*>(codes)[c] = w;
                    if ((lane % L) == 0) scales[c / L] = (uint8_t)f32_biased_exp(p);
                }
            }
        }
    }
}

// e2m1 byte -> (value of low nibble, value of high nibble), built per CTA.
__device__ __forceinline__ void build_e2m1_lut(float2* lut) {
    for (int b = threadIdx.x; b < 256; b += blockDim.x) lut[b] = make_float2(e2m1_decode(b & 15), e2m1_decode(b >> 4));
    __syncthreads();
}

// ----------------------------------------------------------------- NVFP4 ----

// Quantize one 8-element chunk whose block partner is lane ^ 1, given the
// row scale g (g == 0: zero row).  Returns the packed 4 bytes; *scale_byte
// receives the block's e4m3 scale.
// e2m1 codes of RN(v[j] / d) for 8 values, bit-exact, mostly without a
// division.  With r = RN(1/d), q = RN(v * r) lies within 1.5 * 2**-23 * |q| of
// RN(v / d) (two roundings of 2**-24 each, d and r normal).  The e2m1 rounding
// is monotone in |q|, so if the two brackets q * (1 - 2**-21) and
// q * (1 + 2**-21), which enclose RN(v / d), round to the same codes, those
// are the codes of RN(v / d); only when a bracket straddles a rounding
// boundary (rare) or d is out of range is the quotient computed by IEEE
// division.
__device__ __forceinline__ uint32_t e2m1x8_of_quotient(const float v[8], float d) {
    if (d >= 2.3509887e-38f /* 2**-125 */ && d <= 4.2535296e37f /* 2**125 */) {
        const float r = __frcp_rn(d);
        float lo[8], hi[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float q = __fmul_rn(v[j], r);
            lo[j] = __fmul_rn(q, 0.99999952f);  // 1 - 2**-21
            hi[j] = __fmul_rn(q, 1.00000048f);  // 1 + 2**-21
        }
        const uint32_t clo = e2m1x8_encode_hw(lo), chi = e2m1x8_encode_hw(hi);
        if (clo == chi) return clo;
    }
    float q[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) q[j] = __fdiv_rn(v[j], d);
    return e2m1x8_encode_hw(q);
}

// Quantize one 8-element chunk whose block partner is lane ^ 1, given the
// row scale g (g == 0: zero row).  Returns the packed 4 bytes; *scale_byte
// receives the block's e4m3 scale.
__device__ __forceinline__ uint32_t nv_quant_chunk(const float v[8], float g, uint32_t* scale_byte) {
    const float amax_b = group_max<2>(amax8(v));
    if (g == 0.0f) {
        *scale_byte = 0u;
        return 0u;
    }
    const uint32_t s = nv_scale_byte(amax_b, g);
    const float d = __fmul_rn(e4m3_decode(s), g);
    *scale_byte = s;
    return e2m1x8_of_quotient(v, d);
}

// ---- one lane per 16-element NVFP4 block --------------------------------

constexpr float kInv6 = 0.16666667f;        // RN(1/6)
constexpr float kTwoM120 = 7.5231638e-37f;  // 2**-120

// RN(1/g) when g is a normal value whose reciprocal is normal too (the fast
// paths below rely on it), else 0.
__device__ __forceinline__ float nv_recip_or_zero(float g) {
    return (g >= 2.3509887e-38f && g <= 4.2535296e37f) ? __frcp_rn(g) : 0.0f;
}

// Block scale code e4m3(max(RN(RN(a / 6) / g), 2**-9)), bit-exact.  With
// rg = RN(1/g), t1 = RN(RN(a * RN(1/6)) * rg) is within 6 * 2**-24 * t of the
// two-division chain (a normal, g and 1/g normal); the brackets
// t1 * (1 -+ 2**-20), clamped at 2**-9, enclose the chain's value, and the
// e4m3 rounding (to nearest even, saturating) is monotone, so equal codes for
// both brackets are the chain's code.  Otherwise the chain is evaluated.
__device__ __forceinline__ uint32_t nv_scale_code(float a, float g, float rg) {
    if (rg != 0.0f && (a == 0.0f || a >= kTwoM120)) {
        const float t1 = __fmul_rn(__fmul_rn(a, kInv6), rg);
        const float lo = fmaxf(__fmul_rn(t1, 0.99999905f), kE4M3MinSub);  // 1 - 2**-20
        const float hi = fmaxf(__fmul_rn(t1, 1.00000095f), kE4M3MinSub);  // 1 + 2**-20
        const uint32_t c2 = e4m3x2_encode_hw(lo, hi);
        if ((c2 & 0xFFu) == (c2 >> 8)) return c2 & 0xFFu;
    }
    return nv_scale_byte(a, g);
}

// 16 values -> 8 bytes of packed e2m1 codes (low word: elements 0..7) and the
// block's e4m3 scale, for row scale g (0: zero row) with rg = nv_recip_or_zero(g).
__device__ __forceinline__ uint2 nv_quant_block(const float v[16], float g, float rg, uint32_t* scale_byte) {
    if (g == 0.0f) {
        *scale_byte = 0u;
        return make_uint2(0u, 0u);
    }
    const float amax_b = fmaxf(amax8(v), amax8(v + 8));
    const uint32_t s = nv_scale_code(amax_b, g, rg);
    const float d = __fmul_rn(e4m3_decode(s), g);
    *scale_byte = s;
    return make_uint2(e2m1x8_of_quotient(v, d), e2m1x8_of_quotient(v + 8, d));
}

// 16 consecutive elements (32-byte aligned for bf16).  Plain (L1-cached)
// loads: the second half of every line a warp touches is then an L1 hit.
__device__ __forceinline__ void load16(const uint16_t* p, float v[16]) {
    const uint4 a = *reinterpret_cast<const uint4*>(p), b = *reinterpret_cast<const uint4*>(p + 8);
    v[0] = bf16_lo(a.x); v[1] = bf16_hi(a.x); v[2] = bf16_lo(a.y); v[3] = bf16_hi(a.y);
    v[4] = bf16_lo(a.z); v[5] = bf16_hi(a.z); v[6] = bf16_lo(a.w); v[7] = bf16_hi(a.w);
    v[8] = bf16_lo(b.x); v[9] = bf16_hi(b.x); v[10] = bf16_lo(b.y); v[11] = bf16_hi(b.y);
    v[12] = bf16_lo(b.z); v[13] = bf16_hi(b.z); v[14] = bf16_lo(b.w); v[15] = bf16_hi(b.w);
}
__device__ __forceinline__ void load16(const float* p, float v[16]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 a = reinterpret_cast<const float4*>(p)[q];
        v[4 * q] = a.x; v[4 * q + 1] = a.y; v[4 * q + 2] = a.z; v[4 * q + 3] = a.w;
    }
}

// Per-row amax rule: one CTA per row (grid-stride over rows).  Each row is
// staged in shared memory by one bulk copy (TMA engine, completion on an
// mbarrier), double-buffered so the next row streams in while the current one
// is reduced (row amax) and quantized from shared memory.
constexpr uint64_t kRowWaitNs = 1000000000ull;
constexpr int kRowThreads = 256;
constexpr uint32_t kBulkPiece = 32768;

template <typename T>
__device__ __forceinline__ void row_issue(T* dst, const T* src, uint32_t bytes, uint64_t* bar) {
    sm100::mbar_arrive_expect_tx(bar, bytes);
    for (uint32_t off = 0; off < bytes; off += kBulkPiece)
        sm100::bulk_load(reinterpret_cast<uint8_t*>(dst) + off, reinterpret_cast<const uint8_t*>(src) + off,
                         min(kBulkPiece, bytes - off), bar);
}

__device__ __forceinline__ void lds8(const uint16_t* p, float v[8]) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    v[0] = bf16_lo(w.x); v[1] = bf16_hi(w.x); v[2] = bf16_lo(w.y); v[3] = bf16_hi(w.y);
    v[4] = bf16_lo(w.z); v[5] = bf16_hi(w.z); v[6] = bf16_lo(w.w); v[7] = bf16_hi(w.w);
}
__device__ __forceinline__ void lds8(const float* p, float v[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

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
            reinterpret_cast<uint2*>(packed + r * (K / 2))[blk] = pk;
            scales[r * bpr + blk] = (uint8_t)sb;
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
            reinterpret_cast<uint2*>(packed)[b] = pk;
            scales[b] = (uint8_t)sb;
            if (MODE == 0) {
                const uint32_t row = fdiv((uint32_t)b, bpr);
                if ((uint32_t)b == row * bpr.d) g_out[row] = g[u];
            }
        }
    }
}

// Dequantize (all formats).  Item = the EPI consecutive output elements of
// one lane: 8 for bf16 output (one 16-byte store) and 4 for fp32 output (one
// 16-byte store), so consecutive lanes write consecutive 16-byte pieces and a
// warp store instruction covers one contiguous 512-byte span.  FP4 codes are
// decoded through a 256-entry byte -> (low value, high value) table in shared
// memory; e4m3 codes through the hardware cvt (exact).
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
    __shared__ float2 lut[256];
    if (FMT != FMT_FP8) build_e2m1_lut(lut);
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
                sc[u] = scales[blk];
                if (FMT == FMT_NV) gr[u] = g[fdiv((uint32_t)blk, bpr)];
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
                    const float2 d = e4m3x2_decode_hw((word >> (16 * (i & 1))) & 0xFFFFu);
                    v[2 * i] = d.x * p;
                    v[2 * i + 1] = d.y * p;
                }
            } else {
                const float s = (FMT == FMT_MX) ? e8m0_decode(sc[u]) : e4m3_decode(sc[u]);
#pragma unroll
                for (int i = 0; i < EPI / 2; ++i) {
                    const float2 t = lut[(w0[u] >> (8 * i)) & 0xFFu];
                    if (FMT == FMT_MX) {
                        v[2 * i] = t.x * s;
                        v[2 * i + 1] = t.y * s;
                    } else {
                        v[2 * i] = __fmul_rn(__fmul_rn(t.x, s), gr[u]);
                        v[2 * i + 1] = __fmul_rn(__fmul_rn(t.y, s), gr[u]);
                    }
                }
            }
            TOUT* dst = y + it * EPI;
            if (sizeof(TOUT) == 2) {
                store8(reinterpret_cast<uint16_t*>(dst), v);
            } else {
                __stcs(reinterpret_cast<float4*>(dst), make_float4(v[0], v[1], v[2], v[3]));
            }
        }
    }
}

// ------------------------------------------------------- quantize_cache ----
// S lanes per row (S a power of two, 2 <= S <= 32; 32/S rows per warp); lane
// i of a row walks the chunks i, i + S, ...  of the zero-padded row, so the
// L lanes of a block are adjacent.  VEC: rows are 16-byte aligned and C % 8 == 0.

template <typename T, int FMT, int BLOCK, int S, bool VEC>
__global__ void __launch_bounds__(kThreads) cache_kernel(const T* __restrict__ x, T* __restrict__ y, int64_t rows,
                                                         int64_t C) {
    constexpr int L = BLOCK / 8;
    constexpr int RPW = 32 / S;  // rows per warp
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
        float g = 0.0f;
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
            m = group_max<S>(m);
            g = __fdiv_rn(m, kNvGlobalDiv);
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
            const float amax_b = group_max<L>(amax8(v));
            float out[8];
            if (FMT == BSQ_FP8) {
                const float p = pow2_scale(amax_b, kE4M3Max);
                const float inv = exp2_int(127 - f32_biased_exp(p));
#pragma unroll
                for (int j = 0; j < 8; j += 2) {
                    const float2 d = e4m3x2_decode_hw(e4m3x2_encode_hw(v[j] * inv, v[j + 1] * inv));
                    out[j] = d.x * p;
                    out[j + 1] = d.y * p;
                }
            } else if (FMT == BSQ_MXFP4) {
                const float p = pow2_scale(amax_b, kE2M1Max);
                const float inv = exp2_int(127 - f32_biased_exp(p));
                float q[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) q[j] = v[j] * inv;
                const uint32_t pk = e2m1x8_encode_hw(q);
#pragma unroll
                for (int j = 0; j < 8; ++j) out[j] = e2m1_decode((pk >> (4 * j)) & 15u) * p;
            } else {
                if (g == 0.0f) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) out[j] = 0.0f;
                } else {
                    const float s = e4m3_decode(nv_scale_byte(amax_b, g));
                    const float d = __fmul_rn(s, g);
                    const uint32_t pk = e2m1x8_of_quotient(v, d);
#pragma unroll
                    for (int j = 0; j < 8; ++j) out[j] = __fmul_rn(__fmul_rn(e2m1_decode((pk >> (4 * j)) & 15u), s), g);
                }
            }
            if (row_ok && c < cpr && n > 0) {
                if (VEC && n >= 8) store8(yr + c * 8, out);
                else store_n(yr + c * 8, (int)(n < 8 ? n : 8), out);
            }
        }
    }
}

// Fake-quant of one 8-element chunk in registers (the block's lanes are
// adjacent; g is the row scale for NVFP4).
template <int FMT, int L>
__device__ __forceinline__ void cache_chunk(const float v[8], float g, float rg, float out[8]) {
    const float amax_b = group_max<L>(amax8(v));
    if (FMT == BSQ_FP8) {
        const float p = pow2_scale(amax_b, kE4M3Max);
        const float inv = exp2_int(127 - f32_biased_exp(p));
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            const float2 d = e4m3x2_decode_hw(e4m3x2_encode_hw(v[j] * inv, v[j + 1] * inv));
            out[j] = d.x * p;
            out[j + 1] = d.y * p;
        }
    } else if (FMT == BSQ_MXFP4) {
        const float p = pow2_scale(amax_b, kE2M1Max);
        const float inv = exp2_int(127 - f32_biased_exp(p));
        float q[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) q[j] = v[j] * inv;
        const uint32_t pk = e2m1x8_encode_hw(q);
#pragma unroll
        for (int j = 0; j < 8; ++j) out[j] = e2m1_decode((pk >> (4 * j)) & 15u) * p;
    } else {
        if (g == 0.0f) {
#pragma unroll
            for (int j = 0; j < 8; ++j) out[j] = 0.0f;
        } else {
            const float s = e4m3_decode(nv_scale_code(amax_b, g, rg));
            const float d = __fmul_rn(s, g);
            const uint32_t pk = e2m1x8_of_quotient(v, d);
#pragma unroll
            for (int j = 0; j < 8; ++j) out[j] = __fmul_rn(__fmul_rn(e2m1_decode((pk >> (4 * j)) & 15u), s), g);
        }
    }
}

// FP8 / MXFP4 fake-quant when every row is a whole number of blocks and
// 16-byte aligned: the blocks tile the flat tensor, so this is a flat stream
// with U chunks in flight per lane.
template <typename T, int FMT, int BLOCK, int U>
__global__ void __launch_bounds__(kThreads) cache_flat_kernel(const T* __restrict__ x, T* __restrict__ y,
                                                              int64_t nchunks) {
    constexpr int L = BLOCK / 8;
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t base = (int64_t)blockIdx.x * kThreads + (threadIdx.x & ~31); base < nchunks; base += U * stride) {
        float v[U][8];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t c = base + u * stride + lane;
            if (c < nchunks) load8(x + c * 8, v[u]);
            else {
#pragma unroll
                for (int j = 0; j < 8; ++j) v[u][j] = 0.0f;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t c = base + u * stride + lane;
            float out[8];
            cache_chunk<FMT, L>(v[u], 0.0f, 0.0f, out);
            if (c < nchunks) store8(y + c * 8, out);
        }
    }
}

// Row-resident fake-quant: S lanes per row, every lane loads its (at most
// NCH) chunks of the zero-padded row before any arithmetic; NVFP4 reduces
// the row amax over the S lanes.  Handles partial groups and ragged C.
template <typename T, int FMT, int BLOCK, int S, bool VEC, int NCH>
__global__ void __launch_bounds__(kThreads) cache_row_kernel(const T* __restrict__ x, T* __restrict__ y,
                                                             int64_t rows, int64_t C) {
    constexpr int L = BLOCK / 8;
    constexpr int RPW = 32 / S;
    const int lane = threadIdx.x & 31;
    const int sl = lane % S;
    const int64_t cpr = ((C + BLOCK - 1) / BLOCK) * L;
    const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
    const int64_t wid = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    for (int64_t r0 = wid * RPW; r0 < rows; r0 += warps * RPW) {
        const int64_t r = r0 + lane / S;
        const bool row_ok = r < rows;
        const T* xr = x + (row_ok ? r : 0) * C;
        T* yr = y + (row_ok ? r : 0) * C;
        float v[NCH][8];
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            const int64_t c = sl + (int64_t)i * S;
            const int64_t n = C - c * 8;
            if (row_ok && c < cpr && n > 0) {
                if (VEC && n >= 8) load8(xr + c * 8, v[i]);
                else load_n(xr + c * 8, (int)(n < 8 ? n : 8), v[i]);
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) v[i][j] = 0.0f;
            }
            m = fmaxf(m, amax8(v[i]));
        }
        float g = 0.0f, rg = 0.0f;
        if (FMT == BSQ_NVFP4) {
            g = __fdiv_rn(group_max<S>(m), kNvGlobalDiv);
            rg = nv_recip_or_zero(g);
        }
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            if (i * S >= cpr) break;  // uniform across the warp
            const int64_t c = sl + (int64_t)i * S;
            const int64_t n = C - c * 8;
            float out[8];
            cache_chunk<FMT, L>(v[i], g, rg, out);
            if (row_ok && c < cpr && n > 0) {
                if (VEC && n >= 8) store8(yr + c * 8, out);
                else store_n(yr + c * 8, (int)(n < 8 ? n : 8), out);
            }
        }
    }
}

// ----------------------------------------------------------- launchers -----

static int grid_for(int64_t items, int per_thread) {
    const int64_t need = (items + (int64_t)kThreads * per_thread - 1) / ((int64_t)kThreads * per_thread);
    const int64_t cap = (int64_t)sm_count() * 8;
    return (int)std::max<int64_t>(1, std::min(need, cap));
}

}  // namespace bsq

using namespace bsq;

// ------------------------------------------------------------- C ABI -------

BSQ_API const char* bsq_status_string(bsq_status s) {
    switch (s) {
        case BSQ_OK: return "ok";
        case BSQ_ERR_INVALID_ARG: return "invalid argument";
        case BSQ_ERR_UNSUPPORTED: return "unsupported";
        case BSQ_ERR_CUDA: return "CUDA error";
        case BSQ_ERR_DEVICE: return "device-reported error";
    }
    return "unknown status";
}

BSQ_API const char* bsq_last_error(void) { return g_last_error; }

BSQ_API int bsq_version(void) { return 1; }

static bsq_status check_dtype(bsq_dtype t) {
    if (t != BSQ_BF16 && t != BSQ_FP32) return fail(BSQ_ERR_UNSUPPORTED, "dtype %d not supported", (int)t);
    return BSQ_OK;
}

static bsq_status check_matrix(const char* fn, const void* x, int64_t rows, int64_t K, int block) {
    if (rows < 0 || K < 0) return fail(BSQ_ERR_INVALID_ARG, "%s: negative size (rows=%lld, K=%lld)", fn, (long long)rows, (long long)K);
    if (K % block != 0)
        return fail(BSQ_ERR_INVALID_ARG, "%s: K=%lld is not a whole number of %d-column blocks", fn, (long long)K, block);
    if (rows * K > 0 && x == nullptr) return fail(BSQ_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (rows * K / 8 >= (int64_t(1) << 32)) return fail(BSQ_ERR_UNSUPPORTED, "%s: tensor too large", fn);
    return BSQ_OK;
}

#define BSQ_TRY(expr)                      \
    do {                                   \
        bsq_status _s = (expr);            \
        if (_s != BSQ_OK) return _s;       \
    } while (0)

template <typename T>
static bsq_status launch_nv_rowamax(const T* x, int64_t rows, int64_t K, uint8_t* packed, uint8_t* scales,
                                    float* g_out, cudaStream_t st) {
    const int64_t cpr = K / 8;
    if (K <= 65536) {
        const int grid = (int)std::min<int64_t>(rows, (int64_t)sm_count() * (2048 / kRowThreads));
        nv_rowamax_quant_kernel<T><<<grid, kRowThreads, 0, st>>>(x, rows, K, packed, scales, g_out);
        return check_launch("bsq_quantize_nvfp4");
    }
    // long rows: amax pass, then the flat pass with the computed row scales
    const int grid = (int)std::min<int64_t>(rows, (int64_t)sm_count() * 8);
    row_amax_kernel<T><<<grid, kThreads, 0, st>>>(x, rows, K, g_out);
    BSQ_TRY(check_launch("bsq_quantize_nvfp4"));
    (void)cpr;
    const int64_t nblocks = rows * (K / 16);
    nv_flat_quant_kernel<T, 2, 2><<<grid_for(nblocks, 2), kThreads, 0, st>>>(
        x, nblocks, make_fastdiv((uint32_t)(K / 16)), nullptr, nullptr, 0, packed, scales, g_out);
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
        const int64_t nblocks = rows * (K / 16);
        const FastDiv bpr = make_fastdiv((uint32_t)(K / 16));
        if (xt == BSQ_BF16)
            nv_flat_quant_kernel<uint16_t, 0, 2><<<grid_for(nblocks, 2), kThreads, 0, st>>>(
                (const uint16_t*)x, nblocks, bpr, row_scale_in, nullptr, 0, packed, scales_e4m3, row_scale_out);
        else
            nv_flat_quant_kernel<float, 0, 2><<<grid_for(nblocks, 2), kThreads, 0, st>>>(
                (const float*)x, nblocks, bpr, row_scale_in, nullptr, 0, packed, scales_e4m3, row_scale_out);
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
    const int64_t nchunks = rows * (K / 8), nblocks = rows * (K / 16);
    float* partial = (float*)scratch;
    const FastDiv bpr = make_fastdiv((uint32_t)(K / 16));
    if (xt == BSQ_BF16) {
        amax_partial_kernel<uint16_t, 4><<<P, kThreads, 0, st>>>((const uint16_t*)x, nchunks, partial);
        BSQ_TRY(check_launch("bsq_quantize_nvfp4_tensor"));
        nv_flat_quant_kernel<uint16_t, 1, 2><<<grid_for(nblocks, 2), kThreads, 0, st>>>(
            (const uint16_t*)x, nblocks, bpr, nullptr, partial, P, packed, scales_e4m3, tensor_scale_out);
    } else {
        amax_partial_kernel<float, 4><<<P, kThreads, 0, st>>>((const float*)x, nchunks, partial);
        BSQ_TRY(check_launch("bsq_quantize_nvfp4_tensor"));
        nv_flat_quant_kernel<float, 1, 2><<<grid_for(nblocks, 2), kThreads, 0, st>>>(
            (const float*)x, nblocks, bpr, nullptr, partial, P, packed, scales_e4m3, tensor_scale_out);
    }
    return check_launch("bsq_quantize_nvfp4_tensor");
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
    const int64_t nchunks = rows * (K / 8), nblocks = rows * (K / 16);
    const FastDiv bpr = make_fastdiv((uint32_t)(K / 16));
    if (xt == BSQ_BF16) {
        amax_partial_kernel<uint16_t, 4><<<P, kThreads, 0, st>>>((const uint16_t*)x, nchunks, partial);
        BSQ_TRY(check_launch("bsq_quantize_nvfp4_tensor_noalloc"));
        nv_flat_quant_kernel<uint16_t, 1, 2><<<grid_for(nblocks, 2), kThreads, 0, st>>>(
            (const uint16_t*)x, nblocks, bpr, nullptr, partial, P, packed, scales_e4m3, tensor_scale_out);
    } else {
        amax_partial_kernel<float, 4><<<P, kThreads, 0, st>>>((const float*)x, nchunks, partial);
        BSQ_TRY(check_launch("bsq_quantize_nvfp4_tensor_noalloc"));
        nv_flat_quant_kernel<float, 1, 2><<<grid_for(nblocks, 2), kThreads, 0, st>>>(
            (const float*)x, nblocks, bpr, nullptr, partial, P, packed, scales_e4m3, tensor_scale_out);
    }
    return check_launch("bsq_quantize_nvfp4_tensor_noalloc");
}

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
        dequant_kernel<FMT_NV, uint16_t, 16, 4><<<grid_for(nitems, 4), kThreads, 0, st>>>(
            packed, scales_e4m3, row_scale, bpr, nitems, (uint16_t*)y);
    } else {
        const int64_t nitems = rows * K / 4;
        dequant_kernel<FMT_NV, float, 16, 4><<<grid_for(nitems, 4), kThreads, 0, st>>>(
            packed, scales_e4m3, row_scale, bpr, nitems, (float*)y);
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
        flat_quant_kernel<uint16_t, 1, 32, 4><<<grid_for(nchunks, 4), kThreads, 0, st>>>((const uint16_t*)x, nchunks,
                                                                                         packed, scales_e8m0);
    else
        flat_quant_kernel<float, 1, 32, 4><<<grid_for(nchunks, 4), kThreads, 0, st>>>((const float*)x, nchunks, packed,
                                                                                      scales_e8m0);
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
        dequant_kernel<FMT_MX, uint16_t, 32, 4><<<grid_for(nitems, 4), kThreads, 0, st>>>(
            packed, scales_e8m0, nullptr, none, nitems, (uint16_t*)y);
    } else {
        const int64_t nitems = rows * K / 4;
        dequant_kernel<FMT_MX, float, 32, 4><<<grid_for(nitems, 4), kThreads, 0, st>>>(
            packed, scales_e8m0, nullptr, none, nitems, (float*)y);
    }
    return check_launch("bsq_dequantize_mxfp4");
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
    const int grid = grid_for(nchunks, 4);
    cudaStream_t st = (cudaStream_t)stream;
    if (xt == BSQ_BF16) {
        if (block == 32) flat_quant_kernel<uint16_t, 0, 32, 4><<<grid, kThreads, 0, st>>>((const uint16_t*)x, nchunks, codes_e4m3, scales_e8m0);
        else flat_quant_kernel<uint16_t, 0, 16, 4><<<grid, kThreads, 0, st>>>((const uint16_t*)x, nchunks, codes_e4m3, scales_e8m0);
    } else {
        if (block == 32) flat_quant_kernel<float, 0, 32, 4><<<grid, kThreads, 0, st>>>((const float*)x, nchunks, codes_e4m3, scales_e8m0);
        else flat_quant_kernel<float, 0, 16, 4><<<grid, kThreads, 0, st>>>((const float*)x, nchunks, codes_e4m3, scales_e8m0);
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
        if (block == 32) dequant_kernel<FMT_FP8, uint16_t, 32, 4><<<grid_for(nb, 4), kThreads, 0, st>>>(codes_e4m3, scales_e8m0, nullptr, none, nb, (uint16_t*)y);
        else dequant_kernel<FMT_FP8, uint16_t, 16, 4><<<grid_for(nb, 4), kThreads, 0, st>>>(codes_e4m3, scales_e8m0, nullptr, none, nb, (uint16_t*)y);
    } else {
        if (block == 32) dequant_kernel<FMT_FP8, float, 32, 4><<<grid_for(nf, 4), kThreads, 0, st>>>(codes_e4m3, scales_e8m0, nullptr, none, nf, (float*)y);
        else dequant_kernel<FMT_FP8, float, 16, 4><<<grid_for(nf, 4), kThreads, 0, st>>>(codes_e4m3, scales_e8m0, nullptr, none, nf, (float*)y);
    }
    return check_launch("bsq_dequantize_fp8");
}

template <typename T, int FMT, int BLOCK, bool VEC, int S>
static void launch_cache_rows(const T* x, T* y, int64_t rows, int64_t C, int nch, cudaStream_t st) {
    const int64_t rpw = 32 / S;
    const int64_t warps = (rows + rpw - 1) / rpw;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((warps + 7) / 8, (int64_t)sm_count() * 8));
    if (nch <= 1) cache_row_kernel<T, FMT, BLOCK, S, VEC, 1><<<grid, kThreads, 0, st>>>(x, y, rows, C);
    else if (nch <= 2) cache_row_kernel<T, FMT, BLOCK, S, VEC, 2><<<grid, kThreads, 0, st>>>(x, y, rows, C);
    else if (nch <= 3) cache_row_kernel<T, FMT, BLOCK, S, VEC, 3><<<grid, kThreads, 0, st>>>(x, y, rows, C);
    else if (nch <= 4) cache_row_kernel<T, FMT, BLOCK, S, VEC, 4><<<grid, kThreads, 0, st>>>(x, y, rows, C);
    else cache_kernel<T, FMT, BLOCK, S, VEC><<<grid, kThreads, 0, st>>>(x, y, rows, C);
}

template <typename T, int FMT, int BLOCK, bool VEC>
static void launch_cache_s(const T* x, T* y, int64_t rows, int64_t C, cudaStream_t st) {
    const int64_t cpr = ((C + BLOCK - 1) / BLOCK) * (BLOCK / 8);
    if (FMT != BSQ_NVFP4 && VEC && C % BLOCK == 0) {
        const int64_t nchunks = rows * C / 8;
        cache_flat_kernel<T, FMT, BLOCK, 4><<<grid_for(nchunks, 4), kThreads, 0, st>>>(x, y, nchunks);
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
