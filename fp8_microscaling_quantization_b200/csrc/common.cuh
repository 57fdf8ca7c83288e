// common.cuh -- device and host helpers shared by the quantize / dequantize
// / cache kernels of libbsq: element loads and stores, block reductions, the
// block-scale rules and the bit-exact NVFP4 code computations.
#pragma once

#include <algorithm>
#include <cstdint>

#include "formats.cuh"
#include "host_util.h"

namespace bsq {

static inline bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

// ---------------------------------------------------------- device helpers --

constexpr int kThreads = 256;
constexpr float kE2M1Max = 6.0f;       // nvfp4 page E2M1_MAX
constexpr float kE4M3Max = 448.0f;     // nvfp4 page E4M3_MAX
constexpr float kE4M3MinSub = 0.001953125f;  // nvfp4 page E4M3_MIN_SUBNORMAL = 2**-9
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

// Max over the 32 lanes of a warp of a non-negative binary32 (an amax): the
// bit patterns of non-negative floats order as unsigned integers, so one
// redux.sync does it.
__device__ __forceinline__ float warp_max_nonneg(float m) {
    return __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(m)));
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

// MXFP8 block exponent: the MXFP4 rule with e4m3's largest exponent,
// floor(log2(amax)) - 8 (448 = 1.75 * 2**8), zero block -127, clamped.
__device__ __forceinline__ int mx8_exponent(float amax_b) {
    int e = (amax_b == 0.0f) ? -127 : floor_log2_exact(amax_b) - 8;
    return max(-127, min(127, e));
}

// Power-of-two block scale pow2ceil(max(RN(a / M), 2**-126)) for a finite
// a >= 0 and M = m * 2**K, m = 1.75 (448: K = 8, MM = 0x600000) or m = 1.5
// (6: K = 2, MM = 0x400000): its biased exponent, exactly, from the bits of a.
// With a = A * 2**E, A in [1, 2): A / m lies in [1/m, 2/m), which holds no
// power of two but 1, so RN(a / M) is at most 2**(E - K) when A <= m and
// above it when A > m (then A / m >= 1 + 2**-23 / m, which rounds up, away
// from 1).  The floor 2**-126 covers zero, subnormal a and every quotient
// below it.
template <int K, uint32_t MM>
__device__ __forceinline__ uint32_t pow2_scale_biased(float a) {
    const uint32_t b = __float_as_uint(a);
    const int pb = (int)(b >> 23) - K + ((b & 0x7FFFFFu) > MM ? 1 : 0);
    return (uint32_t)max(pb, 1);
}

// NVFP4 block scale byte: e4m3(max((amax_b / 6) / g, 2**-9)).
__device__ __forceinline__ uint32_t nv_scale_byte(float amax_b, float g) {
    float t = __fdiv_rn(__fdiv_rn(amax_b, kE2M1Max), g);
    t = fmaxf(t, kE4M3MinSub);
    return e4m3_encode_sw(t);
}

// ----------------------------------------------------------------- NVFP4 ----

// e2m1 codes of RN(v[j] / d) for 8 values, bit-exact, mostly without a
// division.  With r = RN(1/d), q = RN(v * r) lies within 1.5 * 2**-23 * |q| of
// RN(v / d) (two roundings of 2**-24 each, d and r normal).  The e2m1 rounding
// is monotone in |q|, so if the two brackets q * (1 - 2**-21) and
// q * (1 + 2**-21), which enclose RN(v / d), round to the same codes, those
// are the codes of RN(v / d); only when a bracket straddles a rounding
// boundary (rare) or d is out of range is the quotient computed by IEEE
// division.
__device__ __forceinline__ uint32_t e2m1x8_of_quotient_r(const float v[8], float d, float r);

__device__ __forceinline__ uint32_t e2m1x8_of_quotient(const float v[8], float d) {
    return e2m1x8_of_quotient_r(v, d, __frcp_rn(d));
}

// The same with r = RN(1 / d) supplied by the caller (a per-scale table).
__device__ __forceinline__ uint32_t e2m1x8_of_quotient_r(const float v[8], float d, float r) {
    if (d >= 2.3509887e-38f /* 2**-125 */ && d <= 4.2535296e37f /* 2**125 */) {
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

// ---- lean NVFP4 block: shared reciprocal table, brackets on the reciprocal --
//
// Per-CTA table of RN(1/s) over the e4m3 scale codes (index = code, positive
// finite codes 1..126; the rest 0), filled once per CTA.
__device__ __forceinline__ void fill_inv_e4m3(float* tab) {
    for (int c = threadIdx.x; c < 128; c += blockDim.x)
        tab[c] = (c >= 1 && c <= 126) ? __frcp_rn(e4m3_decode((uint32_t)c)) : 0.0f;
}

// max(|a|, |b|) of each bf16 lane of two bf16x2 words (the sign of the result
// is the XOR of the signs; only the magnitude is used).
__device__ __forceinline__ uint32_t bf16x2_maxabs(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// 16 elements of one NVFP4 block as loaded (bf16: two uint4, fp32: four
// float4), widened to binary32 on use.
template <typename T> struct Raw16;
// 16 bytes from a 32-bit shared-memory address.
__device__ __forceinline__ uint4 lds128(uint32_t saddr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(saddr));
    return v;
}

template <> struct Raw16<uint16_t> {
    uint4 a, b;
    __device__ __forceinline__ void load(const uint16_t* p) {
        a = reinterpret_cast<const uint4*>(p)[0];
        b = reinterpret_cast<const uint4*>(p)[1];
    }
    __device__ __forceinline__ void load_smem(uint32_t saddr) {
        a = lds128(saddr);
        b = lds128(saddr + 16);
    }
    // block amax, exact (bf16 -> binary32 widening is exact)
    __device__ __forceinline__ float amax() const {
        const uint32_t m = bf16x2_maxabs(bf16x2_maxabs(bf16x2_maxabs(a.x, a.y), bf16x2_maxabs(a.z, a.w)),
                                         bf16x2_maxabs(bf16x2_maxabs(b.x, b.y), bf16x2_maxabs(b.z, b.w)));
        return fmaxf(fabsf(bf16_lo(m)), fabsf(bf16_hi(m)));
    }
    __device__ __forceinline__ void half(int h, float v[8]) const {
        const uint4 w = h ? b : a;
        v[0] = bf16_lo(w.x); v[1] = bf16_hi(w.x); v[2] = bf16_lo(w.y); v[3] = bf16_hi(w.y);
        v[4] = bf16_lo(w.z); v[5] = bf16_hi(w.z); v[6] = bf16_lo(w.w); v[7] = bf16_hi(w.w);
    }
};
template <> struct Raw16<float> {
    float4 q[4];
    __device__ __forceinline__ void load(const float* p) {
#pragma unroll
        for (int i = 0; i < 4; ++i) q[i] = reinterpret_cast<const float4*>(p)[i];
    }
    __device__ __forceinline__ void load_smem(uint32_t saddr) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 w = lds128(saddr + 16 * i);
            q[i] = make_float4(__uint_as_float(w.x), __uint_as_float(w.y), __uint_as_float(w.z), __uint_as_float(w.w));
        }
    }
    __device__ __forceinline__ float amax() const {
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            m = fmaxf(fmaxf(m, fmaxf(fabsf(q[i].x), fabsf(q[i].y))), fmaxf(fabsf(q[i].z), fabsf(q[i].w)));
        return m;
    }
    __device__ __forceinline__ void half(int h, float v[8]) const {
        const float4 c = q[2 * h], d = q[2 * h + 1];
        v[0] = c.x; v[1] = c.y; v[2] = c.z; v[3] = c.w; v[4] = d.x; v[5] = d.y; v[6] = d.z; v[7] = d.w;
    }
};

// Two binary32 products at once (packed f32x2 multiply of sm_100a; each lane
// rounds to nearest even exactly as a scalar multiply does).
__device__ __forceinline__ float2 mul_f32x2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 A, B, D;\n\t"
        "mov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
        "mul.rn.f32x2 D, A, B;\n\t"
        "mov.b64 {%0, %1}, D;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// fma of two binary32 pairs at once (packed f32x2 fma of sm_100a; each lane
// rounds once, exactly as a scalar fma does).
__device__ __forceinline__ float2 fma_f32x2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 A, B, C, D;\n\t"
        "mov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\tmov.b64 C, {%6, %7};\n\t"
        "fma.rn.f32x2 D, A, B, C;\n\t"
        "mov.b64 {%0, %1}, D;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// Asynchronous 16-byte global -> shared copies (cp.async, L2 only), grouped
// per thread; a thread waits for its own groups with cp_async_wait.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
                 "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// The block's codes by the plain rule (IEEE division where the brackets
// cannot decide); kept out of line, it runs for a tiny fraction of blocks.
template <typename T>
__device__ __noinline__ uint2 nv_block_codes_slow(Raw16<T> raw, float g, uint32_t s) {
    const float d = __fmul_rn(e4m3_decode(s), g);
    float v[8];
    raw.half(0, v);
    const uint32_t c0 = e2m1x8_of_quotient(v, d);
    raw.half(1, v);
    return make_uint2(c0, e2m1x8_of_quotient(v, d));
}

// Settling a straddled element (the bracket codes of the fp32 NVFP4 path
// differ), bit-exact and still without a division.  An element whose two
// bracket codes differ has exactly one e2m1 rounding boundary b between them
// (0.25, 0.75, 1.25, 1.75, 2.5, 3.5 or 5; the brackets are far narrower than
// the gaps), and |x| lies within 2**-20 of b * d, d = RN(float(s) * g), so
// e = fma(-b, d, |x|) is the exact difference.  With hu half an ulp of b and
// hd half an ulp of the float below b (hu / 2 for b = 0.25, a power of two):
// RN(|x| / d) > b iff e > hu * d, < b iff e < -hd * d, else it equals b, an
// e2m1 tie that rounds to the even code.  (b's significand is even, so the
// roundings of b + hu and b - hd are b itself.)

// Element i of a block held in shared memory at saddr, as binary32.
template <typename T>
__device__ __forceinline__ float elem_smem(uint32_t saddr, int i);
template <>
__device__ __forceinline__ float elem_smem<uint16_t>(uint32_t saddr, int i) {
    uint32_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(saddr + 2u * (uint32_t)i));
    return __uint_as_float(v << 16);
}
template <>
__device__ __forceinline__ float elem_smem<float>(uint32_t saddr, int i) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(saddr + 4u * (uint32_t)i));
    return v;
}

// Settles the nibbles of clo (the lower bracket's codes of the 8 elements at
// shared address half) where the upper bracket's codes differ (set bits of
// diff), by the fma test above.
// Per lower magnitude code k = 0..6 of a straddle: the e2m1 rounding boundary
// b above it, and the half ulps hu (of b) and hd (of the float below b).
struct NvBound {
    float b, hu, hd, pad;
};
__device__ __forceinline__ void fill_nv_bounds(NvBound* t) {
    if (threadIdx.x < 8) {
        const int k = threadIdx.x;
        // e2m1 magnitudes: k < 4: k / 2; then 2, 3, 4, 6; b is the midpoint to the next
        const float b = (k < 4) ? 0.25f + 0.5f * (float)k : (k == 4 ? 2.5f : (k == 5 ? 3.5f : (k == 6 ? 5.0f : 6.0f)));
        const int eb = floor_log2_exact(b);
        t[k].b = b;
        t[k].hu = exp2_int(eb - 24);
        t[k].hd = (k == 0) ? exp2_int(eb - 25) : exp2_int(eb - 24);
        t[k].pad = 0.0f;
    }
}

// Element i (0..7, not known at compile time) of 8 values in registers.
__device__ __forceinline__ float pick8(const float v[8], int i) {
    float x = v[0];
#pragma unroll
    for (int j = 1; j < 8; ++j) x = (i == j) ? v[j] : x;
    return x;
}

// nv_settle_straddles for 8 elements held in registers (v).
__device__ __forceinline__ uint32_t nv_settle_straddles_regs(uint32_t clo, uint32_t diff, const float v[8], float d,
                                                             const NvBound* bounds) {
    while (diff) {
        const int sh = (__ffs(diff) - 1) & ~3;
        diff &= ~(0xFu << sh);
        const uint32_t cl = (clo >> sh) & 0xFu;
        const uint32_t k = cl & 7u;
        const NvBound bd = bounds[k];
        const float e = __fmaf_rn(-bd.b, d, fabsf(pick8(v, sh >> 2)));
        const uint32_t mag = (e > __fmul_rn(bd.hu, d)) ? k + 1u : ((e < -__fmul_rn(bd.hd, d)) ? k : ((k + 1u) & ~1u));
        clo = (clo & ~(0xFu << sh)) | (((cl & 8u) | mag) << sh);
    }
    return clo;
}

template <typename T>
__device__ __forceinline__ uint32_t nv_settle_straddles(uint32_t clo, uint32_t diff, uint32_t half, float d,
                                                        const NvBound* bounds) {
    while (diff) {
        const int sh = (__ffs(diff) - 1) & ~3;  // 4 * nibble index
        diff &= ~(0xFu << sh);
        const uint32_t cl = (clo >> sh) & 0xFu;
        const uint32_t k = cl & 7u;  // the lower magnitude code (lo <= hi in magnitude)
        const NvBound bd = bounds[k];
        const float x = elem_smem<T>(half, sh >> 2);
        const float e = __fmaf_rn(-bd.b, d, fabsf(x));
        const uint32_t mag = (e > __fmul_rn(bd.hu, d)) ? k + 1u : ((e < -__fmul_rn(bd.hd, d)) ? k : ((k + 1u) & ~1u));
        clo = (clo & ~(0xFu << sh)) | (((cl & 8u) | mag) << sh);
    }
    return clo;
}


// The division-free codes of one block (the hot path of the NVFP4 quantize
// kernels): brackets on r = RN(RN(1/s) * rg), and the rare straddled element
// settled by the fma test.  raw holds the block's 16 elements, blk the shared
// address of the same elements (read only for a straddled element), s the
// scale code, g != 0 and rg = nv_recip_or_zero(g).  Returns false only when r
// is out of range; the caller then takes the plain rule (nv_block_codes_slow).
template <typename T>
__device__ __forceinline__ bool nv_block_codes_fast(const Raw16<T>& raw, uint32_t blk, uint32_t s, float g, float rg,
                                                    const float* inv_tab, const NvBound* bounds, uint2* codes) {
    const float r = __fmul_rn(inv_tab[s], rg);
    if (!(r >= 2.3509887e-38f /* 2**-125 */ && r <= 4.2535296e37f /* 2**125 */)) return false;
    const float2 rlo = make_float2(__fmul_rn(r, 0.99999952f), __fmul_rn(r, 0.99999952f));  // 1 - 2**-21
    const float2 rhi = make_float2(__fmul_rn(r, 1.00000048f), __fmul_rn(r, 1.00000048f));  // 1 + 2**-21
    uint32_t clo[2], chi[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float v[8], lo[8], hi[8];
        raw.half(h, v);
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            const float2 l = mul_f32x2(make_float2(v[j], v[j + 1]), rlo);
            const float2 u = mul_f32x2(make_float2(v[j], v[j + 1]), rhi);
            lo[j] = l.x; lo[j + 1] = l.y;
            hi[j] = u.x; hi[j + 1] = u.y;
        }
        clo[h] = e2m1x8_encode_hw(lo);
        chi[h] = e2m1x8_encode_hw(hi);
    }
    const uint32_t d0 = clo[0] ^ chi[0], d1 = clo[1] ^ chi[1];
    if (d0 | d1) {  // rare: a bracket straddles an e2m1 rounding boundary
        const float d = __fmul_rn(e4m3x2_decode_hw(s).x, g);  // RN(float(s) * g); s is a positive code
        if (d0) clo[0] = nv_settle_straddles<T>(clo[0], d0, blk, d, bounds);
        if (d1) clo[1] = nv_settle_straddles<T>(clo[1], d1, blk + 8u * (uint32_t)sizeof(T), d, bounds);
    }
    *codes = make_uint2(clo[0], clo[1]);
    return true;
}

// ---- bf16 NVFP4 block: the correctly rounded quotient, no brackets --------
//
// For bf16 elements the code of every element is the e2m1 rounding of
// q1 = RN(x/d), d = RN(float(s) * g), computed without a division:
//   y  = RN(1/d)                      (once per block)
//   q0 = RN(x * y)
//   r  = RN(q0 * d - x)               (fma)
//   q1 = RN(q0 - r * y)               (fma)
// q1 equals the IEEE quotient RN(x/d) for every bf16 significand and every
// binary32 significand of d (all 2**30 pairs are checked on the CPU by
// tests/test_exact_brackets.py), hence for all x and d whose intermediate
// values stay normal: d in [2**-64, 2**100] and |x| * y <= 2**100 (the block
// amax bounds every element), checked per block; outside that the caller
// takes the plain rule.  Elements below 2**-126 * d only ever give code 0,
// with the sign of x.  The products run on -x and -y, so that x = -0.0 gives
// q1 = -0.0 (and +0.0 gives +0.0), as the division does.
__device__ __forceinline__ void neg_half_bf16(uint4 w, float v[8]) {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(ws[i] * 65536u + 0x80000000u);  // (bits << 16) with the sign bit flipped
        v[2 * i + 1] = __uint_as_float((ws[i] & 0xFFFF0000u) ^ 0x80000000u);
    }
}

// The block's codes (low word: elements 0..7) for the positive scale code s,
// g != 0 and the block amax amax_b.  False when d or the quotients leave the
// range above (the caller then takes nv_block_codes_slow).
__device__ __forceinline__ bool nv_block_codes_bf16(const Raw16<uint16_t>& raw, float amax_b, uint32_t s, float g,
                                                    uint2* codes) {
    const float d = __fmul_rn(e4m3x2_decode_hw(s).x, g);
    if (!(d >= 5.4210109e-20f /* 2**-64 */ && d <= 1.2676506e30f /* 2**100 */)) return false;
    const float y = __frcp_rn(d);
    if (!(__fmul_rn(amax_b, y) <= 1.2676506e30f)) return false;
    const float2 ny = make_float2(-y, -y), d2 = make_float2(d, d);
    uint32_t c[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float nx[8], q[8];
        neg_half_bf16(h ? raw.b : raw.a, nx);
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            const float2 xn = make_float2(nx[j], nx[j + 1]);
            const float2 q0 = mul_f32x2(xn, ny);      // RN(x * y)
            const float2 r = fma_f32x2(q0, d2, xn);   // RN(q0 * d - x)
            const float2 q1 = fma_f32x2(r, ny, q0);   // RN(q0 - r * y)
            q[j] = q1.x;
            q[j + 1] = q1.y;
        }
        c[h] = e2m1x8_encode_hw(q);
    }
    *codes = make_uint2(c[0], c[1]);
    return true;
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

// 8 consecutive elements kept as loaded (bf16: one uint4, fp32: two float4)
// and widened to binary32 on use: a bf16 chunk in flight costs 4 registers.
template <typename T> struct Raw8;
template <> struct Raw8<uint16_t> {
    uint4 r;
    __device__ __forceinline__ void load(const uint16_t* p) { r = *reinterpret_cast<const uint4*>(p); }
    __device__ __forceinline__ void load_cs(const uint16_t* p) { r = __ldcs(reinterpret_cast<const uint4*>(p)); }
    __device__ __forceinline__ void zero() { r = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ void get(float v[8]) const {
        v[0] = bf16_lo(r.x); v[1] = bf16_hi(r.x); v[2] = bf16_lo(r.y); v[3] = bf16_hi(r.y);
        v[4] = bf16_lo(r.z); v[5] = bf16_hi(r.z); v[6] = bf16_lo(r.w); v[7] = bf16_hi(r.w);
    }
};
template <> struct Raw8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float* p) {
        a = reinterpret_cast<const float4*>(p)[0];
        b = reinterpret_cast<const float4*>(p)[1];
    }
    __device__ __forceinline__ void load_cs(const float* p) {
        a = __ldcs(reinterpret_cast<const float4*>(p));
        b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
    }
    __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ void get(float v[8]) const {
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
};

// Grid of a multiple of the SM count: enough CTAs for `items` at
// `per_thread` items per thread, capped at 8 CTAs per SM (grid-stride loops).
static inline int grid_for(int64_t items, int per_thread) {
    const int64_t need = (items + (int64_t)kThreads * per_thread - 1) / ((int64_t)kThreads * per_thread);
    const int64_t cap = (int64_t)sm_count() * 8;
    return (int)std::max<int64_t>(1, std::min(need, cap));
}

// CTAs of KERNEL (kThreads threads, no dynamic shared memory) resident on one
// SM at once, from the occupancy calculator; cached per device.
template <auto KERNEL>
static inline int resident_ctas() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, KERNEL, kThreads, 0) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = 1;
        }
        cache[dev] = n;
    }
    return cache[dev];
}

// Launch a grid-stride KERNEL with one wave of CTAs: enough for `items` at
// `per_thread` items per thread, and no more than the device holds at once.
// Every CTA then starts immediately and gets an equal share of the stream,
// where a grid of several waves leaves SMs idle behind a partial last wave.
template <auto KERNEL, typename... A>
static inline void launch_fit_ctas(int64_t ctas_needed, cudaStream_t st, A... args) {
    const int64_t cap = (int64_t)sm_count() * resident_ctas<KERNEL>();
    const int grid = (int)std::max<int64_t>(1, std::min(ctas_needed, cap));
    KERNEL<<<grid, kThreads, 0, st>>>(args...);
}

template <auto KERNEL, typename... A>
static inline void launch_fit(int64_t items, int per_thread, cudaStream_t st, A... args) {
    const int64_t need = (items + (int64_t)kThreads * per_thread - 1) / ((int64_t)kThreads * per_thread);
    launch_fit_ctas<KERNEL>(need, st, args...);
}

static inline bsq_status check_dtype(bsq_dtype t) {
    if (t != BSQ_BF16 && t != BSQ_FP32) return fail(BSQ_ERR_UNSUPPORTED, "dtype %d not supported", (int)t);
    return BSQ_OK;
}

static inline bsq_status check_matrix(const char* fn, const void* x, int64_t rows, int64_t K, int block) {
    if (rows < 0 || K < 0) return fail(BSQ_ERR_INVALID_ARG, "%s: negative size (rows=%lld, K=%lld)", fn, (long long)rows, (long long)K);
    if (K % block != 0)
        return fail(BSQ_ERR_INVALID_ARG, "%s: K=%lld is not a whole number of %d-column blocks", fn, (long long)K, block);
    // 2**35 elements at most: every kernel's 8-element chunk and 16-block
    // index then fits in 32 bits (tested before rows * K can overflow)
    if (K > 0 && rows > ((int64_t(1) << 35) - 1) / K) return fail(BSQ_ERR_UNSUPPORTED, "%s: tensor too large", fn);
    if (rows * K > 0 && x == nullptr) return fail(BSQ_ERR_INVALID_ARG, "%s: null pointer", fn);
    return BSQ_OK;
}

#define BSQ_TRY(expr)                      \
    do {                                   \
        bsq_status _s = (expr);            \
        if (_s != BSQ_OK) return _s;       \
    } while (0)


}  // namespace bsq
