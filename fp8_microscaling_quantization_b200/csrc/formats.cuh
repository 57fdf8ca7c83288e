// formats.cuh -- device-side encode/decode of the microscaling element and
// scale formats, written from the format definitions:
//   e2m1      1 sign, 2 exponent (bias 1), 1 mantissa bit: magnitudes
//             {0, 0.5, 1, 1.5, 2, 3, 4, 6}; the NeMo AutoModel mxfp4 page's
//             _FP4_E2M1_TABLE decodes code 8 to +0.0.
//   e4m3fn    1 sign, 4 exponent (bias 7), 3 mantissa bits, subnormals,
//             max 448, S.1111.111 = NaN, no infinity.
//   e8m0fnu   unsigned biased exponent: 2**(code - 127), 0xFF = NaN.
// All arithmetic is IEEE binary32 round-to-nearest-even with subnormals kept
// (the library is built without fast-math / flush-to-zero).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace bsq {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two binary32 -> packed bf16x2 (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Exponent of a binary32 as stored (biased), 0 for zero / subnormal.
__device__ __forceinline__ int f32_biased_exp(float a) { return (__float_as_uint(a) >> 23) & 0xFF; }

// floor(log2(a)) for finite a > 0, exact, subnormals included.
__device__ __forceinline__ int floor_log2_exact(float a) {
    uint32_t b = __float_as_uint(a) & 0x7FFFFFFFu;
    int e = (int)(b >> 23);
    if (e != 0) return e - 127;
    // subnormal: value = m * 2**-149, floor(log2) = index of the top set bit - 149
    return (31 - __clz((int)b)) - 149;
}

// 2**e as a binary32 for e in [-149, 127] (subnormal results built exactly).
__device__ __forceinline__ float exp2_int(int e) {
    if (e >= -126) return __uint_as_float((uint32_t)(e + 127) << 23);
    return __uint_as_float(1u << (e + 149));
}

// ------------------------------------------------------------------ e4m3 --

// Nearest finite e4m3 code, ties to even, saturating at 448 (software; used
// for block scales, one per block).  The quantum of a value's e4m3 binade is
// 2**(max(floor(log2 a), -6) - 3); the code is (binade + 6) * 8 + the value in
// quanta rounded to an integer, which carries into the exponent field by
// itself when the rounding reaches the next binade.
__device__ __forceinline__ uint32_t e4m3_encode_sw(float x) {
    uint32_t sign = (__float_as_uint(x) >> 24) & 0x80u;
    float a = fabsf(x);
    if (!(a < 448.0f)) return sign | 0x7Eu;
    int e = f32_biased_exp(a) - 127;
    if (e < -6) e = -6;
    float m = rintf(a * exp2_int(3 - e));  // exact scaling by a power of two
    return sign | (uint32_t)((e + 6) * 8 + (int)m);
}

__device__ __forceinline__ float e4m3_decode(uint32_t c) {
    uint32_t e = (c >> 3) & 15u, m = c & 7u;
    float v;
    if (e == 0) v = (float)m * 0.001953125f;  // m * 2**-9
    else v = __uint_as_float(((e + 120u) << 23) | (m << 20));
    if (e == 15u && m == 7u) v = __uint_as_float(0x7FC00000u);
    return (c & 0x80u) ? -v : v;
}

// Two binary32 -> two e4m3 bytes (hardware cvt, round to nearest even,
// saturating to +-448): `lo` in the low byte.
__device__ __forceinline__ uint32_t e4m3x2_encode_hw(float lo, float hi) {
    uint32_t out;
    asm("{\n\t.reg .b16 t;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\t"
        "cvt.u32.u16 %0, t;\n\t}"
        : "=r"(out)
        : "f"(hi), "f"(lo));
    return out;
}

// Two e4m3 bytes (low half of w16) -> two binary32 (exact, via f16).
__device__ __forceinline__ float2 e4m3x2_decode_hw(uint32_t w16) {
    uint32_t h2;
    asm("{\n\t.reg .b16 t;\n\t"
        "cvt.u16.u32 t, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
        : "=r"(h2)
        : "r"(w16));
    __half2 h = *reinterpret_cast<__half2*>(&h2);
    return __half22float2(h);
}

// ------------------------------------------------------------------ e2m1 --

// Four pairs of binary32 -> four bytes of packed e2m1 (hardware cvt, round to
// nearest even, saturating to +-6).  v[2i] goes to the low nibble of byte i.
__device__ __forceinline__ uint32_t e2m1x8_encode_hw(const float v[8]) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return out;
}

// Four bytes of packed e2m1 codes -> eight binary32 values (code 2i + j from
// nibble j of byte i), by the hardware conversion to f16x2 and f16 -> f32
// (both exact).  The conversion gives -0.0 for code 8, so code 8 is first
// turned into code 0 on the integer pipe: a nibble keeps its sign bit only
// when its magnitude bits are nonzero (magnitude + 7 carries into bit 3
// exactly then, and never out of the nibble).  The result is the table's
// +0.0 for code 8 and every other value unchanged.
__device__ __forceinline__ void e2m1x8_decode_raw(uint32_t w, float v[8]);
__device__ __forceinline__ void e2m1x8_decode_hw(uint32_t w, float v[8]) {
    const uint32_t mag = w & 0x77777777u;
    const uint32_t nonzero = (mag + 0x77777777u) & 0x88888888u;
    e2m1x8_decode_raw(mag | (w & nonzero), v);
}


// The same decode without the +0.0: code 8 gives -0.0 (for callers that fold
// the sign of zero into a later fma with +0.0).
__device__ __forceinline__ void e2m1x8_decode_raw(uint32_t w, float v[8]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t h2;
        asm("{\n\t.reg .b8 t;\n\t"
            "cvt.u8.u32 t, %1;\n\t"
            "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
            : "=r"(h2)
            : "r"(w >> (8 * i)));
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

// Four bytes of packed e2m1 codes -> four f16x2 words (codes 2i, 2i + 1 in
// word i), code 8 turned into code 0 first as in e2m1x8_decode_hw.  Every
// e2m1 value is exact in f16.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t h[4]) {
    const uint32_t mag = w & 0x77777777u;
    w = mag | (w & ((mag + 0x77777777u) & 0x88888888u));
#pragma unroll
    for (int i = 0; i < 4; ++i)
        asm("{\n\t.reg .b8 t;\n\t"
            "cvt.u8.u32 t, %1;\n\t"
            "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
            : "=r"(h[i])
            : "r"(w >> (8 * i)));
}

// The two f16 values of e2 times the f16 value in the low half of s2, as
// binary32 (a mixed-precision fma with -0.0 added: the products of an e2m1
// and an e4m3 value have at most 6 significant bits, so they are exact, and
// x + -0.0 is x for every x, -0.0 and +0.0 included).
__device__ __forceinline__ float2 mul_f16_to_f32(uint32_t e2, uint32_t s2) {
    float2 d;
    asm("{\n\t.reg .f16 el, eh, s, sh;\n\t"
        "mov.b32 {el, eh}, %2;\n\tmov.b32 {s, sh}, %3;\n\t"
        "fma.rn.f32.f16 %0, el, s, 0f80000000;\n\t"
        "fma.rn.f32.f16 %1, eh, s, 0f80000000;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "r"(e2), "r"(s2));
    return d;
}

// e4m3 byte (low byte of c) -> its value as f16 in the low half of an
// f16x2 word (exact: every e4m3 value, subnormals included, is an f16 normal).
__device__ __forceinline__ uint32_t e4m3_to_f16x2(uint32_t c) {
    uint32_t h2;
    asm("{\n\t.reg .b16 t;\n\t"
        "cvt.u16.u32 t, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
        : "=r"(h2)
        : "r"(c & 0xFFu));
    return h2;
}

// e8m0 byte -> 2**(code - 127) as binary32 (code 0 is the subnormal 2**-127,
// 0xFF is NaN).
__device__ __forceinline__ float e8m0_decode(uint32_t c) {
    c &= 0xFFu;
    if (c == 0xFFu) return __uint_as_float(0x7FC00000u);
    if (c == 0u) return __uint_as_float(0x00400000u);
    return __uint_as_float(c << 23);
}

}  // namespace bsq
