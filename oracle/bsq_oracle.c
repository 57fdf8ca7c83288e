/*
 * bsq_oracle.c -- plain, slow, scalar CPU oracle for block-scaled microscaling
 * quantization: NVFP4, MXFP4, MXFP8, FP8 with a power-of-two block scale, the
 * cache fake-quant and the static two-level NVFP4 fake-quant.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant generator with the CUDA library; nothing in the
 * product path may call it.
 *
 * Every value is computed one element at a time, in IEEE binary32 with
 * round-to-nearest-even (the build uses -O2 -ffp-contract=off, no fast-math,
 * so no FMA contraction and subnormals are kept), in the order the pages
 * write the formulas.  Rounding to the small formats (e2m1, e4m3, bf16) is
 * done by enumerating / comparing against the representable values, not by
 * bit tricks, so it can be checked by eye.
 *
 * Sources (NeMo AutoModel API documentation and the ModelOpt quantizer source):
 *   [NV]  "nemo_automodel.components.quantization.nvfp4" (v0.7): module text,
 *         quantize_nvfp4, quantize_nvfp4_modelopt, dequantize_nvfp4,
 *         E2M1_MAX, E4M3_MAX, E4M3_MIN_SUBNORMAL, NVFP4_BLOCK_SIZE.
 *   [MX]  "nemo_automodel.components.quantization.mxfp4": module text,
 *         quantize_mxfp4, dequantize_mxfp4, _FP4_E2M1_TABLE,
 *         _FP4_E2M1_MIDPOINTS, _FP4_BYTE_TABLE, MXFP4_BLOCK_SIZE.
 *   [CQ]  "nemo_automodel.components.models.deepseek_v41.quantization":
 *         quantize_cache, _power_of_two_ceiling, _CacheQuantization.
 *   [KV]  "nemo_automodel ... quantization" model-filter page:
 *         dequantize_kv_cache, _dequantize_kv_cache_fused_cuda (the
 *         list-of-blocks NVFP4 KV cache and its contiguous output layout).
 *   [MO]  ModelOpt "tensor_quantizer.py": _FP8_E4M3_MIN_POSITIVE,
 *         StaticBlockScaleQuantizer._block_scale_from_amax, maxbound, is_mxfp
 *         and _real_quantize (MXFP8: e4m3 elements, one e8m0 scale per 32).
 *
 * Readings where the pages are silent are marked "READING:" and are the same
 * readings the repository's design notes list.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define O_BF16 0
#define O_F32 1

#define O_FMT_FP8 0
#define O_FMT_MXFP4 1
#define O_FMT_NVFP4 2

/* [NV] E2M1_MAX = 6.0, E4M3_MAX = 448.0, E4M3_MIN_SUBNORMAL = 2**-9. */
static const float E2M1_MAX = 6.0f;
static const float E4M3_MAX = 448.0f;
static const double E4M3_MIN_SUBNORMAL = 1.0 / 512.0;
/* Smallest positive normal binary32, 2**-126 (domain floor of the
 * power-of-two ceiling, [CQ] _power_of_two_ceiling: "positive normal"). */
static const double F32_MIN_NORMAL = 1.1754943508222875e-38;

/* ------------------------------------------------------------------------ */
/* scalar helpers                                                            */
/* ------------------------------------------------------------------------ */

static float bits_f32(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }
static uint32_t f32_bits(float f) { uint32_t b; memcpy(&b, &f, 4); return b; }

/* bf16 is the top half of a binary32: widening is exact. */
float o_bf16_to_f32(uint16_t h) { return bits_f32((uint32_t)h << 16); }

/* Value of a bf16 magnitude pattern (sign bit clear) as a double; the pattern
 * just past the largest finite value stands for 2**128 so that overflow is
 * decided like any other rounding step. */
static double bf16_mag_value(uint32_t m) {
    if (m >= 0x7F80u) return ldexp(1.0, 128);
    return (double)bits_f32(m << 16);
}

/* binary32 -> bf16, round to nearest, ties to even: pick the nearer of the
 * two bf16 neighbours of |f| (truncation and truncation + 1 ulp). */
uint16_t o_f32_to_bf16(float f) {
    uint32_t b = f32_bits(f);
    uint16_t sign = (uint16_t)((b >> 16) & 0x8000u);
    if (isnan(f)) return (uint16_t)(sign | 0x7FC0u);
    if (isinf(f)) return (uint16_t)(sign | 0x7F80u);
    uint32_t mag = b & 0x7FFFFFFFu;
    uint32_t lo = mag >> 16, hi = lo + 1;
    double a = fabs((double)f);
    double elo = a - bf16_mag_value(lo), ehi = bf16_mag_value(hi) - a;
    uint32_t r;
    if (elo < ehi) r = lo;
    else if (ehi < elo) r = hi;
    else r = (lo & 1u) ? hi : lo;
    return (uint16_t)(sign | r);
}

/* [MX] _FP4_E2M1_TABLE: codes 0..7 are the magnitudes
 * {0, 0.5, 1, 1.5, 2, 3, 4, 6}; codes 8..15 are their negatives, and the
 * printed table holds 0.0 (not -0.0) at code 8. */
static const float E2M1_TABLE[16] = {0.0f,  0.5f,  1.0f,  1.5f,  2.0f,  3.0f,  4.0f,  6.0f,
                                     0.0f, -0.5f, -1.0f, -1.5f, -2.0f, -3.0f, -4.0f, -6.0f};
/* [MX] _FP4_E2M1_MIDPOINTS. */
static const float E2M1_MIDPOINTS[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};

float o_e2m1_val(int code) { return E2M1_TABLE[code & 15]; }

/* Round a binary32 to the nearest e2m1 code.  The magnitude index is the
 * number of midpoints below |q|.  READING: a value exactly on a midpoint goes
 * to the neighbour with the even index (round half to even, the IEEE rule);
 * magnitudes above 6 saturate to 6; the sign is the sign bit of q, so -0.0
 * and negatives that round to zero give code 8. */
int o_e2m1_round(float q) {
    float a = fabsf(q);
    int idx = 0;
    for (int i = 0; i < 7; ++i) {
        if (a > E2M1_MIDPOINTS[i]) idx = i + 1;
        else if (a == E2M1_MIDPOINTS[i] && ((i + 1) % 2) == 0) idx = i + 1;
    }
    return idx | (signbit(q) ? 8 : 0);
}

/* float8_e4m3fn: 1 sign, 4 exponent (bias 7), 3 mantissa bits, subnormals
 * at exponent 0, S.1111.111 is NaN, no infinity ([MO] and [NV]: max 448,
 * smallest subnormal = smallest normal / 8). */
float o_e4m3_val(int code) {
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double v = (e == 0) ? (m / 8.0) * ldexp(1.0, -6) : (1.0 + m / 8.0) * ldexp(1.0, e - 7);
    return (float)(s ? -v : v);
}

/* Round to the nearest finite e4m3 value by enumerating all 127 positive
 * finite codes.  READING: ties go to the even code (even mantissa); values
 * beyond 448 saturate to 448 (nearest finite value); sign from the sign bit. */
int o_e4m3_round(float x) {
    double a = fabs((double)x);
    int best = 0;
    double best_err = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double err = fabs(a - (double)o_e4m3_val(c));
        if (err < best_err || (err == best_err && (c & 1) == 0)) {
            best = c;
            best_err = err;
        }
    }
    return best | (signbit(x) ? 0x80 : 0);
}

/* float8_e8m0fnu: unsigned biased exponent, value 2**(code-127), 0xFF = NaN. */
float o_e8m0_val(int code) {
    code &= 0xFF;
    if (code == 0xFF) return NAN;
    return ldexpf(1.0f, code - 127);
}

/* floor(log2(a)) for finite a > 0, exactly (frexp writes a = f * 2**e with
 * f in [0.5, 1), subnormals included).  READING: the mathematical floor, not
 * a rounded float log2. */
int o_floor_log2(float a) {
    int e;
    frexpf(a, &e);
    return e - 1;
}

/* [CQ] _power_of_two_ceiling: round a positive normal binary32 up to a power
 * of two; a power of two maps to itself. */
float o_pow2_ceil(float a) {
    int e = o_floor_log2(a);
    float p = ldexpf(1.0f, e);
    return (p == a) ? a : ldexpf(1.0f, e + 1);
}

/* ------------------------------------------------------------------------ */
/* element access                                                            */
/* ------------------------------------------------------------------------ */

static float load_elem(const void* x, int dt, int64_t i) {
    if (dt == O_BF16) return o_bf16_to_f32(((const uint16_t*)x)[i]);
    return ((const float*)x)[i];
}

static void store_elem(void* y, int dt, int64_t i, float v) {
    if (dt == O_BF16) ((uint16_t*)y)[i] = o_f32_to_bf16(v);
    else ((float*)y)[i] = v;
}

/* Two e2m1 codes per byte, even column in the low nibble ([NV], [MX]). */
static void put_nibble(uint8_t* packed, int64_t col, int code) {
    uint8_t* b = &packed[col / 2];
    if (col % 2 == 0) *b = (uint8_t)((*b & 0xF0) | (code & 15));
    else *b = (uint8_t)((*b & 0x0F) | ((code & 15) << 4));
}

static int get_nibble(const uint8_t* packed, int64_t col) {
    uint8_t b = packed[col / 2];
    return (col % 2 == 0) ? (b & 15) : (b >> 4);
}

static float block_amax(const void* x, int dt, int64_t start, int64_t n) {
    float m = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(load_elem(x, dt, start + i));
        if (a > m) m = a;
    }
    return m;
}

/* ------------------------------------------------------------------------ */
/* NVFP4 ([NV] quantize_nvfp4 / quantize_nvfp4_modelopt / dequantize_nvfp4)  */
/* ------------------------------------------------------------------------ */

/* Block scale byte and divisor for one 16-block of a row with row scale g:
 *   block_scale = e4m3(amax(block) / 6 / global)         ([NV] quantize_nvfp4)
 * clamped from below at the e4m3 smallest subnormal 2**-9 before the cast
 * ([NV] E4M3_MIN_SUBNORMAL; [MO] _block_scale_from_amax clamps the block
 * scale at the same value in e4m3 units). */
static int nvfp4_block_scale(float amax_b, float g) {
    float t = (amax_b / E2M1_MAX) / g;
    if (t < (float)E4M3_MIN_SUBNORMAL) t = (float)E4M3_MIN_SUBNORMAL;
    return o_e4m3_round(t);
}

/* Quantize one row of K values (K % 16 == 0) with row scale g.
 * READING: g == 0 (an all-zero row under the per-row rule, or a given zero
 * scale) writes scale bytes 0x00 and codes 0. */
static void nvfp4_quantize_row(const void* x, int dt, int64_t base, int64_t K, float g,
                               uint8_t* packed_row, uint8_t* scales_row) {
    for (int64_t b = 0; b < K / 16; ++b) {
        if (g == 0.0f) {
            scales_row[b] = 0;
            for (int j = 0; j < 16; ++j) put_nibble(packed_row, b * 16 + j, 0);
            continue;
        }
        float amax_b = block_amax(x, dt, base + b * 16, 16);
        int s = nvfp4_block_scale(amax_b, g);
        scales_row[b] = (uint8_t)s;
        /* code = round_to_e2m1(w / (block_scale * global)) */
        float d = o_e4m3_val(s) * g;
        for (int j = 0; j < 16; ++j) {
            float q = load_elem(x, dt, base + b * 16 + j) / d;
            put_nibble(packed_row, b * 16 + j, o_e2m1_round(q));
        }
    }
}

/* Per-row rule: global = amax(row) / (6 * 448); with g_in, the given row
 * scales replace the amax rule.  Returns 0, or -1 for K % 16 != 0
 * ([NV] _check_last_dim). */
int o_quantize_nvfp4(const void* x, int dt, int64_t rows, int64_t K, const float* g_in,
                     uint8_t* packed, uint8_t* scales, float* g_out) {
    if (K % 16 != 0) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        float g;
        if (g_in) {
            g = g_in[r];
        } else {
            float amax = block_amax(x, dt, r * K, K);
            g = amax / (E2M1_MAX * E4M3_MAX);
        }
        g_out[r] = g;
        nvfp4_quantize_row(x, dt, r * K, K, g, packed + r * (K / 2), scales + r * (K / 16));
    }
    return 0;
}

/* ModelOpt checkpoint layout: one tensor scale amax(tensor) / (6 * 448) for
 * the whole matrix ([NV] quantize_nvfp4_modelopt: weight, weight_scale,
 * weight_scale_2). */
int o_quantize_nvfp4_tensor(const void* x, int dt, int64_t rows, int64_t K, uint8_t* packed,
                            uint8_t* scales, float* tensor_scale) {
    if (K % 16 != 0) return -1;
    float amax = block_amax(x, dt, 0, rows * K);
    float g = amax / (E2M1_MAX * E4M3_MAX);
    *tensor_scale = g;
    for (int64_t r = 0; r < rows; ++r)
        nvfp4_quantize_row(x, dt, r * K, K, g, packed + r * (K / 2), scales + r * (K / 16));
    return 0;
}

/* value = e2m1 * float(e4m3 block scale) * row scale, binary32 intermediates
 * left to right, one final rounding to the output dtype ([NV] dequantize_nvfp4). */
int o_dequantize_nvfp4(const uint8_t* packed, const uint8_t* scales, const float* g,
                       int64_t rows, int64_t K, void* y, int dt) {
    if (K % 16 != 0) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            float v = o_e2m1_val(get_nibble(packed + r * (K / 2), k));
            float s = o_e4m3_val(scales[r * (K / 16) + k / 16]);
            float prod = v * s;
            float val = prod * g[r];
            store_elem(y, dt, r * K + k, val);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Paged NVFP4 KV cache ([KV] dequantize_kv_cache)                          */
/* ------------------------------------------------------------------------ */

/* A list of nblocks quantized blocks; block b holds block_tokens * heads rows
 * of 128 values (row = token-in-block * heads + head): e2m1 codes
 * values[b] [rows, 64], e4m3 scales scales[b] [rows, 8] and one amax[b].
 * Its global scale is amax[b] / (6 * 448) (the scale rule's e2m1 and e4m3
 * maxima) and its rows dequantize as in dequantize_nvfp4.  Output
 * [1, nblocks * block_tokens, heads, 128]: token t of block b is output token
 * b * block_tokens + t.
 * READING: from_blocked (the swizzled scale layout) is not on the pages, so
 * the scales are the row-major [rows, 8] layout the other NVFP4 functions use. */
int o_dequantize_kv_cache_nvfp4(const uint8_t* const* values, const uint8_t* const* scales,
                                const float* amax, int64_t nblocks, int64_t block_tokens,
                                int64_t heads, void* y, int dt) {
    const int64_t rows = block_tokens * heads;
    const int elem = (dt == O_BF16) ? 2 : 4;
    float* g = (float*)malloc(sizeof(float) * (size_t)(rows > 0 ? rows : 1));
    if (!g) return -2;
    for (int64_t b = 0; b < nblocks; ++b) {
        const float gb = amax[b] / (E2M1_MAX * E4M3_MAX);
        for (int64_t r = 0; r < rows; ++r) g[r] = gb;
        /* block b's rows are the contiguous output range starting at token b * block_tokens */
        void* yb = (char*)y + (size_t)(b * rows * 128) * (size_t)elem;
        o_dequantize_nvfp4(values[b], scales[b], g, rows, 128, yb, dt);
    }
    free(g);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Static two-level NVFP4 fake-quant ([MO] StaticBlockScaleQuantizer:        */
/* _block_scale_from_amax with quantize=True, _amax_to_scale, _clamp_scale,  */
/* _fake_quantize)                                                           */
/* ------------------------------------------------------------------------ */

/* Calibrated per-16-block amax and a global amax (both given):
 *   per_tensor_scale pts = _amax_to_scale(global_amax, 6)
 *                        = A/6, or 1e-8 where A/6 <= 1e-8
 *   min_value = (E4M3 smallest subnormal / 448) * pts
 *   scale_b   = _amax_to_scale(amax_b, 6, min_value)
 *             = amax_b/6, or min_value where amax_b/6 <= min_value
 *   scale_q   = scaled_e4m3(scale_b, pts): scale_b as an e4m3 number in the
 *               units that map pts to 448
 *   y         = cast(e2m1(x / scale_q) * scale_q)
 * binary32 throughout; Python float constants enter as binary32 (torch
 * evaluates a float32 tensor op with a Python scalar in float32).
 * READING: the pages print neither scaled_e4m3 nor
 * static_blockwise_fp4_fake_quant.  Per the comment at min_value, scaled_e4m3
 * maps pts to 448: f = 448 / pts, code = e4m3(scale_b * f), and the same map
 * inverted gives the physical scale, scale_q = e4m3 value / f.  The static
 * path is taken to compute what the LSQ path prints with pre = post amax. */
void o_nvfp4_static_scale(float amax_b, float global_amax, float* scale_q, int* code) {
    const float one_e8 = 1e-8f;
    float pts = global_amax / 6.0f;
    if (pts <= one_e8) pts = one_e8;
    const float c0 = (float)(E4M3_MIN_SUBNORMAL / 448.0);
    const float min_value = c0 * pts;
    float sb = amax_b / 6.0f;
    if (sb <= min_value) sb = min_value;
    const float f = 448.0f / pts;
    *code = o_e4m3_round(sb * f);
    *scale_q = o_e4m3_val(*code) / f;
}

int o_fake_quantize_nvfp4_static(const void* x, int dt, int64_t rows, int64_t K,
                                 const float* block_amax, float global_amax, void* y) {
    if (K % 16 != 0) return -1;
    int64_t nblocks = rows * K / 16;
    for (int64_t b = 0; b < nblocks; ++b) {
        float scale_q;
        int code;
        o_nvfp4_static_scale(block_amax[b], global_amax, &scale_q, &code);
        for (int j = 0; j < 16; ++j) {
            float q = load_elem(x, dt, b * 16 + j) / scale_q;
            float w = o_e2m1_val(o_e2m1_round(q));
            store_elem(y, dt, b * 16 + j, w * scale_q);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* MXFP4 ([MX] quantize_mxfp4 / dequantize_mxfp4)                            */
/* ------------------------------------------------------------------------ */

/* Block scale exponent 2**(floor(log2(amax)) - 2) ([MX] quantize_mxfp4).
 * READING: amax == 0 takes the smallest e8m0 exponent, -127; the exponent is
 * clamped to the e8m0 range [-127, 127]. */
static int mxfp4_block_exponent(float amax_b) {
    int e = (amax_b == 0.0f) ? -127 : o_floor_log2(amax_b) - 2;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

int o_quantize_mxfp4(const void* x, int dt, int64_t rows, int64_t K, uint8_t* packed,
                     uint8_t* scales) {
    if (K % 32 != 0) return -1;
    int64_t nblocks = rows * K / 32;
    for (int64_t b = 0; b < nblocks; ++b) {
        float amax_b = block_amax(x, dt, b * 32, 32);
        int e = mxfp4_block_exponent(amax_b);
        scales[b] = (uint8_t)(e + 127);
        float scale = ldexpf(1.0f, e);
        for (int j = 0; j < 32; ++j) {
            float q = load_elem(x, dt, b * 32 + j) / scale;
            put_nibble(packed, b * 32 + j, o_e2m1_round(q));
        }
    }
    return 0;
}

/* value = e2m1 * 2**(scale code - 127) ([MX] dequantize_mxfp4). */
int o_dequantize_mxfp4(const uint8_t* packed, const uint8_t* scales, int64_t rows, int64_t K,
                       void* y, int dt) {
    if (K % 32 != 0) return -1;
    for (int64_t i = 0; i < rows * K; ++i) {
        float v = o_e2m1_val(get_nibble(packed, i));
        float val = v * o_e8m0_val(scales[i / 32]);
        store_elem(y, dt, i, val);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* MXFP8 ([MO] is_mxfp(8), _real_quantize: num_bits (4, 3), scale_bits        */
/* (8, 0), block 32)                                                          */
/* ------------------------------------------------------------------------ */

/* READING: the pages name MXFP8 (e4m3 elements, an e8m0 scale per block of
 * 32) but do not print its quantize body.  The scale follows [MX]
 * quantize_mxfp4's rule with the element format's largest binary exponent in
 * place of e2m1's: 2**(floor(log2(amax)) - 8), since E4M3_MAX = 448 =
 * 1.75 * 2**8 as E2M1_MAX = 6 = 1.5 * 2**2.  amax == 0 and the e8m0 range
 * clamp as in MXFP4.  amax / scale lies in [256, 512), so the top of a block
 * can exceed 448 and saturates there (e4m3_round saturates). */
static int mxfp8_block_exponent(float amax_b) {
    int e = (amax_b == 0.0f) ? -127 : o_floor_log2(amax_b) - 8;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

int o_quantize_mxfp8(const void* x, int dt, int64_t rows, int64_t K, uint8_t* codes,
                     uint8_t* scales) {
    if (K % 32 != 0) return -1;
    int64_t nblocks = rows * K / 32;
    for (int64_t b = 0; b < nblocks; ++b) {
        int e = mxfp8_block_exponent(block_amax(x, dt, b * 32, 32));
        scales[b] = (uint8_t)(e + 127);
        float scale = ldexpf(1.0f, e);
        for (int j = 0; j < 32; ++j)
            codes[b * 32 + j] = (uint8_t)o_e4m3_round(load_elem(x, dt, b * 32 + j) / scale);
    }
    return 0;
}

/* value = e4m3 * 2**(scale code - 127). */
int o_dequantize_mxfp8(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t K,
                       void* y, int dt) {
    if (K % 32 != 0) return -1;
    for (int64_t i = 0; i < rows * K; ++i) {
        float val = o_e4m3_val(codes[i]) * o_e8m0_val(scales[i / 32]);
        store_elem(y, dt, i, val);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* FP8 with a power-of-two block scale ([CQ] quantize_cache "fp8",           */
/* _power_of_two_ceiling)                                                    */
/* ------------------------------------------------------------------------ */

/* READING: scale = pow2ceil(amax / E_MAX) with the argument floored at the
 * smallest positive normal 2**-126 (the helper is defined on positive normal
 * values only; an all-zero block lands on the floor). */
static float pow2_block_scale(float amax_b, float fmt_max) {
    float a = amax_b / fmt_max;
    if (a < (float)F32_MIN_NORMAL) a = (float)F32_MIN_NORMAL;
    return o_pow2_ceil(a);
}

/* Stored form: e4m3 codes, one byte per element, and the scale's exponent as
 * an e8m0 byte per block. */
int o_quantize_fp8(const void* x, int dt, int64_t rows, int64_t K, int block, uint8_t* codes,
                   uint8_t* scales) {
    if ((block != 16 && block != 32) || K % block != 0) return -1;
    int64_t nblocks = rows * K / block;
    for (int64_t b = 0; b < nblocks; ++b) {
        float p = pow2_block_scale(block_amax(x, dt, b * block, block), E4M3_MAX);
        scales[b] = (uint8_t)(o_floor_log2(p) + 127);
        for (int j = 0; j < block; ++j)
            codes[b * block + j] = (uint8_t)o_e4m3_round(load_elem(x, dt, b * block + j) / p);
    }
    return 0;
}

int o_dequantize_fp8(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t K,
                     int block, void* y, int dt) {
    if ((block != 16 && block != 32) || K % block != 0) return -1;
    for (int64_t i = 0; i < rows * K; ++i) {
        float val = o_e4m3_val(codes[i]) * o_e8m0_val(scales[i / block]);
        store_elem(y, dt, i, val);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* quantize_cache ([CQ] quantize_cache, _CacheQuantization)                  */
/* ------------------------------------------------------------------------ */

/* Fake-quant of [rows, C] in the input dtype: each row is zero-padded up to a
 * whole number of blocks ("a final partial group is zero-padded internally"),
 * quantized and dequantized in binary32, cast once to the dtype, and the pad
 * is dropped.  READINGS: fp8 uses scale pow2ceil(amax/448) with e4m3 values;
 * mxfp4 uses scale pow2ceil(amax/6) with e2m1 values (the page's only scale
 * helper is the power-of-two ceiling); nvfp4 uses the per-row NVFP4 rule over
 * the padded row.  The input is never modified. */
int o_quantize_cache(int fmt, int block, const void* x, void* y, int dt, int64_t rows, int64_t C) {
    if (block != 16 && block != 32) return -1;
    if (fmt != O_FMT_FP8 && fmt != O_FMT_MXFP4 && fmt != O_FMT_NVFP4) return -1;
    int64_t P = ((C + block - 1) / block) * block;
    float* row = (float*)malloc(sizeof(float) * (size_t)(P > 0 ? P : 1));
    float* out = (float*)malloc(sizeof(float) * (size_t)(P > 0 ? P : 1));
    if (!row || !out) { free(row); free(out); return -2; }
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < P; ++c) row[c] = (c < C) ? load_elem(x, dt, r * C + c) : 0.0f;
        float g = 0.0f;
        if (fmt == O_FMT_NVFP4) g = block_amax(row, O_F32, 0, P) / (E2M1_MAX * E4M3_MAX);
        for (int64_t b = 0; b < P / block; ++b) {
            float amax_b = block_amax(row, O_F32, b * block, block);
            float p = 0.0f, s = 0.0f, d = 0.0f;
            if (fmt == O_FMT_FP8) p = pow2_block_scale(amax_b, E4M3_MAX);
            else if (fmt == O_FMT_MXFP4) p = pow2_block_scale(amax_b, E2M1_MAX);
            else if (g != 0.0f) { s = o_e4m3_val(nvfp4_block_scale(amax_b, g)); d = s * g; }
            for (int j = 0; j < block; ++j) {
                float v = row[b * block + j];
                float dq;
                if (fmt == O_FMT_FP8) {
                    dq = o_e4m3_val(o_e4m3_round(v / p)) * p;
                } else if (fmt == O_FMT_MXFP4) {
                    dq = o_e2m1_val(o_e2m1_round(v / p)) * p;
                } else if (g == 0.0f) {
                    dq = 0.0f;
                } else {
                    float prod = o_e2m1_val(o_e2m1_round(v / d)) * s;
                    dq = prod * g;
                }
                out[b * block + j] = dq;
            }
        }
        for (int64_t c = 0; c < C; ++c) store_elem(y, dt, r * C + c, out[c]);
    }
    free(row);
    free(out);
    return 0;
}

/* Straight-through backward: the gradient passes unchanged
 * ([CQ] _CacheQuantization.backward). */
int o_quantize_cache_backward(const void* grad_out, void* grad_in, int dt, int64_t n) {
    size_t bytes = (size_t)n * (dt == O_BF16 ? 2 : 4);
    if (grad_in != grad_out) memmove(grad_in, grad_out, bytes);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* array helpers for the pins (elementwise, same scalar functions)           */
/* ------------------------------------------------------------------------ */

void o_e2m1_round_array(const float* q, uint8_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)o_e2m1_round(q[i]);
}
void o_e4m3_round_array(const float* x, uint8_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)o_e4m3_round(x[i]);
}
void o_f32_to_bf16_array(const float* x, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = o_f32_to_bf16(x[i]);
}
void o_pow2_ceil_array(const float* x, float* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = o_pow2_ceil(x[i]);
}
void o_floor_log2_array(const float* x, int32_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = o_floor_log2(x[i]);
}
