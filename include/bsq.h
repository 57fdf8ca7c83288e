/*
 * bsq.h -- C ABI of libbsq: block-scaled microscaling quantization for
 * NVIDIA B200 (sm_100a).
 *
 * Formats (NeMo AutoModel API pages "nemo_automodel.components.quantization.nvfp4",
 * "...quantization.mxfp4" and "...models.deepseek_v41.quantization"; the
 * ModelOpt tensor_quantizer page for MXFP8 and the static two-level NVFP4
 * quantizer; the NeMo AutoModel model-filter page for the NVFP4 KV cache):
 *   NVFP4 -- e2m1 codes, one float8_e4m3fn scale per 16 columns and one fp32
 *            scale per row (or per tensor, the ModelOpt checkpoint layout).
 *   MXFP4 -- e2m1 codes, one float8_e8m0fnu scale per 32 columns.
 *   MXFP8 -- float8_e4m3fn codes, one float8_e8m0fnu scale per 32 columns.
 *   FP8   -- float8_e4m3fn codes with a power-of-two block scale, stored as an
 *            e8m0 exponent byte per block.
 * Two e2m1 codes share a byte: the even column in the low nibble, the odd
 * column in the high nibble.
 *
 * Conventions for every entry point:
 *   - Tensors are contiguous and row-major; "rows" is the product of all
 *     leading dimensions and K (or C) the last dimension.
 *   - Every data pointer is a DEVICE pointer, owned by the caller.  The
 *     library never allocates or frees device memory and keeps no device
 *     data between calls (the one exception, the file-scope scratch of
 *     bsq_quantize_nvfp4_tensor_noalloc, is described there); it caches only
 *     host-side facts (SM count, occupancy, the tensor-map encoder).  Outputs
 *     are written in place, so buffer addresses stay stable.  Once an entry
 *     point has run on a device outside any stream capture (which fills
 *     those host-side caches), its later calls may be captured into a CUDA
 *     graph on the caller's stream and replayed.  Inputs are never
 *     modified, except that
 *     bsq_fake_quantize_nvfp4_static may be asked to write over its input.
 *   - Work is enqueued on `stream` and is asynchronous.  Only argument
 *     validation runs on the host; a rejected call launches nothing.
 *   - Return value: BSQ_OK, or an error code; bsq_last_error() returns a
 *     thread-local description of the last failure.
 *   - bf16 tensors are passed as their 16-bit patterns.
 *   - NaN or infinite inputs are outside the contract: the kernels finish and
 *     the outputs are unspecified.
 */
#ifndef BSQ_H
#define BSQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t; NULL is the legacy default stream. */
typedef void* bsq_stream_t;

typedef enum {
    BSQ_OK = 0,
    BSQ_ERR_INVALID_ARG = 1, /* null pointer, negative size, K not a whole number of blocks, ... */
    BSQ_ERR_UNSUPPORTED = 2, /* dtype / format / block combination not implemented */
    BSQ_ERR_CUDA = 3,        /* a CUDA runtime or driver call failed (see bsq_last_error) */
    BSQ_ERR_DEVICE = 4       /* a kernel reported bad data through its device error word */
} bsq_status;

typedef enum { BSQ_BF16 = 0, BSQ_FP32 = 1 } bsq_dtype;
typedef enum { BSQ_FP8 = 0, BSQ_MXFP4 = 1, BSQ_NVFP4 = 2, BSQ_MXFP8 = 3 } bsq_format;
typedef enum { BSQ_FWD = 0, BSQ_BWD = 1 } bsq_dir;

/* Bits of the device error word written by bsq_grouped_mm_fp4. */
#define BSQ_DEVERR_BAD_OFFS 1u  /* offs not non-decreasing, negative, or offs[E-1] > T */
#define BSQ_DEVERR_TIMEOUT 2u   /* a pipeline wait gave up after its time limit (1 s, or BSQ_GMM_WAIT_NS) */

const char* bsq_status_string(bsq_status s);
const char* bsq_last_error(void);
int bsq_version(void);

/* Index-check counters of the bounds-checking build (compiled with
 * -DBSQ_DEBUG, shipped as libbsq_debug.so; the quantization pages have no
 * counterpart: this is a diagnostic of the library itself).  In that build
 * every checked device access first tests its index against the extent the
 * kernel was given; a failing check skips the access (no trap) and is
 * counted.  Synchronises the current device, stores the number of failed
 * checks since the previous call in *count and the first one's code in
 * *first_code ((source file id << 16) | line; 0 when none), and clears them.
 * In a normal build: BSQ_ERR_UNSUPPORTED, with *count = *first_code = 0. */
bsq_status bsq_debug_counters(uint32_t* count, uint32_t* first_code);

/* ---------------------------------------------------------------- NVFP4 --
 * nvfp4 page, quantize_nvfp4: along the last dim (K % 16 == 0, else
 * BSQ_ERR_INVALID_ARG -- the page's _check_last_dim), ModelOpt convention
 *   global      = amax(row) / (6 * 448)            (row_scale_in == NULL)
 *   block_scale = e4m3(amax(block) / 6 / global)    floored at 2**-9 before the cast
 *   code        = round_to_e2m1(w / (block_scale * global))
 * e4m3 and e2m1 rounding is to nearest, ties to even, saturating.  An all-zero
 * row (or a given row scale of 0) yields scale bytes 0x00 and codes 0.
 *   x             [rows, K] bf16 or fp32 (xt)
 *   row_scale_in  [rows] fp32 row scales to use instead of the amax rule, or NULL
 *   packed        [rows, K/2] uint8 out
 *   scales_e4m3   [rows, K/16] float8_e4m3fn out
 *   row_scale_out [rows] fp32 out (the row scale used; may equal row_scale_in) */
bsq_status bsq_quantize_nvfp4(const void* x, bsq_dtype xt, int64_t rows, int64_t K,
                              const float* row_scale_in, uint8_t* packed, uint8_t* scales_e4m3,
                              float* row_scale_out, bsq_stream_t stream);

/* nvfp4 page, quantize_nvfp4_modelopt: one tensor scale amax(x) / (6 * 448)
 * for the whole [rows, K] matrix (the checkpoint's weight_scale_2), then the
 * per-row algorithm above with that scale on every row.  Two passes over x.
 *   tensor_scale_out  device fp32 scalar out
 *   scratch           caller-owned device buffer of at least
 *                     bsq_nvfp4_tensor_scratch_bytes(rows, K) bytes, 16-byte
 *                     aligned; it holds per-block partial maxima between the
 *                     two passes and needs no initialisation. */
size_t bsq_nvfp4_tensor_scratch_bytes(int64_t rows, int64_t K);
bsq_status bsq_quantize_nvfp4_tensor(const void* x, bsq_dtype xt, int64_t rows, int64_t K,
                                     uint8_t* packed, uint8_t* scales_e4m3, float* tensor_scale_out,
                                     void* scratch, size_t scratch_bytes, bsq_stream_t stream);

/* Same computation and outputs as bsq_quantize_nvfp4_tensor, for callers
 * that cannot provide a scratch buffer -- e.g. a serving engine that reserves
 * all device memory at start-up and allows no allocation afterwards, or a
 * plain C caller without a device allocator.  (The quantization pages have no
 * counterpart: this is a property of the library, not of the method.)
 *   - Allocates nothing: the partial maxima live in a 16 KiB array inside the
 *     library (4096 floats), held on every GPU that loads it until exit.
 *   - Shapes whose first pass would need more than 4096 partial maxima
 *     (only possible on a GPU with more than 512 SMs) are rejected with
 *     BSQ_ERR_UNSUPPORTED.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  The address is kept for the rest of the
 *     process: after cudaDeviceReset (or anything else that destroys and
 *     re-creates the device's primary context) it no longer names the array,
 *     so do not call this entry point on that device again in the process.
 *   - All calls share the one array: calls whose kernels overlap on the GPU
 *     (concurrent streams) race and give wrong results.  Serialise them.
 *     Nothing needs clearing between calls. */
bsq_status bsq_quantize_nvfp4_tensor_noalloc(const void* x, bsq_dtype xt, int64_t rows, int64_t K,
                                             uint8_t* packed, uint8_t* scales_e4m3, float* tensor_scale_out,
                                             bsq_stream_t stream);

/* nvfp4 page, dequantize_nvfp4: y = e2m1 * float(e4m3) * row_scale with
 * binary32 intermediates left to right and one final rounding to yt.
 *   packed [rows, K/2], scales_e4m3 [rows, K/16], row_scale [rows] fp32,
 *   y [rows, K] bf16 or fp32 (yt). */
bsq_status bsq_dequantize_nvfp4(const uint8_t* packed, const uint8_t* scales_e4m3,
                                const float* row_scale, int64_t rows, int64_t K, void* y,
                                bsq_dtype yt, bsq_stream_t stream);

/* ----------------------------------------------- paged NVFP4 KV cache ---
 * NeMo AutoModel model-filter page, dequantize_kv_cache: a list of nblocks
 * quantized blocks, block b holding block_tokens * heads rows of 128 values
 * (row = token-in-block * heads + head):
 *   values[b]  e2m1 codes [rows, 64] (two per byte, even column low nibble)
 *   scales[b]  e4m3 scales [rows, 8] (row-major; the pages' swizzled
 *              from_blocked layout is not defined there)
 *   amax[b]    one fp32; the block's global scale is amax / (6 * 448)
 * Output y [1, nblocks * block_tokens, heads, 128] (bf16 or fp32, 16-byte
 * aligned): token t of block b is token b * block_tokens + t, each value
 * (e2m1 * e4m3) * g in binary32 with one final rounding to yt.
 * values, scales and amax are device arrays of nblocks device pointers
 * (8-byte aligned arrays; the pointed-to blocks may have any alignment).
 * One launch for all blocks.  Errors: BSQ_ERR_INVALID_ARG for negative
 * sizes, null or misaligned arrays/output; BSQ_ERR_UNSUPPORTED for more than
 * 2**32 output items in all (an item is 8 bf16 or 4 fp32 outputs) or more
 * than 2**32 outputs in one block.  No blocks, or empty blocks: nothing. */
bsq_status bsq_dequantize_kv_cache_nvfp4(const uint8_t* const* values, const uint8_t* const* scales,
                                         const float* const* amax, int64_t nblocks, int64_t block_tokens,
                                         int64_t heads, void* y, bsq_dtype yt, bsq_stream_t stream);

/* ------------------------------------------- static two-level NVFP4 -----
 * ModelOpt tensor_quantizer page, StaticBlockScaleQuantizer (two-level
 * scaling with an FP8-quantized block scale): fake-quant of x [rows, K]
 * (K % 16 == 0) with a calibrated amax per 16-element block and a global amax A:
 *   pts = A / 6 (1e-8 where A / 6 <= 1e-8),  min_value = (2**-9 / 448) * pts,
 *   sb  = amax_b / 6 (min_value where amax_b / 6 <= min_value),
 *   sq  = e4m3(sb * 448 / pts) / (448 / pts),   y = e2m1(x / sq) * sq,
 * binary32 with one rounding per operation in this order, one final rounding
 * to t.  The pages do not print scaled_e4m3: the 448 / pts map and its
 * inverse as a division by the same factor are this library's reading.
 *   x, y [rows, K] bf16 or fp32 (t), 16-byte aligned; y == x (in place) is
 *   allowed, any other overlap is rejected.  block_amax [rows, K/16] fp32 and
 *   global_amax (one fp32) are device pointers.  The straight-through
 *   backward is the identity: use the gradient as is. */
bsq_status bsq_fake_quantize_nvfp4_static(const void* x, bsq_dtype t, int64_t rows, int64_t K,
                                          const float* block_amax, const float* global_amax, void* y,
                                          bsq_stream_t stream);

/* ---------------------------------------------------------------- MXFP4 --
 * mxfp4 page, quantize_mxfp4: K % 32 == 0; per 32-block scale
 * 2**(floor(log2(amax)) - 2) (exact floor; an all-zero block takes 2**-127;
 * exponent clamped to [-127, 127]), stored as the e8m0 byte exponent + 127;
 * code = round_to_e2m1(w / scale).
 *   x [rows, K] bf16 or fp32; packed [rows, K/2] (int8 container, same bits);
 *   scales_e8m0 [rows, K/32]. */
bsq_status bsq_quantize_mxfp4(const void* x, bsq_dtype xt, int64_t rows, int64_t K,
                              uint8_t* packed, uint8_t* scales_e8m0, bsq_stream_t stream);

/* mxfp4 page, dequantize_mxfp4: y = e2m1 * 2**(scale byte - 127) (exact;
 * scale byte 0xFF is NaN). */
bsq_status bsq_dequantize_mxfp4(const uint8_t* packed, const uint8_t* scales_e8m0, int64_t rows,
                                int64_t K, void* y, bsq_dtype yt, bsq_stream_t stream);

/* ---------------------------------------------------------------- MXFP8 --
 * ModelOpt tensor_quantizer page, is_mxfp(8) / _real_quantize: e4m3 elements
 * with one e8m0 scale per 32-column block.  The pages do not print the
 * quantize body; the scale carries the mxfp4 page's rule over to e4m3's
 * largest exponent: 2**(floor(log2(amax)) - 8) (exact floor; an all-zero block
 * takes 2**-127; exponent clamped to [-127, 127]), stored as exponent + 127;
 * code = e4m3 round-to-nearest-even of w / scale, saturating at +-448 (the
 * block maximum lands in [256, 512) before rounding).  K % 32 == 0.
 *   x [rows, K] bf16 or fp32 (16-byte aligned); codes_e4m3 [rows, K] uint8
 *   (8-byte aligned); scales_e8m0 [rows, K/32]. */
bsq_status bsq_quantize_mxfp8(const void* x, bsq_dtype xt, int64_t rows, int64_t K,
                              uint8_t* codes_e4m3, uint8_t* scales_e8m0, bsq_stream_t stream);

/* y = e4m3 * 2**(scale byte - 127) (exact in fp32; scale byte 0xFF and codes
 * 0x7F / 0xFF are NaN).  y [rows, K] bf16 or fp32 (16-byte aligned). */
bsq_status bsq_dequantize_mxfp8(const uint8_t* codes_e4m3, const uint8_t* scales_e8m0, int64_t rows,
                                int64_t K, void* y, bsq_dtype yt, bsq_stream_t stream);

/* ------------------------------------------------------------------ FP8 --
 * Stored form of the cache page's "fp8" representation: block of `block`
 * (16 or 32) columns, scale p = pow2ceil(max(amax / 448, 2**-126))
 * (deepseek_v41 quantization page, _power_of_two_ceiling), e4m3 code =
 * round(x / p) to nearest even; the scale is stored as log2(p) + 127.
 *   codes_e4m3 [rows, K] uint8 out; scales_e8m0 [rows, K/block] out. */
bsq_status bsq_quantize_fp8(const void* x, bsq_dtype xt, int64_t rows, int64_t K, int block,
                            uint8_t* codes_e4m3, uint8_t* scales_e8m0, bsq_stream_t stream);

/* y = float(e4m3) * 2**(scale byte - 127), one rounding to yt. */
bsq_status bsq_dequantize_fp8(const uint8_t* codes_e4m3, const uint8_t* scales_e8m0, int64_t rows,
                              int64_t K, int block, void* y, bsq_dtype yt, bsq_stream_t stream);

/* ------------------------------------------------------- quantize_cache --
 * deepseek_v41 quantization page, quantize_cache / _CacheQuantization.forward:
 * quantize then dequantize every group of `block` consecutive channels of the
 * [rows, C] input, returning a new tensor of the input dtype.  Any C >= 0: a
 * final partial group is zero-padded internally.  Scale rules:
 *   BSQ_FP8   -- p = pow2ceil(max(amax/448, 2**-126)), e4m3 values
 *   BSQ_MXFP4 -- p = pow2ceil(max(amax/6,   2**-126)), e2m1 values
 *   BSQ_NVFP4 -- the per-row NVFP4 rule above over the zero-padded row
 * block is 16 or 32.  x and y must not overlap (the input is never modified). */
bsq_status bsq_quantize_cache(bsq_format fmt, int block, const void* x, void* y, bsq_dtype t,
                              int64_t rows, int64_t C, bsq_stream_t stream);

/* _CacheQuantization.backward: the straight-through gradient is the identity.
 * grad_in == grad_out is a no-op; otherwise one device-to-device copy of
 * n_elems elements of dtype t. */
bsq_status bsq_quantize_cache_backward(const void* grad_out, void* grad_in, bsq_dtype t,
                                       int64_t n_elems, bsq_stream_t stream);

/* ------------------------------------------------------- grouped GEMM ----
 * nvfp4 page NVFP4GroupedMM / mxfp4 page MXFP4GroupedMM, with the weights
 * dequantized on the fly inside the kernel (never materialised in HBM):
 *   expert e owns rows [offs[e-1], offs[e]) of the activations (offs[-1] = 0);
 *   BSQ_FWD: out[t, :]    = x[t, :]        @ W_e^T   a = x [T, K],        out [T, N]
 *   BSQ_BWD: grad_x[t, :] = grad_out[t, :] @ W_e     a = grad_out [T, N], out [T, K]
 * with W_e the dequantized [N, K] weight.  No weight gradient (frozen base).
 *   fmt         BSQ_MXFP4 (scales e8m0 [E, N, K/32], row_scale NULL) or
 *               BSQ_NVFP4 (scales e4m3 [E, N, K/16], row_scale fp32 [E, N])
 *   a, out      bf16; fp32 accumulation on the tensor cores
 *   packed      uint8 [E, N, K/2]
 *   offs        int32 [E] cumulative token counts, on the device
 *   err         device uint32 word; the caller zeroes it before the call and
 *               reads it after synchronising: BSQ_DEVERR_* bits.  With a bad
 *               offs the output is undefined.
 * Every wait between the kernel's pipeline roles gives up after 1 s: the
 * kernel then sets BSQ_DEVERR_TIMEOUT, lets its outstanding loads and MMAs
 * finish, frees its tensor memory and returns (the output is undefined, the
 * context stays usable).  The environment variable BSQ_GMM_WAIT_NS, read at
 * every call, sets another limit in nanoseconds (a test hook: a limit of a
 * few ns makes the waits run out).
 * Rows at or past offs[E-1] are written as zero.  Requirements: the output
 * width (N for BSQ_FWD, K for BSQ_BWD) a multiple of 128 and K, N multiples
 * of 64; E <= 1024; a, packed, out and row_scale 16-byte aligned.  Other
 * shapes return BSQ_ERR_UNSUPPORTED. */
bsq_status bsq_grouped_mm_fp4(bsq_format fmt, bsq_dir dir, const void* a, const uint8_t* packed,
                              const uint8_t* scales, const float* row_scale, const int32_t* offs,
                              int E, int64_t T, int64_t N, int64_t K, void* out, uint32_t* err,
                              bsq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BSQ_H */
