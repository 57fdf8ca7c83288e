// grouped_mm.cu -- fused-dequant grouped MoE GEMM on the sm_100a tensor cores.
//
// nvfp4 page NVFP4GroupedMM / mxfp4 page MXFP4GroupedMM: expert e owns rows
// [offs[e-1], offs[e]) of the activations; forward out = x @ W_e^T, backward
// grad_x = grad_out @ W_e, with W_e stored packed (e2m1 + block scales) and
// never materialised in HBM: producer warps dequantize each weight tile into
// shared memory as bf16, in exactly the 128-byte-swizzled layout the tensor
// core reads, and tcgen05 MMAs accumulate fp32 in tensor memory.
//
// The MMA computes the transposed product, D[feature, token]: the weight tile
// (128 output features) is the M = 128 operand A and the expert's tokens (up
// to 256, rounded up to 16) are the N operand B.  Dequantization work per
// tensor-core operation is set by the weight rows of a tile, so this halves it
// against a 256-feature by 128-token tile, and a short expert pads its token
// count only to a multiple of 16.
//
// Persistent, warp-specialised CTA (one per SM, 448 threads):
//   warps 0-3   epilogue: tensor memory -> registers (x row scale for NVFP4
//               forward) -> bf16 -> global; lane = feature, so each store of
//               a token's 32 features is one coalesced 64-byte row piece
//   warps 4-11  A producers: packed weights + scales from global (several
//               k-steps in flight), e2m1 -> bf16 by byte permutes, times the
//               block scale (bf16x2 multiply), swizzled 16-byte shared stores
//   warp 12     B producer: TMA loads of 64-token x 64-k activation boxes
//   warp 13     tensor-memory allocation and the single MMA-issuing thread
// Tile = 128 features x up to 256 tokens, k-step 64; separate rings of 5
// dequantized-weight slots (16 KiB) and 4 activation slots (32 KiB);
// two 256-column fp32 accumulators in tensor memory so the epilogue of one
// tile overlaps the main loop of the next.  Tiles are numbered (expert token
// tile, feature tile) with the feature tile fastest, dealt round-robin to the
// CTAs; every CTA derives the tile table from offs on the device.
//
// Forward: A = 128 weight rows x 64 k (K-major).  Backward: A = W^T, 128 k
// columns x 64 weight rows of the contraction (MN-major); NVFP4's row scale
// lies on the contraction there and is folded into the dequantized weight.
//
// Every mbarrier wait gives up after about a second: the thread records
// BSQ_DEVERR_TIMEOUT in the error word and raises a CTA-wide abort flag, all
// roles wind down, outstanding TMA loads and MMAs are drained (again with a
// time limit) and tensor memory is freed before the CTA exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "formats.cuh"
#include "host_util.h"
#include "tcgen05.cuh"

namespace bsq {
using namespace sm100;

namespace gmm {

constexpr int WM = 128;   // features per tile (MMA M)
constexpr int TN = 256;   // tokens per tile at most (MMA N)
constexpr int BK = 64;
constexpr int WSTAGES = 5;  // dequantized-weight ring (16 KiB slots)
constexpr int XSTAGES = 4;  // activation ring (32 KiB slots)
constexpr int XBOX = 64;  // token rows per TMA box
constexpr int kEpiWarps = 4, kDqWarps = 8;
constexpr int kTmaWarp = kEpiWarps + kDqWarps;  // 12
constexpr int kMmaWarp = kTmaWarp + 1;          // 13
constexpr int kThreads = (kMmaWarp + 1) * 32;   // 448
constexpr uint32_t kWStage = WM * BK * 2;       // 16 KiB dequantized weights
constexpr uint32_t kXStage = TN * BK * 2;       // 32 KiB activations
constexpr uint32_t kXBoxBytes = XBOX * BK * 2;  // 8 KiB
constexpr int kMaxExperts = 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr int kPrefetch = 4;  // k-steps of packed weights in flight per producer thread

constexpr size_t kBarOffset = (size_t)WSTAGES * kWStage + (size_t)XSTAGES * kXStage;
constexpr int kNumBars = 2 * WSTAGES + 2 * XSTAGES + 5;  // w_full/empty, x_full/empty, acc_full[2], acc_empty[2], drain
constexpr size_t kSmemBytes = 1024 /* alignment slack */ + kBarOffset + kNumBars * 8 + 16 /* tmem slot, flags */ +
                              4 * (2 * kMaxExperts + 2);

struct Args {
    const uint8_t* packed;
    const uint8_t* scales;
    const float* row_scale;
    const int32_t* offs;
    uint16_t* out;
    uint32_t* err;
    int E, T, N, K;
};

struct Tile {
    int e;      // expert
    int tok0;   // first token row
    int ntok;   // tokens in the tile (1..256)
    int f0;     // first feature (output column) of the tile
};

struct Shared {
    uint8_t* w;
    uint8_t* x;
    uint64_t* w_full;
    uint64_t* w_empty;
    uint64_t* x_full;
    uint64_t* x_empty;
    uint64_t* acc_full;
    uint64_t* acc_empty;
    uint64_t* drain;
    uint32_t* tmem_slot;
    volatile int* abort;
    int* tt_prefix;  // [E + 1] first token tile of each expert
    int* seg;        // [E + 1] seg[e] = first row of expert e, seg[E] = offs[E-1]
};

__device__ __forceinline__ Shared carve(uint8_t* raw) {
    Shared s;
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    s.w = base;
    s.x = base + WSTAGES * kWStage;
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + kBarOffset);
    s.w_full = bars;
    s.w_empty = bars + WSTAGES;
    s.x_full = bars + 2 * WSTAGES;
    s.x_empty = bars + 2 * WSTAGES + XSTAGES;
    s.acc_full = bars + 2 * WSTAGES + 2 * XSTAGES;
    s.acc_empty = s.acc_full + 2;
    s.drain = s.acc_empty + 2;
    s.tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
    s.abort = reinterpret_cast<volatile int*>(s.tmem_slot + 1);
    s.tt_prefix = reinterpret_cast<int*>(s.tmem_slot + 4);
    s.seg = s.tt_prefix + kMaxExperts + 1;
    return s;
}

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const Shared& sh, uint32_t* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*sh.abort) return false;
        if (globaltimer_ns() - t0 > kWaitNs) {
            *sh.abort = 1;
            atomicOr(err, (uint32_t)BSQ_DEVERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ Tile decode_tile(int t, int f_tiles, int E, const Shared& sh) {
    const int tg = t / f_tiles;
    const int ft = t - tg * f_tiles;
    int lo = 0, hi = E - 1;  // last expert whose first token tile is <= tg
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sh.tt_prefix[mid] <= tg) lo = mid;
        else hi = mid - 1;
    }
    Tile ti;
    ti.e = lo;
    ti.tok0 = sh.seg[lo] + (tg - sh.tt_prefix[lo]) * TN;
    ti.ntok = min(TN, sh.seg[lo + 1] - ti.tok0);
    ti.f0 = ft * WM;
    return ti;
}

// e2m1 x 8 (one 32-bit word, code i in nibble i) -> 4 words of bf16x2, by
// byte permutes over register-resident tables of the bf16 encodings of the
// eight magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}; the sign bit of each code
// picks the negative table.  (Code 8 becomes -0.0, which adds nothing to a
// dot product.)
__device__ __forceinline__ void e2m1x8_to_bf16(uint32_t w, uint32_t out[4]) {
    const uint32_t TL0 = 0xC0800000u, TL1 = 0xC0804000u;   // low bytes, magnitudes 0-3 / 4-7
    const uint32_t THP0 = 0x3F3F3F00u, THP1 = 0x40404040u; // high bytes, positive
    const uint32_t THN0 = 0xBFBFBF80u, THN1 = 0xC0C0C0C0u; // high bytes, negative
    const uint32_t w4 = w << 4;
    const uint32_t selA = w & 0x7777u, selB = (w >> 16) & 0x7777u;
    const uint32_t mA = prmt(w4, w, 0xD9C8u);  // 0xFF bytes where codes 0..3 are negative
    const uint32_t mB = prmt(w4, w, 0xFBEAu);  // codes 4..7
    const uint32_t loA = prmt(TL0, TL1, selA), loB = prmt(TL0, TL1, selB);
    const uint32_t hiA = (prmt(THP0, THP1, selA) & ~mA) | (prmt(THN0, THN1, selA) & mA);
    const uint32_t hiB = (prmt(THP0, THP1, selB) & ~mB) | (prmt(THN0, THN1, selB) & mB);
    out[0] = prmt(loA, hiA, 0x5140u);
    out[1] = prmt(loA, hiA, 0x7362u);
    out[2] = prmt(loB, hiB, 0x5140u);
    out[3] = prmt(loB, hiB, 0x7362u);
}

__device__ __forceinline__ uint32_t bf16_bits_exact(float f) { return __float_as_uint(f) >> 16; }

// Block scale as a bf16x2 multiplier.  MXFP4: 2**(code - 127) (exact in bf16,
// code 0 is the subnormal 2**-127).  NVFP4: the e4m3 value (exact in bf16),
// times the row scale g when it is folded in (one bf16 rounding).
template <int FMT, bool FOLD_G>
__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t code, float g) {
    uint32_t b;
    if (FMT == BSQ_MXFP4) {
        code &= 0xFFu;
        b = (code == 0u) ? 0x0040u : (code == 0xFFu ? 0x7FC0u : (code << 7));
    } else {
        uint32_t e = (code >> 3) & 15u, m = code & 7u;
        float v = (e == 0u) ? (float)m * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
        if (e == 15u && m == 7u) v = __uint_as_float(0x7FC00000u);
        if (FOLD_G) {
            __nv_bfloat16 h = __float2bfloat16_rn(v * g);
            b = *reinterpret_cast<uint16_t*>(&h);
        } else {
            b = bf16_bits_exact(v);
        }
    }
    return b | (b << 16);
}

// One producer thread's share of a k-step: 32 consecutive packed weights.
struct Unit {
    uint4 pk;
    uint32_t sc;  // MXFP4: one e8m0 byte; NVFP4: two e4m3 bytes (16-column halves)
    float g;      // NVFP4 backward row scale
};

// Forward: unit u = (feature row u/2 of the tile, k half u%2).  Backward:
// unit u = (contraction row u/4 of the k-step, 32-column segment u%4 of the
// tile's 128 k columns).
template <int FMT, int DIR>
__device__ __forceinline__ void load_unit(Unit& u, const Args& a, const Tile& ti, int ks, int unit) {
    int64_t row;
    int kcol;  // first weight column (k) of the unit's 32 elements
    if (DIR == BSQ_FWD) {
        row = (int64_t)ti.e * a.N + ti.f0 + (unit >> 1);
        kcol = ks * BK + (unit & 1) * 32;
    } else {
        row = (int64_t)ti.e * a.N + ks * BK + (unit >> 2);
        kcol = ti.f0 + (unit & 3) * 32;
    }
    u.pk = __ldg(reinterpret_cast<const uint4*>(a.packed + row * (a.K / 2) + kcol / 2));
    if (FMT == BSQ_MXFP4) {
        u.sc = __ldg(a.scales + row * (a.K / 32) + kcol / 32);
        u.g = 1.0f;
    } else {
        u.sc = __ldg(reinterpret_cast<const unsigned short*>(a.scales + row * (a.K / 16) + kcol / 16));
        u.g = (DIR == BSQ_BWD) ? __ldg(a.row_scale + row) : 1.0f;
    }
}

// Decode a unit into 16 words of bf16x2 (four 16-byte chunks), block scale applied.
template <int FMT, int DIR>
__device__ __forceinline__ void decode_unit(const Unit& u, uint32_t (&v)[16]) {
    uint32_t s_lo, s_hi;
    if (FMT == BSQ_MXFP4) {
        s_lo = s_hi = scale_bf16x2<FMT, false>(u.sc, 0.0f);
    } else {
        s_lo = scale_bf16x2<FMT, DIR == BSQ_BWD>(u.sc & 0xFFu, u.g);
        s_hi = scale_bf16x2<FMT, DIR == BSQ_BWD>(u.sc >> 8, u.g);
    }
    const uint32_t words[4] = {u.pk.x, u.pk.y, u.pk.z, u.pk.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t t[4];
        e2m1x8_to_bf16(words[i], t);
        const uint32_t sc = (i < 2) ? s_lo : s_hi;
#pragma unroll
        for (int j = 0; j < 4; ++j) v[4 * i + j] = mul_bf16x2(t[j], sc);
    }
}

// Write the decoded unit to its place in the swizzled operand tile.
template <int DIR>
__device__ __forceinline__ void store_unit(const uint32_t (&v)[16], uint32_t w_stage, int unit) {
    // 128-byte shared row of the unit and its first 16-byte chunk in that row
    uint32_t base;
    int r, c0;
    if (DIR == BSQ_FWD) {
        r = unit >> 1;  // K-major: one row per feature, 8-row atoms of 1 KiB
        c0 = (unit & 1) * 4;
        base = w_stage + (r >> 3) * 1024 + (r & 7) * 128;
    } else {
        r = unit >> 2;  // MN-major: one row per contraction index, 64-feature panels
        const int seg = unit & 3;
        c0 = (seg & 1) * 4;
        base = w_stage + (seg >> 1) * (BK * 128) + (r >> 3) * 1024 + (r & 7) * 128;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
        sts128(base + (uint32_t)(((c0 + i) ^ (r & 7)) << 4), v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}

template <int FMT, int DIR>
__global__ void __launch_bounds__(kThreads, 1) grouped_mm_kernel(const __grid_constant__ CUtensorMap tmap_x, Args args) {
    extern __shared__ uint8_t smem_raw[];
    const Shared sh = carve(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = args.E;
    const int f_tiles = (DIR == BSQ_FWD ? args.N : args.K) / WM;
    const int k_steps = (DIR == BSQ_FWD ? args.K : args.N) / BK;
    const int out_w = (DIR == BSQ_FWD ? args.N : args.K);

    if (threadIdx.x == 0) {
        for (int s = 0; s < WSTAGES; ++s) {
            mbar_init(&sh.w_full[s], kDqWarps);
            mbar_init(&sh.w_empty[s], 1);
        }
        for (int s = 0; s < XSTAGES; ++s) {
            mbar_init(&sh.x_full[s], 1);
            mbar_init(&sh.x_empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sh.acc_full[i], 1);
            mbar_init(&sh.acc_empty[i], kEpiWarps);
        }
        mbar_init(sh.drain, 1);
        fence_barrier_init();
        // tile table from offs; reject non-monotone / out-of-range offsets
        int prev = 0, total = 0, bad = 0;
        for (int e = 0; e < E; ++e) {
            const int o = args.offs[e];
            if (o < prev || o > args.T) bad = 1;
            sh.seg[e] = prev;
            sh.tt_prefix[e] = total;
            if (!bad) total += (o - prev + TN - 1) / TN;
            prev = o;
        }
        sh.seg[E] = bad ? 0 : prev;
        sh.tt_prefix[E] = total;
        sh.tmem_slot[1] = 0;  // abort flag
        sh.tmem_slot[2] = bad;
        sh.tmem_slot[3] = bad ? 0 : total;
        if (bad && blockIdx.x == 0) atomicOr(args.err, (uint32_t)BSQ_DEVERR_BAD_OFFS);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(sh.tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp == kTmaWarp && lane == 0) tma_prefetch_desc(&tmap_x);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_slot[0];
    const int bad = sh.tmem_slot[2];
    const int num_tiles = bad ? 0 : sh.tmem_slot[3] * f_tiles;

    if (warp < kEpiWarps) {
        // ---------------------------------------------------------- epilogue
        const int tid = threadIdx.x;  // 0..127
        if (!bad) {  // rows at or past offs[E-1] are zero
            const int tail0 = sh.seg[E];
            const int vec_per_row = out_w / 8;
            for (int r = tail0 + blockIdx.x; r < args.T; r += gridDim.x) {
                uint4* dst = reinterpret_cast<uint4*>(args.out + (int64_t)r * out_w);
                for (int v = tid; v < vec_per_row; v += kEpiWarps * 32) dst[v] = make_uint4(0, 0, 0, 0);
            }
        }
        const int q = warp;  // tensor-memory lane quadrant of this warp = features 32q..32q+31
        int tile_iter = 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++tile_iter) {
            const Tile ti = decode_tile(t, f_tiles, E, sh);
            const int acc = tile_iter & 1;
            if (!wait_bar(&sh.acc_full[acc], (tile_iter >> 1) & 1, sh, args.err)) break;
            tc_fence_after();
            const int f = ti.f0 + q * 32 + lane;
            float gf = 1.0f;
            if (FMT == BSQ_NVFP4 && DIR == BSQ_FWD) gf = __ldg(args.row_scale + (int64_t)ti.e * args.N + f);
            uint16_t* ocol = args.out + (int64_t)ti.tok0 * out_w + f;
            const int chunks = (ti.ntok + 15) >> 4;
#pragma unroll 1
            for (int c = 0; c < chunks; ++c) {
                uint32_t r[16];
                tmem_ld_32x32b_x16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * TN + c * 16), r);
                tmem_ld_wait();
                const int nv = min(16, ti.ntok - c * 16);
                uint16_t* p = ocol + (int64_t)(c * 16) * out_w;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    float v = __uint_as_float(r[j]);
                    if (FMT == BSQ_NVFP4 && DIR == BSQ_FWD) v *= gf;
                    const __nv_bfloat16 h = __float2bfloat16_rn(v);
                    if (j < nv) *p = *reinterpret_cast<const uint16_t*>(&h);
                    p += out_w;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.acc_empty[acc]);
        }
    } else if (warp < kTmaWarp) {
        // ------------------------------------------------- A (weight) producers
        const int dq = threadIdx.x - kEpiWarps * 32;  // 0..255 = unit index
        const uint32_t w_base = smem_u32(sh.w);
        int my_tiles = 0;
        if (num_tiles > (int)blockIdx.x) my_tiles = (num_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1;
        const int items = my_tiles * k_steps;
        // load cursor, kPrefetch k-steps ahead of the stores
        int lt = blockIdx.x, lks = 0;
        Tile lti;
        if (items > 0) lti = decode_tile(lt, f_tiles, E, sh);
        Unit buf[kPrefetch];
#pragma unroll
        for (int b = 0; b < kPrefetch; ++b) {
            if (b < items) {
                load_unit<FMT, DIR>(buf[b], args, lti, lks, dq);
                if (++lks == k_steps) {
                    lks = 0;
                    lt += gridDim.x;
                    if (lt < num_tiles) lti = decode_tile(lt, f_tiles, E, sh);
                }
            }
        }
        bool ok = true;
        for (int it = 0; it < items && ok; it += kPrefetch) {
#pragma unroll
            for (int b = 0; b < kPrefetch; ++b) {
                const int i = it + b;
                if (i < items && ok) {
                    // decode first (off the critical path), refill the buffer, then
                    // wait for the shared-memory slot and only store + signal
                    uint32_t v[16];
                    decode_unit<FMT, DIR>(buf[b], v);
                    if (i + kPrefetch < items) {
                        load_unit<FMT, DIR>(buf[b], args, lti, lks, dq);
                        if (++lks == k_steps) {
                            lks = 0;
                            lt += gridDim.x;
                            if (lt < num_tiles) lti = decode_tile(lt, f_tiles, E, sh);
                        }
                    }
                    const int s = i % WSTAGES;
                    if (!wait_bar(&sh.w_empty[s], ((i / WSTAGES) & 1) ^ 1, sh, args.err)) {
                        ok = false;
                    } else {
                        store_unit<DIR>(v, w_base + s * kWStage, dq);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sh.w_full[s]);
                    }
                }
            }
        }
    } else if (warp == kTmaWarp) {
        // ------------------------------------------- B (activation) producer
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                const Tile ti = decode_tile(t, f_tiles, E, sh);
                const int nbox = (ti.ntok + XBOX - 1) / XBOX;
                for (int ks = 0; ks < k_steps; ++ks, ++it) {
                    const int s = it % XSTAGES;
                    if (!wait_bar(&sh.x_empty[s], ((it / XSTAGES) & 1) ^ 1, sh, args.err)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sh.x_full[s], nbox * kXBoxBytes);
                    for (int b = 0; b < nbox; ++b)
                        tma_load_2d(sh.x + s * kXStage + b * kXBoxBytes, &tmap_x, &sh.x_full[s], ks * BK,
                                    ti.tok0 + b * XBOX);
                }
            }
            if (!ok) {
                // drain the loads still in flight into this CTA's shared memory
                for (int j = (it > XSTAGES ? it - XSTAGES : 0); j < it; ++j)
                    mbar_wait(&sh.x_full[j % XSTAGES], (j / XSTAGES) & 1, kWaitNs);
            }
        }
    } else {
        // ----------------------------------------------------------- MMA
        if (lane == 0) {
            const uint32_t w_base = smem_u32(sh.w), x_base = smem_u32(sh.x);
            int it = 0, tile_iter = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++tile_iter) {
                const Tile ti = decode_tile(t, f_tiles, E, sh);
                const uint32_t n_mma = (uint32_t)((ti.ntok + 15) & ~15);
                const uint32_t idesc = idesc_bf16_ab(WM, n_mma, DIR == BSQ_BWD ? 1u : 0u, 0u);
                const int acc = tile_iter & 1;
                if (!wait_bar(&sh.acc_empty[acc], ((tile_iter >> 1) & 1) ^ 1, sh, args.err)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * TN);
                for (int ks = 0; ks < k_steps; ++ks, ++it) {
                    const int sw = it % WSTAGES, sx = it % XSTAGES;
                    if (!wait_bar(&sh.w_full[sw], (it / WSTAGES) & 1, sh, args.err) ||
                        !wait_bar(&sh.x_full[sx], (it / XSTAGES) & 1, sh, args.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ws = w_base + sw * kWStage, xs = x_base + sx * kXStage;
#pragma unroll
                    for (int k16 = 0; k16 < BK / 16; ++k16) {
                        const uint64_t ad = (DIR == BSQ_FWD) ? smem_desc(ws + k16 * 32, 16, 1024)
                                                             : smem_desc(ws + k16 * 2048, BK * 128, 1024);
                        const uint64_t bd = smem_desc(xs + k16 * 32, 16, 1024);
                        mma_bf16_ss(d_tmem, ad, bd, idesc, (ks | k16) != 0 ? 1u : 0u);
                    }
                    mma_commit(&sh.w_empty[sw]);
                    mma_commit(&sh.x_empty[sx]);
                }
                if (ok) mma_commit(&sh.acc_full[acc]);
            }
            // every MMA this thread issued has completed once `drain` fires
            mma_commit(sh.drain);
            mbar_wait(sh.drain, 0, kWaitNs);
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace gmm

// ----------------------------------------------------------------- host -----

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn(bsq_status* st) {
    static std::mutex mu;
    static EncodeTiledFn fn = nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p) {
            *st = fail(BSQ_ERR_CUDA, "bsq_grouped_mm_fp4: cuTensorMapEncodeTiled unavailable (%s)",
                       cudaGetErrorString(e));
            return nullptr;
        }
        fn = (EncodeTiledFn)p;
    }
    *st = BSQ_OK;
    return fn;
}

template <int FMT, int DIR>
static bsq_status launch_gmm(const CUtensorMap& tmap, const gmm::Args& a, int grid, cudaStream_t st) {
    static std::mutex mu;
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    {
        std::lock_guard<std::mutex> lock(mu);
        if (dev >= 0 && dev < 64 && !attr_set[dev]) {
            cudaError_t e = cudaFuncSetAttribute(gmm::grouped_mm_kernel<FMT, DIR>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gmm::kSmemBytes);
            if (e != cudaSuccess)
                return fail(BSQ_ERR_CUDA, "bsq_grouped_mm_fp4: shared-memory opt-in failed (%s)", cudaGetErrorString(e));
            attr_set[dev] = true;
        }
    }
    gmm::grouped_mm_kernel<FMT, DIR><<<grid, gmm::kThreads, gmm::kSmemBytes, st>>>(tmap, a);
    return check_launch("bsq_grouped_mm_fp4");
}

}  // namespace bsq

using namespace bsq;

BSQ_API bsq_status bsq_grouped_mm_fp4(bsq_format fmt, bsq_dir dir, const void* a, const uint8_t* packed,
                                      const uint8_t* scales, const float* row_scale, const int32_t* offs, int E,
                                      int64_t T, int64_t N, int64_t K, void* out, uint32_t* err,
                                      bsq_stream_t stream) {
    const char* fn = "bsq_grouped_mm_fp4";
    if (fmt != BSQ_MXFP4 && fmt != BSQ_NVFP4) return fail(BSQ_ERR_UNSUPPORTED, "%s: format must be MXFP4 or NVFP4", fn);
    if (dir != BSQ_FWD && dir != BSQ_BWD) return fail(BSQ_ERR_INVALID_ARG, "%s: bad direction", fn);
    if (E < 1 || T < 0 || N <= 0 || K <= 0) return fail(BSQ_ERR_INVALID_ARG, "%s: bad sizes", fn);
    if (E > gmm::kMaxExperts) return fail(BSQ_ERR_UNSUPPORTED, "%s: at most %d experts", fn, gmm::kMaxExperts);
    if (T > (int64_t(1) << 30) || N > (int64_t(1) << 30) || K > (int64_t(1) << 30) || (int64_t)E * N > (int64_t(1) << 31))
        return fail(BSQ_ERR_UNSUPPORTED, "%s: sizes too large", fn);
    const int64_t out_w = (dir == BSQ_FWD) ? N : K, contr = (dir == BSQ_FWD) ? K : N;
    if (out_w % gmm::WM != 0 || contr % gmm::BK != 0 || K % 64 != 0 || N % 64 != 0)
        return fail(BSQ_ERR_UNSUPPORTED, "%s: needs the output width %% %d == 0 and K, N %% %d == 0", fn, gmm::WM,
                    gmm::BK);
    if (!err) return fail(BSQ_ERR_INVALID_ARG, "%s: null error word", fn);
    if (T == 0) return BSQ_OK;
    if (!a || !packed || !scales || !offs || !out || (fmt == BSQ_NVFP4 && !row_scale))
        return fail(BSQ_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (((uintptr_t)a % 16) || ((uintptr_t)packed % 16) || ((uintptr_t)out % 16) || ((uintptr_t)scales % 2) ||
        (row_scale && ((uintptr_t)row_scale % 16)))
        return fail(BSQ_ERR_INVALID_ARG, "%s: misaligned pointer", fn);

    bsq_status st;
    EncodeTiledFn encode = encode_fn(&st);
    if (!encode) return st;
    CUtensorMap tmap;
    const cuuint64_t dims[2] = {(cuuint64_t)contr, (cuuint64_t)T};
    const cuuint64_t strides[1] = {(cuuint64_t)contr * 2};
    const cuuint32_t box[2] = {(cuuint32_t)gmm::BK, (cuuint32_t)gmm::XBOX};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(BSQ_ERR_CUDA, "%s: cuTensorMapEncodeTiled failed (%d)", fn, (int)r);

    gmm::Args args;
    args.packed = packed;
    args.scales = scales;
    args.row_scale = row_scale;
    args.offs = offs;
    args.out = (uint16_t*)out;
    args.err = err;
    args.E = E;
    args.T = (int)T;
    args.N = (int)N;
    args.K = (int)K;
    const int64_t f_tiles = out_w / gmm::WM;
    const int64_t max_tiles = ((T + gmm::TN - 1) / gmm::TN + E) * f_tiles;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(max_tiles, sm_count()));
    cudaStream_t s = (cudaStream_t)stream;
    if (fmt == BSQ_MXFP4)
        return dir == BSQ_FWD ? launch_gmm<BSQ_MXFP4, BSQ_FWD>(tmap, args, grid, s)
                              : launch_gmm<BSQ_MXFP4, BSQ_BWD>(tmap, args, grid, s);
    return dir == BSQ_FWD ? launch_gmm<BSQ_NVFP4, BSQ_FWD>(tmap, args, grid, s)
                          : launch_gmm<BSQ_NVFP4, BSQ_BWD>(tmap, args, grid, s);
}
