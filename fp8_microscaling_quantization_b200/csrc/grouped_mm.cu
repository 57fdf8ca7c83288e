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
// Persistent, warp-specialised CTA (one per SM, 704 threads):
//   warps 0-3   epilogue: tensor memory -> registers (x row scale for NVFP4
//               forward) -> bf16 -> global; lane = feature, so each store of
//               a token's 32 features is one coalesced 64-byte row piece
//   warps 4-19  A producers, one 16-weight unit of the k-step per thread:
//               packed weights + scales from global (several k-steps in
//               flight), e2m1 -> bf16 by byte permutes, times the block scale
//               (bf16x2 multiply), swizzled 16-byte shared stores
//   warp 20     B producer: TMA loads of 64-token x 64-k activation boxes
//   warp 21     tensor-memory allocation and the single MMA-issuing thread
// By default two CTAs of a cluster work as a pair (cta_group::2) on tiles of
// 256 features x up to 512 tokens: each CTA dequantizes its 128 features and
// holds half of the tokens, and every k-step issues two M = 256, N <= 256
// MMAs on the same dequantized weights.  Single CTAs (output widths that are
// not a multiple of 256) take 128 x 256 tiles with two accumulators, so one
// tile's epilogue overlaps the next tile's loop.  k-step 64; a ring of 4
// stages, each a 16 KiB dequantized-weight slot and a 32 KiB activation slot
// with one full and one empty barrier, so the MMA thread waits once and
// commits once per k-step (its per-k-step instruction time, not the tensor
// core, sets the pace of a pipelined loop).  Tiles are numbered (expert token
// tile, feature tile) with the feature tile fastest, dealt round-robin to the
// CTA groups; every CTA derives the tile table from offs on the device.
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
#include <cstdlib>
#include <mutex>

#define BSQ_DBG_FILE 6
#include "debug.cuh"
#include "formats.cuh"
#include "host_util.h"
#include "tcgen05.cuh"

namespace bsq {
using namespace sm100;

namespace gmm {

constexpr int WM = 128;   // features per CTA (the CTA's share of MMA M)
constexpr int TN = 256;   // tokens per MMA at most (MMA N)
constexpr int BK = 64;
constexpr int XBOX = 64;  // token rows per TMA box
// Weights each producer thread converts per k-step (a "unit": 16 or 32
// consecutive packed weights of one row); the producer warp count follows.
// 16 (16 producer warps) keeps more weight loads in flight and measured
// faster in both directions than 32 (8 warps).
#ifndef BSQ_GMM_UNIT
#define BSQ_GMM_UNIT 16
#endif
constexpr int kUE = BSQ_GMM_UNIT;
constexpr int kEpiWarps = 4, kDqWarps = (128 * 64 / kUE) / 32;
constexpr int kTmaWarp = kEpiWarps + kDqWarps;  // 20
constexpr int kMmaWarp = kTmaWarp + 1;          // 21
constexpr int kThreads = (kMmaWarp + 1) * 32;   // 704
constexpr uint32_t kWStage = WM * BK * 2;       // 16 KiB dequantized weights
constexpr uint32_t kXBoxBytes = XBOX * BK * 2;  // 8 KiB
constexpr int kMaxExperts = 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitNs = 1000000000ull;  // default limit of a pipeline wait, and of every drain wait
constexpr int kPrefetch = 4;  // k-steps of packed weights in flight per producer thread

// Shared-memory plan of a CTA group of CG CTAs (1, or a pair with
// cta_group::2): a ring of stages, each the dequantized weight slot of one
// k-step followed by its activation slot.  One "full" barrier per stage
// collects the producer warps' arrivals and the activation bytes, one "empty"
// barrier receives the MMA commit: the MMA thread waits once and commits once
// per k-step.
//
// A single CTA's tile is 128 features x up to 256 tokens, with two 256-column
// accumulators so the epilogue of one tile overlaps the next tile's loop.  A
// pair's tile is 256 features x up to 512 tokens: every k-step issues two
// M = 256, N <= 256 MMAs (tokens 0-255 and 256-511 of the tile) on the same
// dequantized weights, which halves the dequantization per tensor-core FLOP
// for experts with more than 256 tokens; the two MMAs fill the 512 columns of
// tensor memory, so the pair has one accumulator.  Each CTA of a pair holds
// its half of both MMAs' tokens: 2 x 128 rows per stage.
template <int CG>
struct Plan {
    static constexpr int STAGES = 4;
    static constexpr int TT = TN * CG;                       // tokens per tile
    static constexpr int NACC = (CG == 1) ? 2 : 1;           // accumulator buffers
    static constexpr uint32_t kXHalf = (TN / CG) * BK * 2;   // one MMA's share of a CTA: 32 or 16 KiB
    static constexpr uint32_t kXStage = kXHalf * CG;         // 32 KiB
    static constexpr uint32_t kStage = kWStage + kXStage;    // 48 KiB
    static constexpr size_t kBarOffset = (size_t)STAGES * kStage;
    static constexpr int kNumBars = 2 * STAGES + 5;
    static constexpr size_t kSmemBytes = 1024 /* alignment slack */ + kBarOffset + kNumBars * 8 +
                                         16 /* tmem slot, flags */ + 4 * (2 * kMaxExperts + 2);
};

struct Args {
    const uint8_t* packed;
    const uint8_t* scales;
    const float* row_scale;
    const int32_t* offs;
    uint16_t* out;
    uint32_t* err;
    uint64_t wait_ns;  // limit of each pipeline wait (kWaitNs unless BSQ_GMM_WAIT_NS says otherwise)
    int E, T, N, K;
};

struct Tile {
    int e;      // expert
    int tok0;   // first token row
    int ntok;   // tokens in the tile (1..256 for one CTA, 1..512 for a pair)
    int f0;     // first feature (output column) of the tile
};

struct Shared {
    uint8_t* stage;  // stage s: weights at s * kStage, activations kWStage further
    uint64_t* full;
    uint64_t* empty;
    uint64_t* acc_full;
    uint64_t* acc_empty;
    uint64_t* drain;
    uint32_t* tmem_slot;
    volatile int* abort;
    int* tt_prefix;  // [E + 1] first token tile of each expert
    int* seg;        // [E + 1] seg[e] = first row of expert e, seg[E] = offs[E-1]
};

template <int CG>
__device__ __forceinline__ Shared carve(uint8_t* raw) {
    using P = Plan<CG>;
    Shared s;
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    s.stage = base;
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + P::kBarOffset);
    s.full = bars;
    s.empty = bars + P::STAGES;
    s.acc_full = bars + 2 * P::STAGES;
    s.acc_empty = s.acc_full + 2;
    s.drain = s.acc_empty + 2;
    s.tmem_slot = reinterpret_cast<uint32_t*>(bars + P::kNumBars);
    s.abort = reinterpret_cast<volatile int*>(s.tmem_slot + 1);
    s.tt_prefix = reinterpret_cast<int*>(s.tmem_slot + 4);
    s.seg = s.tt_prefix + kMaxExperts + 1;
    return s;
}

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const Shared& sh, const Args& a) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    uint32_t* err = a.err;
    while (!mbar_try_wait(bar, parity)) {
        if (*sh.abort) return false;
        if (globaltimer_ns() - t0 > a.wait_ns) {
            *sh.abort = 1;
            atomicOr(err, (uint32_t)BSQ_DEVERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// The same for all 32 lanes of a warp, with one outcome for the whole warp:
// it gives up if any lane's wait did, so the warp stays converged for the
// warp-collective instructions (__syncwarp, tcgen05.ld) that follow.
__device__ __forceinline__ bool wait_bar_warp(uint64_t* bar, uint32_t parity, const Shared& sh, const Args& a) {
    const bool ok = wait_bar(bar, parity, sh, a);
    return __all_sync(0xffffffffu, ok);
}

// f0 is the first feature of the group's tile (CTA r of a pair owns
// features f0 + 128 r ...).
template <int CG>
__device__ __forceinline__ Tile decode_tile(int t, int f_tiles, int E, const Shared& sh) {
    const int tg = t / f_tiles;
    const int ft = t - tg * f_tiles;
    int lo = 0, hi = E - 1;  // last expert whose first token tile is <= tg
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sh.tt_prefix[mid] <= tg) lo = mid;
        else hi = mid - 1;
    }
    constexpr int TT = Plan<CG>::TT;
    Tile ti;
    ti.e = lo;
    ti.tok0 = sh.seg[lo] + (tg - sh.tt_prefix[lo]) * TT;
    ti.ntok = min(TT, sh.seg[lo + 1] - ti.tok0);
    ti.f0 = ft * WM * CG;
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

// One producer thread's share of a k-step: kUE consecutive packed weights.
struct Unit {
    uint32_t w[kUE / 8];  // packed e2m1 codes, 8 per word
    uint32_t sc;          // MXFP4: one e8m0 byte; NVFP4: kUE/16 e4m3 bytes (16-column blocks)
    float g;              // NVFP4 backward row scale
};

// Place of unit u in the shared operand tile: its row r and first column c.
// Forward (K-major, rows = 128 features, columns = 64 k): r = u / (64/kUE).
// Backward (MN-major, rows = 64 contraction indices, columns = 128 k outputs
// in two 64-column panels): the eight threads of a quarter-warp take
// consecutive rows of ONE panel, so their 16-byte stores land on eight
// different bank groups of the 128-byte swizzle (taking both panels of a row
// would put two stores on each bank group).
template <int DIR>
__device__ __forceinline__ void unit_place(int u, int& r, int& c) {
    if (DIR == BSQ_FWD) {
        constexpr int upr = BK / kUE;
        r = u / upr;
        c = (u % upr) * kUE;
    } else {
        constexpr int upp = 64 / kUE;  // units per row of a panel
        constexpr int rpq = 8 / upp;   // rows per quarter-warp
        const int lane = u & 31;
        r = (u >> 5) * (2 * rpq) + (lane >> 4) * rpq + (lane / upp) % rpq;
        c = ((lane >> 3) & 1) * 64 + (lane % upp) * kUE;
    }
}

// Forward: the unit's row is a feature (weight row), its columns are k.
// Backward: its row is a contraction index (weight row), its columns are k
// outputs of the tile.
template <int FMT, int DIR>
__device__ __forceinline__ void load_unit(Unit& u, const Args& a, const Tile& ti, int ks, int unit) {
    int r, c;
    unit_place<DIR>(unit, r, c);
    int64_t row;
    int kcol;  // first weight column (k) of the unit
    if (DIR == BSQ_FWD) {
        row = (int64_t)ti.e * a.N + ti.f0 + r;
        kcol = ks * BK + c;
    } else {
        row = (int64_t)ti.e * a.N + ks * BK + r;
        kcol = ti.f0 + c;
    }
    if (!BSQ_DOK(row < (int64_t)a.E * a.N && kcol + kUE <= a.K)) {  // debug build: skip, record
        u.w[0] = u.w[kUE / 8 - 1] = 0u;
        u.sc = 0u;
        u.g = 0.0f;
        return;
    }
    const uint8_t* src = a.packed + row * (a.K / 2) + kcol / 2;
    if (kUE == 32) {
        const uint4 t = __ldg(reinterpret_cast<const uint4*>(src));
        u.w[0] = t.x; u.w[1] = t.y; u.w[kUE / 8 - 2] = t.z; u.w[kUE / 8 - 1] = t.w;
    } else {
        const uint2 t = __ldg(reinterpret_cast<const uint2*>(src));
        u.w[0] = t.x; u.w[1] = t.y;
    }
    if (FMT == BSQ_MXFP4) {
        u.sc = __ldg(a.scales + row * (a.K / 32) + kcol / 32);
        u.g = 1.0f;
    } else {
        const uint8_t* sp = a.scales + row * (a.K / 16) + kcol / 16;
        u.sc = (kUE == 32) ? (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(sp)) : (uint32_t)__ldg(sp);
        u.g = (DIR == BSQ_BWD) ? __ldg(a.row_scale + row) : 1.0f;
    }
}

// Decode a unit into kUE/2 words of bf16x2 (16-byte chunks of 8), block scale applied.
template <int FMT, int DIR>
__device__ __forceinline__ void decode_unit(const Unit& u, uint32_t (&v)[kUE / 2]) {
#pragma unroll
    for (int i = 0; i < kUE / 8; ++i) {
        uint32_t sc;
        if (FMT == BSQ_MXFP4) sc = scale_bf16x2<FMT, false>(u.sc, 0.0f);
        else sc = scale_bf16x2<FMT, DIR == BSQ_BWD>((u.sc >> (8 * (i / 2))) & 0xFFu, u.g);
        uint32_t t[4];
        e2m1x8_to_bf16(u.w[i], t);
#pragma unroll
        for (int j = 0; j < 4; ++j) v[4 * i + j] = mul_bf16x2(t[j], sc);
    }
}

// Write the decoded unit to its place in the swizzled operand tile.
template <int DIR>
__device__ __forceinline__ void store_unit(const uint32_t (&v)[kUE / 2], uint32_t w_stage, int unit) {
    // 128-byte shared row of the unit and its first 16-byte chunk in that row
    int r, col;
    unit_place<DIR>(unit, r, col);
    uint32_t base;
    int c0;
    if (DIR == BSQ_FWD) {
        c0 = col / 8;  // K-major: one row per feature, 8-row atoms of 1 KiB
        base = w_stage + (r >> 3) * 1024 + (r & 7) * 128;
    } else {
        c0 = (col % 64) / 8;  // MN-major: one row per contraction index, 64-feature panels
        base = w_stage + (col / 64) * (BK * 128) + (r >> 3) * 1024 + (r & 7) * 128;
    }
#pragma unroll
    for (int i = 0; i < kUE / 8; ++i)
        sts128(base + (uint32_t)(((c0 + i) ^ (r & 7)) << 4), v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}

// Arrive on the barrier at `bar`'s offset in the leader CTA of the group
// (the CTA itself when CG == 1).
template <int CG>
__device__ __forceinline__ void arrive_leader(uint64_t* bar) {
    if (CG == 1) mbar_arrive(bar);
    else mbar_arrive_cluster(mapa_shared(smem_u32(bar), 0));
}

template <int FMT, int DIR, int CG>
__global__ void __launch_bounds__(kThreads, 1) grouped_mm_kernel(const __grid_constant__ CUtensorMap tmap_x, Args args) {
    using P = Plan<CG>;
    extern __shared__ uint8_t smem_raw[];
    const Shared sh = carve<CG>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = args.E;
    const int out_w = (DIR == BSQ_FWD ? args.N : args.K);
    const int f_tiles = out_w / (WM * CG);
    const int k_steps = (DIR == BSQ_FWD ? args.K : args.N) / BK;
    const uint32_t rank = (CG == 2) ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    const int group = blockIdx.x / CG, ngroups = gridDim.x / CG;

    if (threadIdx.x == 0) {
        for (int s = 0; s < P::STAGES; ++s) {
            // every producer warp of the group, plus the leader's activation
            // producer (its arrive carries the expected bytes)
            mbar_init(&sh.full[s], kDqWarps * CG + 1);
            mbar_init(&sh.empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sh.acc_full[i], 1);
            mbar_init(&sh.acc_empty[i], kEpiWarps * CG);
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
            if (!bad) total += (o - prev + P::TT - 1) / P::TT;
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
        if (CG == 1) {
            tmem_alloc(sh.tmem_slot, kTmemCols);
            tmem_relinquish();
        } else {
            tmem_alloc_pair(sh.tmem_slot, kTmemCols);
            tmem_relinquish_pair();
        }
    }
    if (warp == kTmaWarp && lane == 0) tma_prefetch_desc(&tmap_x);
    tc_fence_before();
    __syncthreads();
    if (CG == 2) cluster_sync();  // the peer's barriers exist before any remote arrive
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
        for (int t = group; t < num_tiles; t += ngroups, ++tile_iter) {
            const Tile ti = decode_tile<CG>(t, f_tiles, E, sh);
            const int acc = tile_iter % P::NACC;
            if (!wait_bar_warp(&sh.acc_full[acc], (tile_iter / P::NACC) & 1, sh, args)) break;
            tc_fence_after();
            const int f = ti.f0 + WM * (int)rank + q * 32 + lane;
            float gf = 1.0f;
            if (FMT == BSQ_NVFP4 && DIR == BSQ_FWD) gf = __ldg(args.row_scale + (int64_t)ti.e * args.N + f);
            uint16_t* ocol = args.out + (int64_t)ti.tok0 * out_w + f;
            const int chunks = (ti.ntok + 15) >> 4;
#pragma unroll 1
            for (int c = 0; c < chunks; ++c) {
                uint32_t r[16];
                // token j of the tile is accumulator column j (a pair's second
                // MMA writes columns 256..511)
                tmem_ld_32x32b_x16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * TN + c * 16), r);
                tmem_ld_wait();
                const int nv = min(16, ti.ntok - c * 16);
                uint16_t* p = ocol + (int64_t)(c * 16) * out_w;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    float v = __uint_as_float(r[j]);
                    if (FMT == BSQ_NVFP4 && DIR == BSQ_FWD) v *= gf;
                    const __nv_bfloat16 h = __float2bfloat16_rn(v);
                    if (j < nv && BSQ_DOK(ti.tok0 + c * 16 + j < args.T && f < out_w)) *p = *reinterpret_cast<const uint16_t*>(&h);
                    p += out_w;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_leader<CG>(&sh.acc_empty[acc]);
        }
    } else if (warp < kTmaWarp) {
        // ------------------------------------------------- A (weight) producers
        const int dq = threadIdx.x - kEpiWarps * 32;  // unit index
        const uint32_t st_base = smem_u32(sh.stage);
        int my_tiles = 0;
        if (num_tiles > group) my_tiles = (num_tiles - 1 - group) / ngroups + 1;
        const int items = my_tiles * k_steps;
        // load cursor, kPrefetch k-steps ahead of the stores; this CTA's
        // features start WM * rank into the group's tile
        int lt = group, lks = 0;
        Tile lti;
        auto cursor_tile = [&](int t) {
            Tile ti = decode_tile<CG>(t, f_tiles, E, sh);
            ti.f0 += WM * (int)rank;
            return ti;
        };
        if (items > 0) lti = cursor_tile(lt);
        Unit buf[kPrefetch];
#pragma unroll
        for (int b = 0; b < kPrefetch; ++b) {
            if (b < items) {
                load_unit<FMT, DIR>(buf[b], args, lti, lks, dq);
                if (++lks == k_steps) {
                    lks = 0;
                    lt += ngroups;
                    if (lt < num_tiles) lti = cursor_tile(lt);
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
                    uint32_t v[kUE / 2];
                    decode_unit<FMT, DIR>(buf[b], v);
                    if (i + kPrefetch < items) {
                        load_unit<FMT, DIR>(buf[b], args, lti, lks, dq);
                        if (++lks == k_steps) {
                            lks = 0;
                            lt += ngroups;
                            if (lt < num_tiles) lti = cursor_tile(lt);
                        }
                    }
                    const int s = i % P::STAGES;
                    if (!wait_bar_warp(&sh.empty[s], ((i / P::STAGES) & 1) ^ 1, sh, args)) {
                        ok = false;
                    } else {
                        store_unit<DIR>(v, st_base + s * P::kStage, dq);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) arrive_leader<CG>(&sh.full[s]);
                    }
                }
            }
        }
    } else if (warp == kTmaWarp) {
        // ------------------------------------------- B (activation) producer
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int t = group; t < num_tiles && ok; t += ngroups) {
                const Tile ti = decode_tile<CG>(t, f_tiles, E, sh);
                // tokens of the tile's first and second MMA, rounded up to 16,
                // and this CTA's share (rows) of each
                const int n0 = (min(ti.ntok, TN) + 15) & ~15;
                const int n1 = (CG == 2 && ti.ntok > TN) ? ((ti.ntok - TN + 15) & ~15) : 0;
                const int h0 = n0 / CG, h1 = n1 / CG;
                const int nbox0 = (h0 + XBOX - 1) / XBOX, nbox1 = (h1 + XBOX - 1) / XBOX;
                for (int ks = 0; ks < k_steps; ++ks, ++it) {
                    const int s = it % P::STAGES;
                    if (!wait_bar(&sh.empty[s], ((it / P::STAGES) & 1) ^ 1, sh, args)) {
                        ok = false;
                        break;
                    }
                    uint8_t* dst = sh.stage + s * P::kStage + kWStage;
                    if (CG == 1) {
                        const int nbox = nbox0;
                        mbar_arrive_expect_tx(&sh.full[s], nbox * kXBoxBytes);
                        for (int b = 0; b < nbox; ++b)
                            tma_load_2d(dst + b * kXBoxBytes, &tmap_x, &sh.full[s], ks * BK, ti.tok0 + b * XBOX);
                    } else {
                        // both CTAs' boxes complete on the leader's barrier; the
                        // second MMA's rows go kXHalf into the slot
                        if (leader) mbar_arrive_expect_tx(&sh.full[s], 2 * (nbox0 + nbox1) * kXBoxBytes);
                        const uint32_t bar = mapa_shared(smem_u32(&sh.full[s]), 0);
                        for (int b = 0; b < nbox0; ++b)
                            tma_load_2d_pair(dst + b * kXBoxBytes, &tmap_x, bar, ks * BK,
                                             ti.tok0 + (int)rank * h0 + b * XBOX);
                        for (int b = 0; b < nbox1; ++b)
                            tma_load_2d_pair(dst + P::kXHalf + b * kXBoxBytes, &tmap_x, bar, ks * BK,
                                             ti.tok0 + TN + (int)rank * h1 + b * XBOX);
                    }
                }
            }
            if (!ok && leader) {
                // drain the loads still in flight (a pair's loads all count on
                // the leader's barriers); a stage whose producer warps gave up
                // never completes, and its wait ends at the time limit, long
                // after its bytes have landed
                for (int j = (it > P::STAGES ? it - P::STAGES : 0); j < it; ++j)
                    mbar_wait(&sh.full[j % P::STAGES], (j / P::STAGES) & 1, kWaitNs);
            }
        }
    } else {
        // ------------------------------------------------ MMA (leader only)
        if (lane == 0 && leader) {
            const uint32_t st_base = smem_u32(sh.stage);
            // descriptor advance per 16-wide k slice, in 16-byte units: 32 B
            // along a K-major row; 16 rows of 128 B (2048 B) of the MN-major
            // backward weights
            constexpr uint64_t kAStep = (DIR == BSQ_FWD) ? 2 : 128, kBStep = 2;
            int it = 0, tile_iter = 0;
            bool ok = true;
            for (int t = group; t < num_tiles && ok; t += ngroups, ++tile_iter) {
                const Tile ti = decode_tile<CG>(t, f_tiles, E, sh);
                const uint32_t n0 = (uint32_t)((min(ti.ntok, TN) + 15) & ~15);
                const uint32_t n1 = (CG == 2 && ti.ntok > TN) ? (uint32_t)((ti.ntok - TN + 15) & ~15) : 0u;
                const uint32_t idesc0 = idesc_bf16_ab(WM * CG, n0, DIR == BSQ_BWD ? 1u : 0u, 0u);
                const uint32_t idesc1 = idesc_bf16_ab(WM * CG, n1 ? n1 : 16u, DIR == BSQ_BWD ? 1u : 0u, 0u);
                const int acc = tile_iter % P::NACC;
                if (!wait_bar(&sh.acc_empty[acc], ((tile_iter / P::NACC) & 1) ^ 1, sh, args)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * TN);
                if (CG == 1) {
                    for (int ks = 0; ks < k_steps; ++ks, ++it) {
                        const int s = it % P::STAGES;
                        if (!wait_bar(&sh.full[s], (it / P::STAGES) & 1, sh, args)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t ws = st_base + s * P::kStage;
                        const uint64_t ad0 =
                            (DIR == BSQ_FWD) ? smem_desc(ws, 16, 1024) : smem_desc(ws, BK * 128, 1024);
                        const uint64_t bd0 = smem_desc(ws + kWStage, 16, 1024);
#pragma unroll
                        for (int k16 = 0; k16 < BK / 16; ++k16) {
                            const uint64_t ad = ad0 + kAStep * k16, bd = bd0 + kBStep * k16;
                            const uint32_t accum = (ks | k16) != 0 ? 1u : 0u;
                            mma_bf16_ss(d_tmem, ad, bd, idesc0, accum);
                        }
                        mma_commit(&sh.empty[s]);
                    }
                } else {
                    // Pairs.  The MMA thread's instructions per k-step are on
                    // the critical path (a partial tile's MMAs finish quickly),
                    // so they are kept few: the descriptors of stage 0 are split
                    // into 32-bit halves once, a stage's start address is the
                    // low half plus s * kStage / 16 (the start address field,
                    // bits 0-13, cannot carry: the stages lie below 256 KiB of
                    // shared memory), and the one- or two-MMA choice is made
                    // once per tile.
                    const uint64_t a00 =
                        (DIR == BSQ_FWD) ? smem_desc(st_base, 16, 1024) : smem_desc(st_base, BK * 128, 1024);
                    const uint64_t b00 = smem_desc(st_base + kWStage, 16, 1024);
                    const uint32_t a_lo0 = (uint32_t)a00, a_hi = (uint32_t)(a00 >> 32);
                    const uint32_t b_lo0 = (uint32_t)b00, b_hi = (uint32_t)(b00 >> 32);
                    const uint32_t d1 = d_tmem + TN, xh = (uint32_t)(P::kXHalf >> 4);
                    auto kstep = [&](int ks, bool two) -> bool {
                        const int s = it % P::STAGES;
                        if (!wait_bar(&sh.full[s], (it / P::STAGES) & 1, sh, args)) return false;
                        tc_fence_after();
                        const uint32_t so = (uint32_t)(s * (P::kStage >> 4));
                        const uint32_t al = a_lo0 + so, bl = b_lo0 + so;
                        const uint32_t acc0 = ks != 0 ? 1u : 0u;
#pragma unroll
                        for (int k16 = 0; k16 < BK / 16; ++k16) {
                            const uint32_t accum = k16 != 0 ? 1u : acc0;
                            const uint32_t ak = al + (uint32_t)kAStep * k16, bk = bl + (uint32_t)kBStep * k16;
                            mma_bf16_ss_pair_lh(d_tmem, ak, a_hi, bk, b_hi, idesc0, accum);
                            if (two) mma_bf16_ss_pair_lh(d1, ak, a_hi, bk + xh, b_hi, idesc1, accum);
                        }
                        mma_commit_pair_multicast(&sh.empty[s], 0x3);
                        ++it;
                        return true;
                    };
                    if (n1) {
                        for (int ks = 0; ks < k_steps && ok; ++ks) ok = kstep(ks, true);
                    } else {
                        for (int ks = 0; ks < k_steps && ok; ++ks) ok = kstep(ks, false);
                    }
                }
                if (ok) {
                    if (CG == 1) mma_commit(&sh.acc_full[acc]);
                    else mma_commit_pair_multicast(&sh.acc_full[acc], 0x3);
                }
            }
            // every MMA this thread issued has completed once `drain` fires
            if (CG == 1) mma_commit(sh.drain);
            else mma_commit_pair_multicast(sh.drain, 0x1);
            mbar_wait(sh.drain, 0, kWaitNs);
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (CG == 2) cluster_sync();  // no CTA leaves while its peer may still touch it
    tc_fence_after();
    if (warp == kMmaWarp) {
        if (CG == 1) tmem_dealloc(tmem, kTmemCols);
        else tmem_dealloc_pair(tmem, kTmemCols);
    }
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

template <int FMT, int DIR, int CG>
static bsq_status launch_gmm(const CUtensorMap& tmap, const gmm::Args& a, int64_t max_groups, cudaStream_t st) {
    static std::mutex mu;
    static int max_active[64] = {0};  // co-resident groups per device (0: not yet queried)
    auto kern = gmm::grouped_mm_kernel<FMT, DIR, CG>;
    const size_t smem = gmm::Plan<CG>::kSmemBytes;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.blockDim = dim3(gmm::kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    if (CG == 2) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    {
        std::lock_guard<std::mutex> lock(mu);
        if (max_active[dev] == 0) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess)
                return fail(BSQ_ERR_CUDA, "bsq_grouped_mm_fp4: shared-memory opt-in failed (%s)", cudaGetErrorString(e));
            int n = sm_count() / CG;
            if (CG == 2) {
                cfg.gridDim = dim3(2 * n, 1, 1);
                int clusters = 0;
                if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) == cudaSuccess && clusters > 0) n = clusters;
                cudaGetLastError();
            }
            max_active[dev] = n;
        }
    }
    const int groups = (int)std::max<int64_t>(1, std::min<int64_t>(max_groups, max_active[dev]));
    cfg.gridDim = dim3(groups * CG, 1, 1);
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tmap, a);
    if (e != cudaSuccess) return fail(BSQ_ERR_CUDA, "bsq_grouped_mm_fp4: launch failed (%s)", cudaGetErrorString(e));
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
    // BSQ_GMM_WAIT_NS (a positive integer, in ns) shortens the limit of each
    // pipeline wait; tests use it to make the waits run out on purpose
    args.wait_ns = gmm::kWaitNs;
    if (const char* w = getenv("BSQ_GMM_WAIT_NS")) {
        char* end = nullptr;
        const unsigned long long v = strtoull(w, &end, 10);
        if (end != w && *end == '\0' && v > 0) args.wait_ns = v;
    }
    args.E = E;
    args.T = (int)T;
    args.N = (int)N;
    args.K = (int)K;
    // CTA pairs (256 features x 512 tokens per tile, cta_group::2) wherever
    // the output width is a multiple of 256: they dequantize each weight tile
    // once for twice the tokens and measured 15-25% faster than single CTAs.
    // The environment variable BSQ_GMM_CTA_PAIR=0 selects single CTAs.
    const char* pair_env = getenv("BSQ_GMM_CTA_PAIR");
    const bool pairs_off = pair_env && pair_env[0] == '0';
    const int cg = (!pairs_off && out_w % (2 * gmm::WM) == 0) ? 2 : 1;
    const int64_t f_tiles = out_w / (gmm::WM * cg);
    const int64_t tile_tok = (int64_t)gmm::TN * cg;
    const int64_t max_groups = ((T + tile_tok - 1) / tile_tok + E) * f_tiles;
    cudaStream_t s = (cudaStream_t)stream;
    if (cg == 2) {
        if (fmt == BSQ_MXFP4)
            return dir == BSQ_FWD ? launch_gmm<BSQ_MXFP4, BSQ_FWD, 2>(tmap, args, max_groups, s)
                                  : launch_gmm<BSQ_MXFP4, BSQ_BWD, 2>(tmap, args, max_groups, s);
        return dir == BSQ_FWD ? launch_gmm<BSQ_NVFP4, BSQ_FWD, 2>(tmap, args, max_groups, s)
                              : launch_gmm<BSQ_NVFP4, BSQ_BWD, 2>(tmap, args, max_groups, s);
    }
    if (fmt == BSQ_MXFP4)
        return dir == BSQ_FWD ? launch_gmm<BSQ_MXFP4, BSQ_FWD, 1>(tmap, args, max_groups, s)
                              : launch_gmm<BSQ_MXFP4, BSQ_BWD, 1>(tmap, args, max_groups, s);
    return dir == BSQ_FWD ? launch_gmm<BSQ_NVFP4, BSQ_FWD, 1>(tmap, args, max_groups, s)
                          : launch_gmm<BSQ_NVFP4, BSQ_BWD, 1>(tmap, args, max_groups, s);
}

#ifdef BSQ_DEBUG
cudaError_t bsq_dbg_take_gmm(uint32_t* count, uint32_t* first) { return bsq::dbg_take(count, first); }
#endif
