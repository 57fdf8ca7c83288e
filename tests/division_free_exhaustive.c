/* Exhaustive checks of the kernels' division-free arithmetic (test code; it
 * links the oracle's library for o_pow2_ceil).
 *
 * 1. Corrected quotient.  For every bf16 significand X in [1, 2) (128 of
 *    them) and every binary32 significand D in [1, 2) (2**23): with
 *    y = RN(1/D), q0 = RN((-X)(-y)), r = RN(q0 D - X) by one fma and
 *    q1 = RN(q0 - r y) by one fma, q1 equals the IEEE quotient RN(X / D).
 *    Exponents only scale the operands, so this covers every bf16 x and
 *    binary32 d for which no step leaves the normal range.
 * 2. Power-of-two scale from the bits of the amax.  For M = 448 = 1.75 * 2**8
 *    (K = 8, MM = 0x600000) and M = 6 = 1.5 * 2**2 (K = 2, MM = 0x400000),
 *    and every non-negative finite binary32 a: the biased exponent
 *    max(biased(a) - K + [mantissa(a) > MM], 1) is that of the oracle's
 *    pow2_ceil(max(RN(a / M), 2**-126)).
 *
 * fmaf is the C library's correctly rounded fused multiply-add; the build
 * keeps contraction off so every other operation rounds on its own.
 * Usage: division_free_exhaustive [threads]; exits 0 when nothing fails. */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

float o_pow2_ceil(float a);

static float f_of(uint32_t b) {
    float f;
    memcpy(&f, &b, 4);
    return f;
}
static uint32_t bits_of(float f) {
    uint32_t b;
    memcpy(&b, &f, 4);
    return b;
}

typedef struct {
    int t, nt;
    uint64_t bad_cq, bad_p448, bad_p6;
    uint32_t first_cq, first_p448, first_p6;
} Job;

static void note(uint64_t* bad, uint32_t* first, uint32_t v) {
    if ((*bad)++ == 0) *first = v;
}

static uint32_t pow2_by_bits(uint32_t a, int K, uint32_t MM) {
    int pb = (int)(a >> 23) - K + ((a & 0x7FFFFFu) > MM ? 1 : 0);
    return (uint32_t)(pb < 1 ? 1 : pb);
}

static uint32_t pow2_by_division(float a, float M) {
    float q = a / M;
    if (q < 0x1p-126f) q = 0x1p-126f;
    return bits_of(o_pow2_ceil(q)) >> 23;
}

static void* run(void* arg) {
    Job* j = (Job*)arg;
    /* 1: rows of D significands for each X, split over the threads */
    for (uint32_t kx = 0; kx < 128; ++kx) {
        const float X = 1.0f + (float)kx / 128.0f;
        for (uint32_t dm = (uint32_t)j->t; dm < (1u << 23); dm += (uint32_t)j->nt) {
            const float D = f_of(0x3F800000u | dm);
            const float y = 1.0f / D;
            const float nx = -X, ny = -y;
            const float q0 = nx * ny;
            const float r = fmaf(q0, D, nx);
            const float q1 = fmaf(r, ny, q0);
            if (bits_of(q1) != bits_of(X / D)) note(&j->bad_cq, &j->first_cq, (kx << 23) | dm);
        }
    }
    /* 2: every non-negative finite pattern, blocks of 2**16 dealt round robin */
    const uint64_t kBlock = (uint64_t)1 << 16, nblocks = (uint64_t)0x7F800000u / kBlock;
    for (uint64_t blk = (uint64_t)j->t; blk < nblocks; blk += (uint64_t)j->nt) {
        for (uint64_t i = blk * kBlock; i < (blk + 1) * kBlock; ++i) {
            const uint32_t a = (uint32_t)i;
            const float af = f_of(a);
            if (pow2_by_bits(a, 8, 0x600000u) != pow2_by_division(af, 448.0f)) note(&j->bad_p448, &j->first_p448, a);
            if (pow2_by_bits(a, 2, 0x400000u) != pow2_by_division(af, 6.0f)) note(&j->bad_p6, &j->first_p6, a);
        }
    }
    return NULL;
}

int main(int argc, char** argv) {
    int nt = argc > 1 ? atoi(argv[1]) : 8;
    if (nt < 1) nt = 1;
    if (nt > 256) nt = 256;
    Job* jobs = calloc((size_t)nt, sizeof(Job));
    pthread_t* th = calloc((size_t)nt, sizeof(pthread_t));
    if (!jobs || !th) return 2;
    for (int t = 0; t < nt; ++t) {
        jobs[t].t = t;
        jobs[t].nt = nt;
        if (pthread_create(&th[t], NULL, run, &jobs[t]) != 0) return 2;
    }
    uint64_t bc = 0, b448 = 0, b6 = 0;
    uint32_t fc = 0, f448 = 0, f6 = 0;
    for (int t = 0; t < nt; ++t) {
        pthread_join(th[t], NULL);
        if (jobs[t].bad_cq && !bc) fc = jobs[t].first_cq;
        if (jobs[t].bad_p448 && !b448) f448 = jobs[t].first_p448;
        if (jobs[t].bad_p6 && !b6) f6 = jobs[t].first_p6;
        bc += jobs[t].bad_cq;
        b448 += jobs[t].bad_p448;
        b6 += jobs[t].bad_p6;
    }
    printf("corrected_quotient failures %llu first 0x%08x\n", (unsigned long long)bc, fc);
    printf("pow2_448 failures %llu first 0x%08x\n", (unsigned long long)b448, f448);
    printf("pow2_6 failures %llu first 0x%08x\n", (unsigned long long)b6, f6);
    free(jobs);
    free(th);
    return (bc || b448 || b6) ? 1 : 0;
}
