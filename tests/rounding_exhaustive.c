/* Exhaustive check of the oracle's roundings (test code; it links the
 * oracle's library and calls o_e2m1_round, o_e4m3_round, o_f32_to_bf16,
 * o_floor_log2 and o_pow2_ceil).
 *
 * Every finite binary32 bit pattern x is checked for:
 *   - e2m1: the code's magnitude is a nearest value of |x| among the printed
 *     magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}, a tie going to the even index,
 *     and every |x| above 6 gives 6; the sign bit is the sign bit of x;
 *   - bf16: the result equals round-to-nearest-even by the integer rounding
 *     bias (bits + 0x7FFF + lsb) >> 16, an independent formulation, which
 *     also carries overflow to infinity;
 *   - both: the codes of the positive patterns never decrease as the
 *     patterns increase (monotone).
 * e4m3 (whose oracle enumerates all 127 codes per call) is checked the same
 * way against the values of the format (bias 7, 3 mantissa bits, subnormals
 * at exponent 0; every |x| above 448 gives 448) on every positive pattern
 * of the binades [2**-10, 2**9), which hold every rounding decision between
 * two codes, and on every 1024th pattern elsewhere (negatives included).
 * Distances are taken in binary64, exact wherever two codes compete.
 * On every positive finite pattern a: floor_log2 gives the e with
 * 2**e <= a < 2**(e+1); on every positive normal, the power-of-two ceiling
 * is a power of two p with a <= p < 2a (+inf above 2**127, where 2a has no
 * binary32 power of two).
 *
 * Usage: rounding_exhaustive [threads]; prints one line per rounding with
 * its count of failures and exits 0 when there are none. */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

int o_e2m1_round(float q);
int o_e4m3_round(float x);
uint16_t o_f32_to_bf16(float f);
int o_floor_log2(float a);
float o_pow2_ceil(float a);

static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
static double E4M3_MAG[127];

static float f_of(uint32_t b) {
    float f;
    memcpy(&f, &b, 4);
    return f;
}

/* k is a nearest index of m among the ascending vals[0..n-1], ties to the
 * even index; checking the two neighbours suffices for sorted values. */
static int is_nearest(const double* vals, int n, double m, int k) {
    if (k < 0 || k >= n) return 0;
    const double d = fabs(m - vals[k]);
    for (int j = k - 1; j <= k + 1; j += 2) {
        if (j < 0 || j >= n) continue;
        const double dj = fabs(m - vals[j]);
        if (dj < d || (dj == d && (k & 1))) return 0;
    }
    return 1;
}

typedef struct {
    int t, nt;
    uint64_t bad_e2m1, bad_bf16, bad_e4m3, n_e4m3, bad_log2, bad_pow2;
    uint32_t first_e2m1, first_bf16, first_e4m3, first_log2, first_pow2;
} Job;

static void note(uint64_t* bad, uint32_t* first, uint32_t b) {
    if ((*bad)++ == 0) *first = b;
}

/* whether the magnitude index k is right for |x| = m */
static int e2m1_ok(double m, int k) { return m > 6.0 ? k == 7 : is_nearest(E2M1_MAG, 8, m, k); }
static int e4m3_ok(double m, int k) { return m > 448.0 ? k == 126 : is_nearest(E4M3_MAG, 127, m, k); }

/* whether the e4m3 rounding of pattern b is checked: every positive pattern
 * with a biased exponent in [117, 136) (|x| in [2**-10, 2**9)), every
 * 1024th pattern otherwise */
static int e4m3_checked(uint32_t b) {
    const uint32_t ex = (b >> 23) & 0xFFu;
    return ((b >> 31) == 0 && ex >= 117 && ex < 136) || (b & 1023u) == 0;
}

/* Blocks of 2**16 patterns, dealt round robin to the threads. */
static void* run(void* arg) {
    Job* j = (Job*)arg;
    const uint64_t kBlock = (uint64_t)1 << 16, nblocks = ((uint64_t)1 << 32) / kBlock;
    for (uint64_t blk = (uint64_t)j->t; blk < nblocks; blk += (uint64_t)j->nt) {
        const uint64_t lo = blk * kBlock, hi = lo + kBlock;
        /* the codes of the pattern before the block, for the monotone check */
        int prev2 = -1, prev4 = -1;
        uint32_t prevb = 0;
        if (lo > 0 && lo < 0x7F800000u) {
            const float xp = f_of((uint32_t)(lo - 1));
            prev2 = o_e2m1_round(xp) & 7;
            prevb = o_f32_to_bf16(xp);
        }
        for (uint64_t i = lo; i < hi; ++i) {
            const uint32_t b = (uint32_t)i;
            const uint32_t mag = b & 0x7FFFFFFFu;
            if (mag >= 0x7F800000u) continue; /* inf and NaN are outside the contract */
            const float x = f_of(b);
            const int neg = (int)(b >> 31);
            const double m = fabs((double)x);
            const int c2 = o_e2m1_round(x);
            if (((c2 >> 3) & 1) != neg || !e2m1_ok(m, c2 & 7)) note(&j->bad_e2m1, &j->first_e2m1, b);
            const uint16_t r = o_f32_to_bf16(x);
            if (r != (uint16_t)((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16)) note(&j->bad_bf16, &j->first_bf16, b);
            int c4 = -1;
            if (e4m3_checked(b)) {
                c4 = o_e4m3_round(x);
                j->n_e4m3++;
                if (((c4 >> 7) & 1) != neg || !e4m3_ok(m, c4 & 0x7F)) note(&j->bad_e4m3, &j->first_e4m3, b);
            }
            if (!neg && mag != 0) {
                const int e = o_floor_log2(x);
                if (!(ldexp(1.0, e) <= m && m < ldexp(1.0, e + 1))) note(&j->bad_log2, &j->first_log2, b);
                if (mag >= 0x00800000u) { /* normal */
                    const float p = o_pow2_ceil(x);
                    uint32_t pb;
                    memcpy(&pb, &p, 4);
                    const int ok = (m > ldexp(1.0, 127)) ? (pb == 0x7F800000u)
                                                         : ((pb & 0x807FFFFFu) == 0 && pb != 0 && (double)p >= m &&
                                                            (double)p < 2.0 * m);
                    if (!ok) note(&j->bad_pow2, &j->first_pow2, b);
                }
            }
            if (!neg) { /* ascending values */
                if ((c2 & 7) < prev2 || r < prevb) note(&j->bad_e2m1, &j->first_e2m1, b);
                prev2 = c2 & 7;
                prevb = r;
                if (c4 >= 0) {
                    if ((c4 & 0x7F) < prev4) note(&j->bad_e4m3, &j->first_e4m3, b);
                    prev4 = c4 & 0x7F;
                }
            }
        }
    }
    return NULL;
}

int main(int argc, char** argv) {
    int nt = argc > 1 ? atoi(argv[1]) : 8;
    if (nt < 1) nt = 1;
    if (nt > 256) nt = 256;
    for (int k = 0; k < 127; ++k) {
        const int e = k >> 3, mm = k & 7;
        E4M3_MAG[k] = e ? ldexp(8.0 + mm, e - 10) : ldexp((double)mm, -9);
    }
    Job* jobs = calloc((size_t)nt, sizeof(Job));
    pthread_t* th = calloc((size_t)nt, sizeof(pthread_t));
    if (!jobs || !th) return 2;
    for (int t = 0; t < nt; ++t) {
        jobs[t].t = t;
        jobs[t].nt = nt;
        if (pthread_create(&th[t], NULL, run, &jobs[t]) != 0) return 2;
    }
    uint64_t be = 0, bb = 0, b4 = 0, n4 = 0, bl = 0, bp = 0;
    uint32_t fe = 0, fb = 0, f4 = 0, fl = 0, fp = 0;
    for (int t = 0; t < nt; ++t) {
        pthread_join(th[t], NULL);
        if (jobs[t].bad_e2m1 && !be) fe = jobs[t].first_e2m1;
        if (jobs[t].bad_bf16 && !bb) fb = jobs[t].first_bf16;
        if (jobs[t].bad_e4m3 && !b4) f4 = jobs[t].first_e4m3;
        if (jobs[t].bad_log2 && !bl) fl = jobs[t].first_log2;
        if (jobs[t].bad_pow2 && !bp) fp = jobs[t].first_pow2;
        bl += jobs[t].bad_log2;
        bp += jobs[t].bad_pow2;
        be += jobs[t].bad_e2m1;
        bb += jobs[t].bad_bf16;
        b4 += jobs[t].bad_e4m3;
        n4 += jobs[t].n_e4m3;
    }
    printf("e2m1 failures %llu first 0x%08x\n", (unsigned long long)be, fe);
    printf("bf16 failures %llu first 0x%08x\n", (unsigned long long)bb, fb);
    printf("e4m3 failures %llu first 0x%08x checked %llu\n", (unsigned long long)b4, f4, (unsigned long long)n4);
    printf("floor_log2 failures %llu first 0x%08x\n", (unsigned long long)bl, fl);
    printf("pow2_ceil failures %llu first 0x%08x\n", (unsigned long long)bp, fp);
    free(jobs);
    free(th);
    return (be || bb || b4 || bl || bp) ? 1 : 0;
}
