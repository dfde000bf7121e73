/* Exhaustive check of the oracle's two minifloat encoders over every
 * binary32 bit pattern (TEST INFRASTRUCTURE). Each input is rounded again
 * by brute force, independently of the oracle's method: the nearest of the
 * format's representable magnitudes found by a scan (E2M1, 8 magnitudes) or
 * a bisection of the sorted table of all 127 finite non-negative E4M3
 * magnitudes, a tie going to the code with an even mantissa bit, values
 * beyond the largest magnitude saturating, the sign copied, NaN mapped as
 * the oracle's contract states (E4M3: 0x7F with the sign; E2M1: the signed
 * zero code). OCP MX v1.0 (E2M1) and OCP OFP8 (E4M3) define the formats.
 * Prints the mismatch count per encoder and exits non-zero on any mismatch. */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

extern uint32_t orc_e4m3_rne_sat(float x);
extern uint32_t orc_e2m1_rne_sat(float y);

static const double kE2m1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
static double kE4m3[127]; /* codes 0x00..0x7E, ascending */

static uint32_t brute_e2m1(uint32_t bits) {
    float y;
    memcpy(&y, &bits, 4);
    const uint32_t sign = bits >> 31;
    if (isnan(y)) return sign << 3;
    const double a = fabs((double)y);
    if (isinf(a) || a >= kE2m1[7]) return (sign << 3) | 7u; /* saturate (and keep the scan exact) */
    uint32_t best = 0;
    double bd = a;
    for (uint32_t c = 1; c < 8; ++c) {
        const double d = fabs(a - kE2m1[c]);
        if (d < bd || (d == bd && (c & 1u) == 0u)) {
            best = c;
            bd = d;
        }
    }
    return (sign << 3) | best;
}

static uint32_t brute_e4m3(uint32_t bits) {
    float x;
    memcpy(&x, &bits, 4);
    const uint32_t sign = bits >> 31;
    if (isnan(x)) return (sign << 7) | 0x7Fu;
    const double a = fabs((double)x);
    if (isinf(a) || a >= kE4m3[126]) return (sign << 7) | 0x7Eu;
    int lo = 0, hi = 126; /* kE4m3[lo] <= a < kE4m3[hi] */
    while (hi - lo > 1) {
        const int mid = (lo + hi) / 2;
        if (kE4m3[mid] <= a) lo = mid; else hi = mid;
    }
    uint32_t code;
    const double dl = a - kE4m3[lo], dh = kE4m3[hi] - a;
    if (dl < dh) code = (uint32_t)lo;
    else if (dh < dl) code = (uint32_t)hi;
    else code = (lo & 1) == 0 ? (uint32_t)lo : (uint32_t)hi;
    return (sign << 7) | code;
}

typedef struct {
    uint64_t begin, end;
    uint64_t bad_e2m1, bad_e4m3;
    uint32_t first_e2m1, first_e4m3;
} Range;

static void *work(void *arg) {
    Range *r = (Range *)arg;
    for (uint64_t b = r->begin; b < r->end; ++b) {
        const uint32_t bits = (uint32_t)b;
        float v;
        memcpy(&v, &bits, 4);
        if (orc_e2m1_rne_sat(v) != brute_e2m1(bits)) {
            if (r->bad_e2m1++ == 0) r->first_e2m1 = bits;
        }
        if (orc_e4m3_rne_sat(v) != brute_e4m3(bits)) {
            if (r->bad_e4m3++ == 0) r->first_e4m3 = bits;
        }
    }
    return NULL;
}

int main(int argc, char **argv) {
    /* E4M3 magnitudes from the format definition: subnormals m/8 * 2^-6, normals (1 + m/8) * 2^(e-7) */
    for (int c = 0; c < 127; ++c) {
        const int e = c >> 3, m = c & 7;
        kE4m3[c] = e == 0 ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
    }
    int threads = argc > 1 ? atoi(argv[1]) : 8;
    if (threads < 1) threads = 1;
    if (threads > 256) threads = 256;
    Range rs[256];
    pthread_t tid[256];
    const uint64_t total = 1ull << 32;
    for (int t = 0; t < threads; ++t) {
        memset(&rs[t], 0, sizeof(Range));
        rs[t].begin = total * (uint64_t)t / (uint64_t)threads;
        rs[t].end = total * (uint64_t)(t + 1) / (uint64_t)threads;
        pthread_create(&tid[t], NULL, work, &rs[t]);
    }
    uint64_t bad2 = 0, bad8 = 0;
    for (int t = 0; t < threads; ++t) {
        pthread_join(tid[t], NULL);
        if (rs[t].bad_e2m1 && !bad2) printf("first E2M1 mismatch: input bits 0x%08x\n", rs[t].first_e2m1);
        if (rs[t].bad_e4m3 && !bad8) printf("first E4M3 mismatch: input bits 0x%08x\n", rs[t].first_e4m3);
        bad2 += rs[t].bad_e2m1;
        bad8 += rs[t].bad_e4m3;
    }
    printf("e2m1_mismatches=%llu e4m3_mismatches=%llu inputs=%llu\n", (unsigned long long)bad2,
           (unsigned long long)bad8, (unsigned long long)total);
    return (bad2 || bad8) ? 1 : 0;
}
