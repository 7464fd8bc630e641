/*
 * Exhaustive check of the oracle's E2M1 and E4M3 rounding against rules written
 * independently of it:
 *   - E2M1: every FP32 bit pattern in [0, 8] (and its negation) is compared to
 *     a hand-derived table of decision points (the midpoints between adjacent
 *     E2M1 magnitudes, with the tie going to the even code).
 *   - E4M3: the 127 finite non-negative values are read from argv (the test
 *     takes them from torch's float8_e4m3fn decoding); every 16th FP32 pattern
 *     in [0, 480] and every pattern within +-64 ulps of each midpoint is
 *     compared with a binary-search nearest-value rule (ties to even code,
 *     saturation to 448 above it).
 * Prints "mismatches <e2m1> <e4m3> checked <n2> <n4>" and exits 0.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

extern void oracle_e2m1_encode_many(const float* y, int64_t n, uint8_t* out);
extern void oracle_e4m3_encode_many(const float* x, int64_t n, uint8_t* out);

static float from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static uint8_t e2m1_rule(float a)
{
    /* decision points between 0|0.5|1|1.5|2|3|4|6; "<=" where the tie goes down */
    if (a <= 0.25f) return 0;   /* tie 0.25 -> code 0 (even) */
    if (a < 0.75f) return 1;    /* tie 0.75 -> code 2 */
    if (a <= 1.25f) return 2;   /* tie 1.25 -> code 2 */
    if (a < 1.75f) return 3;    /* tie 1.75 -> code 4 */
    if (a <= 2.5f) return 4;    /* tie 2.5  -> code 4 */
    if (a < 3.5f) return 5;     /* tie 3.5  -> code 6 */
    if (a <= 5.0f) return 6;    /* tie 5    -> code 6 */
    return 7;
}

static double E4[127];

static uint8_t e4m3_rule(float af)
{
    double a = af;
    if (a >= E4[126]) return 126;
    int lo = 0, hi = 126;            /* E4[lo] <= a < E4[hi] */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (E4[mid] <= a) lo = mid; else hi = mid;
    }
    double dl = a - E4[lo], dh = E4[hi] - a;
    if (dl < dh) return (uint8_t)lo;
    if (dh < dl) return (uint8_t)hi;
    return (uint8_t)((lo % 2 == 0) ? lo : hi);
}

#define CHUNK (1 << 22)

int main(int argc, char** argv)
{
    if (argc != 128) {
        fprintf(stderr, "need 127 E4M3 values\n");
        return 2;
    }
    for (int i = 0; i < 127; ++i) E4[i] = atof(argv[1 + i]);

    long long bad2 = 0, bad4 = 0, n2 = 0, n4 = 0;

    /* E2M1: all patterns 0x00000000 .. 0x41000000 (0 .. 8.0), both signs,
     * split into chunks checked in parallel. */
    const uint64_t top2 = 0x41000000u;
    const int64_t nchunks = (int64_t)((top2 + CHUNK) / CHUNK);
#pragma omp parallel for schedule(dynamic) reduction(+ : bad2, n2)
    for (int64_t job = 0; job < 2 * nchunks; ++job) {
        int sign = (int)(job / nchunks);
        uint64_t base = (uint64_t)(job % nchunks) * CHUNK;
        float* b = malloc(sizeof(float) * CHUNK);
        uint8_t* g = malloc(CHUNK);
        int64_t n = 0;
        for (uint64_t u = base; u <= top2 && u < base + CHUNK; ++u)
            b[n++] = from_bits((uint32_t)u | (sign ? 0x80000000u : 0u));
        oracle_e2m1_encode_many(b, n, g);
        for (int64_t i = 0; i < n; ++i) {
            uint8_t want = e2m1_rule(fabsf(b[i])) | (sign ? 8 : 0);
            if (g[i] != want) ++bad2;
        }
        n2 += n;
        free(b);
        free(g);
    }
    float* buf = malloc(sizeof(float) * CHUNK);
    uint8_t* got = malloc(CHUNK);
    /* beyond 8: a sparse sweep up to +inf saturates to 6 */
    {
        int64_t n = 0;
        for (uint64_t u = top2; u <= 0x7f800000u; u += 4099) buf[n++] = from_bits((uint32_t)u);
        oracle_e2m1_encode_many(buf, n, got);
        for (int64_t i = 0; i < n; ++i)
            if (got[i] != 7) ++bad2;
        n2 += n;
    }

    /* E4M3: every 16th pattern up to 480 (chunks in parallel), then +-64 ulps
     * around each midpoint. */
    const uint64_t top4 = to_bits(480.0f);
    const uint64_t span4 = (uint64_t)CHUNK * 16;
    const int64_t nchunks4 = (int64_t)((top4 + span4) / span4);
#pragma omp parallel for schedule(dynamic) reduction(+ : bad4, n4)
    for (int64_t job = 0; job < nchunks4; ++job) {
        float* b = malloc(sizeof(float) * CHUNK);
        uint8_t* g = malloc(CHUNK);
        int64_t n = 0;
        for (uint64_t u = (uint64_t)job * span4; u <= top4 && u < (uint64_t)(job + 1) * span4; u += 16)
            b[n++] = from_bits((uint32_t)u);
        oracle_e4m3_encode_many(b, n, g);
        for (int64_t i = 0; i < n; ++i)
            if (g[i] != e4m3_rule(b[i])) ++bad4;
        n4 += n;
        free(b);
        free(g);
    }
    int64_t n = 0;
    /* beyond 480: a sparse sweep up to +inf saturates to 448 */
    for (uint64_t u = top4; u <= 0x7f800000u; u += 4099) buf[n++] = from_bits((uint32_t)u);
    for (int i = 0; i < 127; ++i) {
        double mid = (i < 126) ? 0.5 * (E4[i] + E4[i + 1]) : 464.0;
        uint32_t c = to_bits((float)mid);
        for (int d = -64; d <= 64; ++d) {
            if ((int64_t)c + d < 0) continue;
            buf[n++] = from_bits(c + d);
        }
    }
    oracle_e4m3_encode_many(buf, n, got);
    for (int64_t i = 0; i < n; ++i)
        if (got[i] != e4m3_rule(buf[i])) {
            if (bad4 < 5) fprintf(stderr, "e4m3 %a got %x want %x\n", buf[i], got[i], e4m3_rule(buf[i]));
            ++bad4;
        }
    n4 += n;

    printf("mismatches %lld %lld checked %lld %lld\n", bad2, bad4, n2, n4);
    free(buf);
    free(got);
    return 0;
}
