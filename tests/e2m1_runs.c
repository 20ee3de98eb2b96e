/* e2m1_runs.c -- test helper: the run-length form of an E2M1 encoder over
 * every binary32 bit pattern of one sign up to a bound.
 *
 * e2m1_runs(enc, sign, hi, starts, codes, cap) evaluates enc(v) for v = the
 * float with bits (sign << 31) | u, for every u in [0, hi], and writes the
 * runs of equal codes in order: run k covers u in [starts[k], starts[k+1])
 * (the last one up to hi) with code codes[k].  Returns the number of runs, or
 * -1 if there are more than cap.  The scan is split over OpenMP threads; each
 * chunk's runs are merged at the chunk borders.  The encoder is passed in (the
 * oracle's, from its own library), so this file holds no arithmetic of the
 * method. */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef uint8_t (*enc_fn)(float);

#define CHUNKS 256
#define CHUNK_CAP 64

static float from_bits(uint32_t u)
{
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

int e2m1_runs(enc_fn enc, uint32_t sign, uint32_t hi, uint32_t *starts, uint8_t *codes, int cap)
{
    static uint32_t cs[CHUNKS][CHUNK_CAP];
    static uint8_t cc[CHUNKS][CHUNK_CAP];
    static int cn[CHUNKS];
    const uint64_t total = (uint64_t)hi + 1u;
    int overflow = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(|: overflow)
    for (int c = 0; c < CHUNKS; ++c) {
        const uint64_t lo = total * (uint64_t)c / CHUNKS, up = total * (uint64_t)(c + 1) / CHUNKS;
        int n = 0;
        int prev = -1;
        for (uint64_t u = lo; u < up; ++u) {
            const int code = enc(from_bits((sign << 31) | (uint32_t)u));
            if (code != prev) {
                if (n == CHUNK_CAP) { overflow = 1; break; }
                cs[c][n] = (uint32_t)u;
                cc[c][n] = (uint8_t)code;
                ++n;
                prev = code;
            }
        }
        cn[c] = n;
    }
    if (overflow) return -1;
    int n = 0;
    for (int c = 0; c < CHUNKS; ++c)
        for (int k = 0; k < cn[c]; ++k) {
            if (n > 0 && codes[n - 1] == cc[c][k]) continue;   /* same run across a chunk border */
            if (n == cap) return -1;
            starts[n] = cs[c][k];
            codes[n] = cc[c][k];
            ++n;
        }
    return n;
}
