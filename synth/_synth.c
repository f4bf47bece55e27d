/* Seeded N(0,1) draws for the synthetic workloads: splitmix64 + Box-Muller.
 *
 * splitmix64 is the generator of Steele, Lea & Flood (OOPSLA 2014): the state
 * advances by GAMMA and each output is mix64(state).  Output k (k >= 1) of a
 * stream started at state s is mix64(s + k * GAMMA), so any element can be
 * drawn independently and the loop below is parallel over element pairs.
 *
 * Element 2m and 2m+1 of a normal sequence come from outputs 2m+1 and 2m+2:
 *   u1 = (a >> 11 + 1) * 2^-53 in (0, 1],  u2 = (b >> 11) * 2^-53 in [0, 1)
 *   r  = sqrt(-2 ln u1);  z[2m] = r cos(2 pi u2);  z[2m+1] = r sin(2 pi u2)
 * All in IEEE double; no fast-math.
 */
#include <math.h>
#include <stdint.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t synth_draw(uint64_t seed, uint64_t k) { return mix64(seed + k * GAMMA); }

/* out[i] = element (start + i) of the normal sequence of the stream at state s. */
void synth_normals(uint64_t s, int64_t start, int64_t n, double* out) {
    const double two_pi = 6.283185307179586476925286766559;
    const double tiny = 1.0 / 9007199254740992.0; /* 2^-53 */
    int64_t p0 = start >> 1;
    int64_t p1 = (start + n + 1) >> 1;
#pragma omp parallel for schedule(static)
    for (int64_t p = p0; p < p1; ++p) {
        uint64_t a = mix64(s + (uint64_t)(2 * p + 1) * GAMMA);
        uint64_t b = mix64(s + (uint64_t)(2 * p + 2) * GAMMA);
        double u1 = ((double)(a >> 11) + 1.0) * tiny;
        double u2 = (double)(b >> 11) * tiny;
        double r = sqrt(-2.0 * log(u1));
        int64_t e0 = 2 * p, e1 = 2 * p + 1;
        if (e0 >= start && e0 < start + n) out[e0 - start] = r * cos(two_pi * u2);
        if (e1 >= start && e1 < start + n) out[e1 - start] = r * sin(two_pi * u2);
    }
}
