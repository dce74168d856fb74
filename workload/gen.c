/* Counter-based normal generator for the synthetic sink workloads.
 *
 * SplitMix64 (Steele, Lea, Flood, OOPSLA 2014) keyed by (seed, stream); two
 * consecutive outputs give one Box-Muller pair (cos -> even element, sin -> odd
 * element).  Holds no attention arithmetic. */
#include <math.h>
#include <stdint.h>

static inline uint64_t mix64(uint64_t z) {
    z ^= z >> 30; z *= 0xBF58476D1CE4E5B9ULL;
    z ^= z >> 27; z *= 0x94D049BB133111EBULL;
    z ^= z >> 31; return z;
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
    return mix64(seed * 0x100000001B3ULL + stream * 0x9E3779B1ULL);
}

/* uniform double in (0,1] from counter n of the keyed stream */
static inline double unif(uint64_t key, uint64_t n) {
    uint64_t bits = mix64(key + (n + 1) * 0x9E3779B97F4A7C15ULL) >> 11;
    return ((double)bits + 1.0) * (1.0 / 9007199254740992.0);
}

void wl_uniforms(uint64_t seed, uint64_t stream, uint64_t start, uint64_t count, double* out) {
    uint64_t key = stream_key(seed, stream);
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)count; ++i) out[i] = unif(key, start + (uint64_t)i);
}

void wl_normals(uint64_t seed, uint64_t stream, uint64_t start, uint64_t count, float* out) {
    const double two_pi = 6.283185307179586476925286766559;
    uint64_t key = stream_key(seed, stream);
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)count; ++i) {
        uint64_t e = start + (uint64_t)i, pr = e >> 1;
        double u1 = unif(key, 2 * pr), u2 = unif(key, 2 * pr + 1);
        double r = sqrt(-2.0 * log(u1)), th = two_pi * u2;
        out[i] = (float)((e & 1) ? r * sin(th) : r * cos(th));
    }
}

/* Raw SplitMix64 outputs from an explicit state: out[i] is the (i+1)-th output
 * of the generator started at `state` (the sequence unif() draws from, before
 * the top 53 bits are kept). */
void wl_splitmix64(uint64_t state, uint64_t count, uint64_t* out) {
    for (uint64_t i = 0; i < count; ++i) out[i] = mix64(state + (i + 1) * 0x9E3779B97F4A7C15ULL);
}
