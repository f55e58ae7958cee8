/*
 * Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU
 * oracle.  This file holds no decoder arithmetic: it only turns (seed, stream,
 * element index) into reproducible numbers.
 *
 * Generator: SplitMix64 (Steele, Lea & Flood, "Fast Splittable Pseudorandom
 * Number Generators", OOPSLA 2014) used counter-style: output i of stream
 * `key` is the SplitMix64 finaliser applied to key + (i+1)*golden_gamma.
 * Every element depends only on (seed, stream, index), so the values do not
 * depend on thread count, chunking or the machine.
 *
 * Normal draws: Irwin-Hall sum of eight 16-bit uniforms (two SplitMix64
 * outputs), centred and divided by its exact standard deviation, scaled by
 * `std`, rounded to fp32 and then to bf16 (round to nearest even).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t sm64_at(uint64_t key, uint64_t i) {
    uint64_t z = key + (i + 1ULL) * GOLDEN_GAMMA;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
    return sm64_at(sm64_at(seed, 0x5EEDULL), stream);
}

static inline uint16_t f32_to_bf16_bits(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u); /* NaN */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

static inline double irwin_hall8(uint64_t key, uint64_t i) {
    uint64_t a = sm64_at(key, 2ULL * i), b = sm64_at(key, 2ULL * i + 1ULL);
    int64_t s = 0;
    for (int k = 0; k < 4; k++) {
        s += (int64_t)((a >> (16 * k)) & 0xffffULL);
        s += (int64_t)((b >> (16 * k)) & 0xffffULL);
    }
    /* mean 8 * 65535/2, variance 8 * (65536^2 - 1)/12 */
    const double mean = 262140.0;
    const double sd = sqrt(2.0 * 4294967295.0 / 3.0);
    return ((double)s - mean) / sd;
}

/* out[i] = bf16(fp32(std * z_i)), z_i ~ approx N(0,1).  Bits written as uint16. */
void synth_normal_bf16(uint16_t *out, int64_t n, uint64_t seed, uint64_t stream, double std) {
    const uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) {
        float f = (float)(std * irwin_hall8(key, (uint64_t)i));
        out[i] = f32_to_bf16_bits(f);
    }
}

/* Same draws, kept in double (for tests of the generator itself). */
void synth_normal_f64(double *out, int64_t n, uint64_t seed, uint64_t stream, double std) {
    const uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) out[i] = std * irwin_hall8(key, (uint64_t)i);
}

/* Uniform integers in [lo, hi] (inclusive), multiply-shift mapping of the top 32 bits. */
void synth_uniform_int64(int64_t *out, int64_t n, uint64_t seed, uint64_t stream, int64_t lo, int64_t hi) {
    const uint64_t key = stream_key(seed, stream);
    const uint64_t span = (uint64_t)(hi - lo) + 1ULL;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) {
        uint64_t r = sm64_at(key, (uint64_t)i) >> 32;
        out[i] = lo + (int64_t)((r * span) >> 32);
    }
}

int synth_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
