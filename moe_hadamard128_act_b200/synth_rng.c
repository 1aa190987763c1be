/*
 * synth_rng.c -- counter-based random numbers for the seeded synthetic inputs.
 * Random numbers only: no part of the quantized layer's arithmetic lives here.
 *
 * Value i of a stream with key k is mix64(k + (i + 1) * 0x9E3779B97F4A7C15),
 * mix64 being the splitmix64 output function (Steele, Lea and Flood, "Fast
 * splittable pseudorandom number generators", OOPSLA 2014).  Uniform doubles
 * take the top 53 bits.  Normal i comes from the Box-Muller transform of the
 * uniform pair (2p, 2p+1), p = i / 2: the cosine branch for even i, the sine
 * branch for odd i.  Every value is a pure function of (key, i) computed with
 * scalar libm calls, so any slice regenerates bit for bit.
 *
 * Build: gcc -O2 -fopenmp -fno-fast-math -fPIC -shared
 */
#include <math.h>
#include <stdint.h>

static inline uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static inline uint64_t draw(uint64_t key, int64_t i) { return mix64(key + (uint64_t)(i + 1) * 0x9E3779B97F4A7C15ull); }

static inline double u01(uint64_t key, int64_t i) { return (double)(draw(key, i) >> 11) * (1.0 / 9007199254740992.0); }

uint64_t synth_mix64(uint64_t z) { return mix64(z); }

void synth_uniform01(uint64_t key, int64_t start, int64_t count, double* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < count; ++j) out[j] = u01(key, start + j);
}

static inline double normal_at(uint64_t key, int64_t i)
{
    const int64_t p = i >> 1;
    const double r = sqrt(-2.0 * log1p(-u01(key, 2 * p)));
    const double th = 6.283185307179586 * u01(key, 2 * p + 1);
    return (i & 1) ? r * sin(th) : r * cos(th);
}

void synth_normal(uint64_t key, int64_t start, int64_t count, double* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < count; ++j) out[j] = normal_at(key, start + j);
}

/* fp32 of std * normal: the weight tensors, without an fp64 intermediate array. */
void synth_normal_f32(uint64_t key, int64_t start, int64_t count, double std, float* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < count; ++j) out[j] = (float)(std * normal_at(key, start + j));
}

/* Integers uniform in [lo, hi] (hi - lo < 256): lo + floor(u01 * (hi - lo + 1)), stored as int8 bytes. */
void synth_uniform_int8(uint64_t key, int64_t start, int64_t count, int lo, int hi, int8_t* out)
{
    const double span = (double)(hi - lo + 1);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < count; ++j) out[j] = (int8_t)(lo + (int)floor(u01(key, start + j) * span));
}
