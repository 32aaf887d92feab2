/*
 * Seeded, counter-based value generator for the synthetic decode workloads.
 *
 * Holds none of the attention or planning arithmetic: it only turns
 * (seed, stream, element index) into a bf16 bit pattern, so that the same
 * element always gets the same value whatever order or thread produces it.
 *
 * Value of element i: splitmix64's finaliser (Steele, Lea & Flood, "Fast
 * splittable pseudorandom number generators", OOPSLA 2014) applied to a
 * counter built from (seed, stream, i) gives 64 random bits; their top and
 * bottom 24 bits are two uniforms in (0, 1); the Box-Muller transform of the
 * pair gives one standard normal; an optional per-row factor multiplies it;
 * the float is rounded to bf16 (round to nearest, ties to even).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static inline uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

static inline float normal_at(uint64_t key, uint64_t i)
{
    uint64_t h = mix64(key + (i + 1) * 0x9E3779B97F4A7C15ULL);
    float u1 = ((float)(h >> 40) + 0.5f) * (1.0f / 16777216.0f);
    float u2 = ((float)(h & 0xFFFFFFu) + 0.5f) * (1.0f / 16777216.0f);
    return sqrtf(-2.0f * logf(u1)) * cosf(6.283185307179586f * u2);
}

/*
 * out[i] = bf16(normal(seed, stream, first + i) * factor[(first + i) / row_len])
 * for i in [0, n).  factor may be NULL (all ones).
 */
void fca_gen_normal_bf16(uint16_t *out, int64_t n, int64_t first, uint64_t seed,
                         uint64_t stream, const float *row_factor, int64_t row_len)
{
    uint64_t key = mix64(seed * 0xD1B54A32D192ED03ULL + stream * 0xABC98388FB8FAC03ULL + 1);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        int64_t g = first + i;
        float v = normal_at(key, (uint64_t)g);
        if (row_factor) v *= row_factor[g / row_len];
        out[i] = f32_to_bf16_rne(v);
    }
}
