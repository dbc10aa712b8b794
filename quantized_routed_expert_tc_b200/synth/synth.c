/*
 * synth.c -- seeded, counter-based synthetic inputs.
 *
 * Holds none of the layer's arithmetic: it only draws numbers.  Both the CPU
 * oracle (in tests) and the CUDA path consume the arrays it writes, so the two
 * sides see identical inputs.
 *
 * Generator: every value is a pure function of (seed, stream, index).
 *   mix(z)      = the SplitMix64 output function (Steele, Lea and Flood,
 *                 "Fast splittable pseudorandom number generators", 2014):
 *                 z += 0x9E3779B97F4A7C15; z = (z ^ z>>30) * 0xBF58476D1CE4E5B9;
 *                 z = (z ^ z>>27) * 0x94D049BB133111EB; return z ^ z>>31.
 *   key         = mix(mix(seed) ^ stream)
 *   u(i)        = ((mix(key + i) >> 11) + 1) * 2^-53, in (0, 1]
 *   normals     : Box-Muller on the pair (u(2j), u(2j+1)) gives elements
 *                 2j (cosine branch) and 2j+1 (sine branch), in double.
 * Values are rounded once to f32 (or to bf16, nearest-even, for bf16 inputs).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static inline uint64_t mix64(uint64_t z)
{
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream)
{
    return mix64(mix64(seed) ^ stream);
}

static inline double unif(uint64_t key, uint64_t i)
{
    return (double)((mix64(key + i) >> 11) + 1) * (1.0 / 9007199254740992.0);
}

/* Box-Muller pairs j covering [offset, offset + n): each pair is computed
 * once and gives the two elements 2j and 2j+1 (those inside the range). */
#define FOR_PAIRS(BODY)                                                        \
    const uint64_t key = stream_key(seed, stream);                             \
    const int64_t j0 = offset >> 1, j1 = (offset + n + 1) >> 1;                \
    _Pragma("omp parallel for schedule(static, 32768)")                        \
    for (int64_t j = j0; j < j1; ++j) {                                        \
        double u1 = unif(key, (uint64_t)(2 * j));                              \
        double u2 = unif(key, (uint64_t)(2 * j + 1));                          \
        double r = sqrt(-2.0 * log(u1));                                       \
        double th = 6.283185307179586476925286766559 * u2;                     \
        double z[2] = {r * cos(th), r * sin(th)};                              \
        for (int q = 0; q < 2; ++q) {                                          \
            int64_t i = 2 * j + q - offset;                                    \
            if (i < 0 || i >= n) continue;                                     \
            BODY                                                               \
        }                                                                      \
    }

/* out[i] = f32(mean + std * z(offset + i)), i < n */
void synth_normal_f32(uint64_t seed, uint64_t stream, int64_t offset, int64_t n,
                      double mean, double std, float *out)
{
    FOR_PAIRS(out[i] = (float)(mean + std * z[q]);)
}

static inline uint16_t to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lower = u & 0xFFFFu, upper = u >> 16;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
    return (uint16_t)upper;
}

/* bf16 inputs: the same normal values, rounded to f32 then to bf16. */
void synth_normal_bf16(uint64_t seed, uint64_t stream, int64_t offset, int64_t n,
                       double mean, double std, uint16_t *out)
{
    FOR_PAIRS(out[i] = to_bf16((float)(mean + std * z[q]));)
}

/* uniform doubles in (0, 1] (for tests that want them) */
void synth_uniform_f64(uint64_t seed, uint64_t stream, int64_t offset, int64_t n,
                       double *out)
{
    const uint64_t key = stream_key(seed, stream);
    for (int64_t i = 0; i < n; ++i) out[i] = unif(key, (uint64_t)(offset + i));
}
