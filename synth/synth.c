/*
 * Seeded synthetic-input generator (hot loops of synth/__init__.py).
 *
 * Holds no SharQ arithmetic: it only draws random numbers. Every value is a
 * pure function of (seed, stream, element index), so any row range can be
 * generated on its own and the result does not depend on the thread count.
 *
 *   draw i of stream (seed, stream): mix64(key + (i + 1) * GOLDEN),
 *     key = mix64(seed * GOLDEN ^ stream)   (splitmix64, Steele et al. 2014)
 *   uniform: top 53 bits * 2^-53
 *   normals 2j, 2j+1: Box-Muller on uniforms 2j (as 1 - u) and 2j+1
 *   Student-t(3) element i: Z0 / sqrt((Z1^2 + Z2^2 + Z3^2) / 3) with
 *     Z0..Z3 = normals 4i .. 4i+3
 *   fp16: clamp to +-65504, then round to nearest even (_Float16 conversion)
 */
#include <math.h>
#include <stdint.h>

#define GOLDEN 0x9E3779B97F4A7C15ull

static inline uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static inline uint64_t key_of(uint64_t seed, uint64_t stream)
{
    return mix64((seed * GOLDEN) ^ stream);
}

static inline double uniform_at(uint64_t key, uint64_t i)
{
    return (double)(mix64(key + (i + 1) * GOLDEN) >> 11) * 0x1.0p-53;
}

/* Normals 2j and 2j+1. */
static inline void normal_pair(uint64_t key, uint64_t j, double *z0, double *z1)
{
    double u1 = 1.0 - uniform_at(key, 2 * j);
    double u2 = uniform_at(key, 2 * j + 1);
    double r = sqrt(-2.0 * log(u1));
    double th = 6.283185307179586 * u2;
    *z0 = r * cos(th);
    *z1 = r * sin(th);
}

static inline uint16_t to_half_bits(double v)
{
    if (v > 65504.0)
        v = 65504.0;
    if (v < -65504.0)
        v = -65504.0;
    _Float16 h = (_Float16)v;
    uint16_t b;
    __builtin_memcpy(&b, &h, 2);
    return b;
}

void synth_normal(uint64_t seed, uint64_t stream, int64_t start, int64_t count, double *out)
{
    uint64_t key = key_of(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        uint64_t g = (uint64_t)(start + i);
        double z0, z1;
        normal_pair(key, g >> 1, &z0, &z1);
        out[i] = (g & 1) ? z1 : z0;
    }
}

/* out[r][c] = fp16(student_t3(element (row0 + r) * k + c) * gain[c]). */
void synth_student_fp16(uint64_t seed, uint64_t stream, int64_t row0, int64_t rows, int64_t k,
                        const double *gain, uint16_t *out)
{
    uint64_t key = key_of(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < k; ++c) {
            uint64_t i = (uint64_t)((row0 + r) * k + c);
            double z0, z1, z2, z3;
            normal_pair(key, 2 * i, &z0, &z1);
            normal_pair(key, 2 * i + 1, &z2, &z3);
            double t = z0 / sqrt((z1 * z1 + z2 * z2 + z3 * z3) / 3.0);
            out[r * k + c] = to_half_bits(t * gain[c]);
        }
}

/* out[r][c] = fp16(normal(element (row0 + r) * k + c) * gain[c]). */
void synth_normal_fp16(uint64_t seed, uint64_t stream, int64_t row0, int64_t rows, int64_t k,
                       const double *gain, uint16_t *out)
{
    uint64_t key = key_of(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < k; ++c) {
            uint64_t i = (uint64_t)((row0 + r) * k + c);
            double z0, z1;
            normal_pair(key, i >> 1, &z0, &z1);
            out[r * k + c] = to_half_bits(((i & 1) ? z1 : z0) * gain[c]);
        }
}
