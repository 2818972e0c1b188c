/*
 * synth.c -- seeded synthetic inputs shared by the tests, the oracle runs and bench.py.
 *
 * Holds none of the layer's arithmetic: only random numbers and their rounding to
 * binary16.  Every value is a pure function of (seed, stream, index), so any slice can
 * be generated independently and in parallel.
 *
 *   splitmix64 (S. Vigna's published generator): the generator seeded with s yields, as
 *   its i-th output (i = 0, 1, ...), mix(s + (i + 1) * 0x9E3779B97F4A7C15), where mix is
 *   the published splitmix64 finaliser.  A stream key is output #stream of the generator
 *   seeded with the user seed; element i of a stream is output #i of the generator seeded
 *   with the stream key.
 *   uniform  = (u64 >> 11) * 2^-53                   in [0, 1)
 *   normals  = Box-Muller on the uniform pair (2p, 2p+1):
 *              r = sqrt(-2 ln(1 - u0)), z(2p) = r cos(2 pi u1), z(2p+1) = r sin(2 pi u1)
 *   binary16 = the double value rounded to float, then to binary16 (both to nearest even).
 */
#include <math.h>
#include <stdint.h>

#define GOLDEN_GAMMA 0x9E3779B97F4A7C15ULL

static uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t synth_u64(uint64_t key, uint64_t index) { return mix64(key + (index + 1) * GOLDEN_GAMMA); }

uint64_t synth_stream_key(uint64_t seed, uint64_t stream) { return synth_u64(seed, stream); }

static double uniform01(uint64_t key, uint64_t index)
{
    return (double)(synth_u64(key, index) >> 11) * (1.0 / 9007199254740992.0);
}

double synth_uniform(uint64_t key, uint64_t index) { return uniform01(key, index); }

double synth_normal(uint64_t key, uint64_t index)
{
    uint64_t pair = index / 2;
    double u0 = uniform01(key, 2 * pair);
    double u1 = uniform01(key, 2 * pair + 1);
    double r = sqrt(-2.0 * log(1.0 - u0));
    double angle = 6.283185307179586 * u1;
    return (index & 1) ? r * sin(angle) : r * cos(angle);
}

static uint16_t to_half_bits(double v)
{
    _Float16 h = (_Float16)(float)v;
    uint16_t bits;
    __builtin_memcpy(&bits, &h, sizeof bits);
    return bits;
}

/* out[i*cols + j] = binary16(mean + std * z(i*cols + j) * col_factor[j]); col_factor may be NULL */
void synth_normal_matrix_f16(uint64_t key, int64_t rows, int64_t cols, double mean, double std,
                             const double *col_factor, uint16_t *out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t j = 0; j < cols; ++j) {
            uint64_t idx = (uint64_t)(i * cols + j);
            double f = col_factor ? col_factor[j] : 1.0;
            out[idx] = to_half_bits(mean + std * synth_normal(key, idx) * f);
        }
}

/* `count` distinct column indices of [0, n), by a partial Fisher-Yates shuffle driven by
 * the stream `key`; returned in the order drawn.  scratch must hold n int32. */
void synth_choose_distinct(uint64_t key, int64_t n, int64_t count, int32_t *scratch, int32_t *out)
{
    for (int64_t i = 0; i < n; ++i) scratch[i] = (int32_t)i;
    for (int64_t i = 0; i < count; ++i) {
        uint64_t span = (uint64_t)(n - i);
        int64_t j = i + (int64_t)(synth_u64(key, (uint64_t)i) % span);
        int32_t t = scratch[i];
        scratch[i] = scratch[j];
        scratch[j] = t;
        out[i] = scratch[i];
    }
}
