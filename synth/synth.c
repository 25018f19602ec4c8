/*
 * Seeded, counter-based input generator for the WKV workloads.
 *
 * This file draws the synthetic inputs (w, u, k, v, mu, x) that both the
 * fp64 oracle and the CUDA path consume.  It holds none of the WKV
 * arithmetic: it only turns (seed, stream, index) into numbers with a stated
 * distribution, so that any single element can be regenerated on its own
 * (the oracle can recompute a sampled channel of a 137 GB warm-up without
 * materialising the rest).
 *
 * Generator: SplitMix64 (G. L. Steele, D. Lea, C. H. Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014), used as a counter-based
 * hash: the n-th 64-bit word of a stream is mix64(key + n * GAMMA), with the
 * stream key itself derived from (seed, stream) by the same mixer.
 * Uniforms take the top 53 bits, offset by one half so they lie strictly in
 * (0, 1).  Normals use the Box-Muller transform (G. E. P. Box, M. E. Muller,
 * "A note on the generation of random normal deviates", Ann. Math. Stat.
 * 1958), cosine branch only, one normal per element from two uniforms of the
 * same element.  Everything is computed in double and rounded once to fp32.
 *
 * Element i of a stream is a pure function of (seed, stream, i), so the
 * result does not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream)
{
    return mix64(mix64(seed + SYNTH_GAMMA) + (stream + 1) * SYNTH_GAMMA);
}

/* Word number `ctr` of the stream with key `key`. */
static inline uint64_t word_at(uint64_t key, uint64_t ctr)
{
    return mix64(key + (ctr + 1) * SYNTH_GAMMA);
}

/* Uniform in the open interval (0, 1) with 53 random bits. */
static inline double unit_open(uint64_t x)
{
    return ((double)(x >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

static inline double normal_at(uint64_t key, uint64_t idx)
{
    const double two_pi = 6.283185307179586476925286766559;
    double u1 = unit_open(word_at(key, 2 * idx));
    double u2 = unit_open(word_at(key, 2 * idx + 1));
    return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

static inline double uniform_at(uint64_t key, uint64_t idx)
{
    return unit_open(word_at(key, 2 * idx));
}

/* out[i] = mean + std * N(0,1) at element (offset + i). */
void synth_normal_f32(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n,
                      double mean, double std, float* out)
{
    uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = (float)(mean + std * normal_at(key, offset + (uint64_t)i));
}

/* out[i] = lo + (hi - lo) * U(0,1) at element (offset + i). */
void synth_uniform_f32(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n,
                       double lo, double hi, float* out)
{
    uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = (float)(lo + (hi - lo) * uniform_at(key, offset + (uint64_t)i));
}

/* out[i] = exp(lo + (hi - lo) * U(0,1)): a log-uniform positive rate. */
void synth_exp_uniform_f32(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n,
                           double lo, double hi, float* out)
{
    uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = (float)exp(lo + (hi - lo) * uniform_at(key, offset + (uint64_t)i));
}

/* Where U(0,1) < prob at element (offset + i), overwrite inout[i] with value. */
void synth_spike_f32(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n,
                     double prob, double value, float* inout)
{
    uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        if (uniform_at(key, offset + (uint64_t)i) < prob) inout[i] = (float)value;
}

/* Gathered forms: element idx[i] of the stream, for sampled recomputation. */
void synth_normal_f32_at(uint64_t seed, uint64_t stream, const int64_t* idx, int64_t n,
                         double mean, double std, float* out)
{
    uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = (float)(mean + std * normal_at(key, (uint64_t)idx[i]));
}

void synth_spike_f32_at(uint64_t seed, uint64_t stream, const int64_t* idx, int64_t n,
                        double prob, double value, float* inout)
{
    uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        if (uniform_at(key, (uint64_t)idx[i]) < prob) inout[i] = (float)value;
}

/* Raw 64-bit words, exposed so tests can check the mixer against its definition. */
void synth_words(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, uint64_t* out)
{
    uint64_t key = stream_key(seed, stream);
    for (int64_t i = 0; i < n; ++i) out[i] = word_at(key, offset + (uint64_t)i);
}
