/*
 * synth.c - seeded synthetic inputs for the pooled-wave MoE dispatch/combine path.
 *
 * Every value is a pure function of (seed, stream, index): a counter-based
 * SplitMix64 stream (Steele, Lea & Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014), uniform doubles from its top 53 bits and normals by
 * the Box-Muller transform (cosine branch).  Any slice can be regenerated on its
 * own and the output does not depend on the number of OpenMP threads.
 *
 * This file only makes inputs (router logits, latent rows, per-expert scales).
 * It holds none of the routing, packing or combining arithmetic; the CUDA
 * library and the CPU oracle both consume what it writes.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>

#define SM64_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t sm64_mix(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Starting state of the stream (seed, stream). */
static inline uint64_t stream_key(uint64_t seed, uint64_t stream)
{
    return sm64_mix(sm64_mix(seed + SM64_GAMMA) + (stream + 1) * SM64_GAMMA);
}

/* i-th output of the SplitMix64 sequence that starts at `key`. */
static inline uint64_t draw_u64(uint64_t key, uint64_t i)
{
    return sm64_mix(key + (i + 1) * SM64_GAMMA);
}

static inline double draw_uniform(uint64_t key, uint64_t i)
{
    return (double)(draw_u64(key, i) >> 11) * 0x1.0p-53; /* [0, 1) */
}

/* n-th standard normal of the stream: uniforms 2n and 2n+1, Box-Muller. */
static inline double draw_normal(uint64_t key, uint64_t n)
{
    double u1 = draw_uniform(key, 2 * n);
    double u2 = draw_uniform(key, 2 * n + 1);
    double r = sqrt(-2.0 * log(1.0 - u1)); /* 1-u1 in (0,1] */
    return r * cos(6.283185307179586 * u2);
}

/* fp32 -> bf16 bits, round to nearest even (finite inputs). */
static inline uint16_t f32_bits_to_bf16(float f)
{
    union { float f; uint32_t u; } v;
    v.f = f;
    uint32_t u = v.u;
    return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

/* stream ids */
enum { ST_LOGIT = 1, ST_SEQBIAS = 2, ST_X = 3, ST_SCALE = 4, ST_PERM = 5, ST_DOUT = 6 };
/* streams >= 16 are free for named matrices (activations, projection weights) */

/*
 * Router logits, row-major [T, E] fp32.
 *   kind 0: iid N(0,1)
 *   kind 1: N(0,1) + sigma_b * N(0,1) bias drawn per (sequence, expert),
 *           sequence = t / seq_len
 *   kind 2: N(0,1) - ln(rank_e), rank_e = 1 + pi(e), pi a seeded permutation
 *           (Zipf popularity with exponent 1 over a shuffled expert order)
 * The sum is formed in double and rounded once to fp32.
 */
int synth_logits_rows(int kind, int64_t t0, int64_t T, int32_t E, int64_t seq_len,
                      double sigma_b, uint64_t seed, float *out);

int synth_logits(int kind, int64_t T, int32_t E, int64_t seq_len, double sigma_b,
                 uint64_t seed, float *out)
{
    return synth_logits_rows(kind, 0, T, E, seq_len, sigma_b, seed, out);
}

/* Rows t0 .. t0+T-1 of the same logits (a slice of a larger batch). */
int synth_logits_rows(int kind, int64_t t0, int64_t T, int32_t E, int64_t seq_len,
                      double sigma_b, uint64_t seed, float *out)
{
    if (t0 < 0 || T < 0 || E <= 0 || !out) return -1;
    if (kind == 1 && seq_len <= 0) return -1;
    const uint64_t kz = stream_key(seed, ST_LOGIT);
    const uint64_t kb = stream_key(seed, ST_SEQBIAS);
    double lnrank[4096];
    if (kind == 2) {
        if (E > 4096) return -1;
        const uint64_t kp = stream_key(seed, ST_PERM);
        for (int32_t e = 0; e < E; ++e) {
            uint64_t ke = draw_u64(kp, (uint64_t)e);
            int64_t before = 0; /* position of e when experts are sorted by key, ties by id */
            for (int32_t f = 0; f < E; ++f) {
                uint64_t kf = draw_u64(kp, (uint64_t)f);
                if (kf < ke || (kf == ke && f < e)) ++before;
            }
            lnrank[e] = log((double)(1 + before));
        }
    }
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < T; ++i) {
        const int64_t t = t0 + i;
        for (int32_t e = 0; e < E; ++e) {
            double v = draw_normal(kz, (uint64_t)t * (uint64_t)E + (uint64_t)e);
            if (kind == 1) {
                uint64_t s = (uint64_t)(t / seq_len);
                v += sigma_b * draw_normal(kb, s * (uint64_t)E + (uint64_t)e);
            } else if (kind == 2) {
                v -= lnrank[e];
            }
            out[i * E + e] = (float)v;
        }
    }
    return 0;
}

/* Latent rows t0 .. t0+T-1, row-major [T, D] bf16 bits: N(0,1) rounded to
 * fp32, then to bf16 (RNE). */
int synth_x_bf16_rows(int64_t t0, int64_t T, int32_t D, uint64_t seed, uint16_t *out)
{
    if (t0 < 0 || T < 0 || D <= 0 || !out) return -1;
    const uint64_t kx = stream_key(seed, ST_X);
    const int64_t n = T * (int64_t)D, i0 = t0 * (int64_t)D;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = f32_bits_to_bf16((float)draw_normal(kx, (uint64_t)(i0 + i)));
    return 0;
}

int synth_x_bf16(int64_t T, int32_t D, uint64_t seed, uint16_t *out)
{
    return synth_x_bf16_rows(0, T, D, seed, out);
}

/* Upstream gradient dL/dout, row-major [T, D] fp32: N(0,1) rounded to fp32. */
int synth_dout_f32(int64_t T, int32_t D, uint64_t seed, float *out)
{
    if (T < 0 || D <= 0 || !out) return -1;
    const uint64_t kd = stream_key(seed, ST_DOUT);
    const int64_t n = T * (int64_t)D;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = (float)draw_normal(kd, (uint64_t)i);
    return 0;
}

/* A named bf16 matrix [rows, cols]: N(0, std^2) rounded to fp32, then to bf16
 * (activations and synthetic random-init projection weights). */
int synth_matrix_bf16(int64_t rows, int64_t cols, double std, uint64_t seed, uint64_t stream,
                      uint16_t *out)
{
    if (rows < 0 || cols <= 0 || !out || stream < 16) return -1;
    const uint64_t km = stream_key(seed, stream);
    const int64_t n = rows * cols;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = f32_bits_to_bf16((float)(std * draw_normal(km, (uint64_t)i)));
    return 0;
}

/* Per-expert scales s_e ~ U(lo, hi), fp32. */
int synth_scales(int32_t E, double lo, double hi, uint64_t seed, float *out)
{
    if (E <= 0 || !out) return -1;
    const uint64_t ks = stream_key(seed, ST_SCALE);
    for (int32_t e = 0; e < E; ++e)
        out[e] = (float)(lo + (hi - lo) * draw_uniform(ks, (uint64_t)e));
    return 0;
}

/* Raw stream access, for the generator's own tests. */
uint64_t synth_u64(uint64_t seed, uint64_t stream, uint64_t i)
{
    return draw_u64(stream_key(seed, stream), i);
}

double synth_normal(uint64_t seed, uint64_t stream, uint64_t n)
{
    return draw_normal(stream_key(seed, stream), n);
}
