/*
 * synth.c -- host (CPU) build of the seeded synthetic-input generator.
 * The definition lives in synth_core.h; this file only fills arrays.
 * Build with -ffp-contract=off so no multiply-add is fused.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SYNTH_FN static inline
#define SYNTH_ADD(a, b) ((a) + (b))
#define SYNTH_SUB(a, b) ((a) - (b))
#define SYNTH_MUL(a, b) ((a) * (b))
#define SYNTH_DIV(a, b) ((a) / (b))
#define SYNTH_SQRT(a) sqrt(a)
#include "synth_core.h"

uint64_t synth_u64(uint64_t seed, uint64_t stream, uint64_t i)
{
    return synth_u64_k(synth_key(seed, stream), i);
}

double synth_normal(uint64_t seed, uint64_t stream, uint64_t i)
{
    return synth_normal_k(synth_key(seed, stream), i);
}

/* out[i] = fp32(sigma * z[offset + i]) */
void synth_fill_normal_f32(float* out, int64_t n, uint64_t seed, uint64_t stream,
                           double sigma, int64_t offset)
{
    uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = (float)(sigma * synth_normal_k(key, (uint64_t)(offset + i)));
}

/* out[i] = bf16_rne(fp32(sigma * z[offset + i])) */
void synth_fill_normal_bf16(uint16_t* out, int64_t n, uint64_t seed, uint64_t stream,
                            double sigma, int64_t offset)
{
    uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        float f = (float)(sigma * synth_normal_k(key, (uint64_t)(offset + i)));
        uint32_t b;
        memcpy(&b, &f, 4);
        out[i] = synth_f32_to_bf16_bits(b);
    }
}

/* router logits: out[t][e] = fp32(z_le[t*E+e]) + fp32(bias_sigma * z_b[e])
 * (one fp32 addition); bias_sigma == 0 means no bias term. */
void synth_fill_logits(float* out, int64_t T, int64_t E, uint64_t seed, uint64_t stream,
                       uint64_t bias_stream, double bias_sigma)
{
    uint64_t key = synth_key(seed, stream);
    uint64_t bkey = synth_key(seed, bias_stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < T * E; ++i) {
        float l = (float)synth_normal_k(key, (uint64_t)i);
        if (bias_sigma != 0.0) {
            float b = (float)(bias_sigma * synth_normal_k(bkey, (uint64_t)(i % E)));
            l = l + b;
        }
        out[i] = l;
    }
}
