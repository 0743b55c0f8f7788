/*
 * synth_cuda.cu -- device (GPU) build of the seeded synthetic-input generator.
 * The definition lives in synth_core.h; every double operation is an
 * explicitly rounded intrinsic so nothing is contracted into an FMA, which
 * keeps the values bit-identical to the host build in synth.c.
 */
#include <cuda_runtime.h>
#include <stdint.h>

#define SYNTH_FN static __device__ __forceinline__
#define SYNTH_ADD(a, b) __dadd_rn((a), (b))
#define SYNTH_SUB(a, b) __dsub_rn((a), (b))
#define SYNTH_MUL(a, b) __dmul_rn((a), (b))
#define SYNTH_DIV(a, b) __ddiv_rn((a), (b))
#define SYNTH_SQRT(a) __dsqrt_rn(a)
#include "synth_core.h"

static __global__ void k_fill_f32(float* out, int64_t n, uint64_t seed, uint64_t stream, double sigma, int64_t offset)
{
    const uint64_t key = synth_key(seed, stream);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        out[i] = __double2float_rn(__dmul_rn(sigma, synth_normal_k(key, (uint64_t)(offset + i))));
}

static __global__ void k_fill_bf16(uint16_t* out, int64_t n, uint64_t seed, uint64_t stream, double sigma, int64_t offset)
{
    const uint64_t key = synth_key(seed, stream);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        float f = __double2float_rn(__dmul_rn(sigma, synth_normal_k(key, (uint64_t)(offset + i))));
        out[i] = synth_f32_to_bf16_bits(__float_as_uint(f));
    }
}

static __global__ void k_fill_logits(float* out, int64_t T, int64_t E, uint64_t seed, uint64_t stream,
                                     uint64_t bias_stream, double bias_sigma)
{
    const uint64_t key = synth_key(seed, stream);
    const uint64_t bkey = synth_key(seed, bias_stream);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < T * E;
         i += (int64_t)gridDim.x * blockDim.x) {
        float l = __double2float_rn(synth_normal_k(key, (uint64_t)i));
        if (bias_sigma != 0.0) {
            float b = __double2float_rn(__dmul_rn(bias_sigma, synth_normal_k(bkey, (uint64_t)(i % E))));
            l = __fadd_rn(l, b);
        }
        out[i] = l;
    }
}

static int grid_for(int64_t n)
{
    int64_t g = (n + 255) / 256;
    if (g > 148 * 64) g = 148 * 64;
    if (g < 1) g = 1;
    return (int)g;
}

extern "C" int synth_cuda_fill_normal_f32(float* out, int64_t n, uint64_t seed, uint64_t stream,
                                          double sigma, int64_t offset, cudaStream_t st)
{
    if (n <= 0) return 0;
    k_fill_f32<<<grid_for(n), 256, 0, st>>>(out, n, seed, stream, sigma, offset);
    return (int)cudaGetLastError();
}

extern "C" int synth_cuda_fill_normal_bf16(uint16_t* out, int64_t n, uint64_t seed, uint64_t stream,
                                           double sigma, int64_t offset, cudaStream_t st)
{
    if (n <= 0) return 0;
    k_fill_bf16<<<grid_for(n), 256, 0, st>>>(out, n, seed, stream, sigma, offset);
    return (int)cudaGetLastError();
}

extern "C" int synth_cuda_fill_logits(float* out, int64_t T, int64_t E, uint64_t seed, uint64_t stream,
                                      uint64_t bias_stream, double bias_sigma, cudaStream_t st)
{
    if (T * E <= 0) return 0;
    k_fill_logits<<<grid_for(T * E), 256, 0, st>>>(out, T, E, seed, stream, bias_stream, bias_sigma);
    return (int)cudaGetLastError();
}
