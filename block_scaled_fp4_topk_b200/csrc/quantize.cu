// quantize.cu -- activations (bf16 / fp32) -> MXFP4, NVFP4 or MXFP8.
//
// MXFP4: "DGX Spark native FP4 matrix instructions ..." sec. 1 (E2M1 element
// with a UE8M0 scale per 32) under the OCP MX shared-exponent rule.
// NVFP4: same page, sec. 1 (kind::mxf4nvf4, UE4M3 scale per 16) with an fp32
// tensor scale.  MXFP8: the FP8 (E4M3) activations of the FP8 x FP4 GEMM
// ("[DeepSeek V4] Triton FP4 optimisation in practice", "Step 0") with a
// UE8M0 scale per 32 under the same OCP rule.  One thread quantises one block; its 32 (MX) or 16 (NV)
// inputs are read with 16-byte loads, so a warp streams contiguous memory.
#include "common.cuh"
#include "kernels.cuh"

namespace ds4g {

template <typename T>
__device__ __forceinline__ void load_block(const T* p, float* v, int n);

template <>
__device__ __forceinline__ void load_block<float>(const float* p, float* v, int n)
{
    const float4* q = reinterpret_cast<const float4*>(p);
    for (int i = 0; i < n / 4; ++i) {
        float4 f = q[i];
        v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
    }
}

template <>
__device__ __forceinline__ void load_block<uint16_t>(const uint16_t* p, float* v, int n)
{
    const uint4* q = reinterpret_cast<const uint4*>(p);
    for (int i = 0; i < n / 8; ++i) {
        uint4 u = q[i];
        uint32_t w[4] = {u.x, u.y, u.z, u.w};
        for (int j = 0; j < 4; ++j) {
            v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
            v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    }
}

// one MX block of 32 values -> 16 packed bytes + scale byte
__device__ __forceinline__ void quant_mx_block(const float* v, uint4& packed, uint8_t& scale)
{
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    int X = mx_shared_exp(amax);
    scale = (uint8_t)(X + 127);
    float inv = exp2i(-X);
    uint32_t w[4] = {0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < 32; i += 2)
        w[i >> 3] |= e2m1x2(__fmul_rn(v[i], inv), __fmul_rn(v[i + 1], inv)) << (4 * (i & 7));
    packed = make_uint4(w[0], w[1], w[2], w[3]);
}

// one NV block of 16 values -> 8 packed bytes + scale byte
__device__ __forceinline__ void quant_nv_block(const float* v, float g, uint2& packed, uint8_t& scale)
{
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    float six_g = __fmul_rn(6.0f, g);
    uint32_t s = ue4m3_encode(__fdiv_rn(amax, six_g));
    scale = (uint8_t)s;
    float ds = ue4m3_value(s);
    float denom = __fmul_rn(ds, g);
    uint32_t w[2] = {0, 0};
    if (ds == 0.0f) {
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i >> 3] |= ((__float_as_uint(v[i]) >> 28) & 8u) << (4 * (i & 7));
    } else {
#pragma unroll
        for (int i = 0; i < 16; i += 2)
            w[i >> 3] |= e2m1x2(__fdiv_rn(v[i], denom), __fdiv_rn(v[i + 1], denom)) << (4 * (i & 7));
    }
    packed = make_uint2(w[0], w[1]);
}

// one MXFP8 block of 32 values -> 32 E4M3 bytes + scale byte (OCP MX rule
// with the E4M3 element, whose largest exponent is 8)
__device__ __forceinline__ void quant_mx8_block(const float* v, uint4* codes, uint8_t& scale)
{
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const int X = mx_shared_exp<8>(amax);
    scale = (uint8_t)(X + 127);
    const float inv = exp2i(-X);
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        w[i] = e4m3x2(__fmul_rn(v[4 * i], inv), __fmul_rn(v[4 * i + 1], inv)) |
               (e4m3x2(__fmul_rn(v[4 * i + 2], inv), __fmul_rn(v[4 * i + 3], inv)) << 16);
    codes[0] = make_uint4(w[0], w[1], w[2], w[3]);
    codes[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

template <typename T>
__global__ void k_quant_mx8(const T* __restrict__ x, int64_t nblocks, uint8_t* __restrict__ data,
                            uint8_t* __restrict__ scales)
{
    for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < nblocks;
         b += (int64_t)gridDim.x * blockDim.x) {
        float v[32];
        load_block<T>(x + b * 32, v, 32);
        uint8_t s;
        quant_mx8_block(v, reinterpret_cast<uint4*>(data) + 2 * b, s);
        scales[b] = s;
    }
}

template <typename T>
__global__ void k_quant_mx(const T* __restrict__ x, int64_t nblocks, int64_t K,
                           uint8_t* __restrict__ data, uint8_t* __restrict__ scales)
{
    for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < nblocks;
         b += (int64_t)gridDim.x * blockDim.x) {
        float v[32];
        load_block<T>(x + b * 32, v, 32);
        uint4 p;
        uint8_t s;
        quant_mx_block(v, p, s);
        reinterpret_cast<uint4*>(data)[b] = p;
        scales[b] = s;
    }
}

// amax of |x| over n elements into *amax_bits (fp32 bits; non-negative floats
// order like unsigned integers)
template <typename T>
__global__ void k_amax(const T* __restrict__ x, int64_t n, unsigned int* amax_bits)
{
    float m = 0.f;
    for (int64_t i = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) * 8; i < n;
         i += (int64_t)gridDim.x * blockDim.x * 8) {
        float v[8];
        load_block<T>(x + i, v, 8);
#pragma unroll
        for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

// g = amax / 2688 (1 if amax is 0), fp32 IEEE division
__global__ void k_g_from_amax(const unsigned int* amax_bits, float* g)
{
    float a = __uint_as_float(*amax_bits);
    *g = (a == 0.0f) ? 1.0f : __fdiv_rn(a, 2688.0f);
}

template <typename T>
__global__ void k_quant_nv(const T* __restrict__ x, int64_t nblocks, const float* __restrict__ g_ptr,
                           uint8_t* __restrict__ data, uint8_t* __restrict__ scales)
{
    const float g = *g_ptr;
    for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < nblocks;
         b += (int64_t)gridDim.x * blockDim.x) {
        float v[16];
        load_block<T>(x + b * 16, v, 16);
        uint2 p;
        uint8_t s;
        quant_nv_block(v, g, p, s);
        reinterpret_cast<uint2*>(data)[b] = p;
        scales[b] = s;
    }
}

static int grid_1d(int64_t work, int threads)
{
    int64_t g = ceil_div(work, threads);
    int64_t cap = (int64_t)kNumSMs * 16;
    return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

cudaError_t launch_quantize(const void* x, int dtype, int64_t rows, int64_t K, int fmt, const float* g_in,
                            uint8_t* data, uint8_t* scales, float* g_out, void* ws, cudaStream_t st)
{
    const int64_t n = rows * K;
    if (n == 0) return cudaSuccess;
    if (fmt == DS4G_MXFP8) {
        const int64_t nb = n / 32;
        if (dtype == DS4G_BF16)
            k_quant_mx8<uint16_t><<<grid_1d(nb, 256), 256, 0, st>>>((const uint16_t*)x, nb, data, scales);
        else
            k_quant_mx8<float><<<grid_1d(nb, 256), 256, 0, st>>>((const float*)x, nb, data, scales);
        return cudaGetLastError();
    }
    if (fmt == DS4G_MXFP4) {
        const int64_t nb = n / 32;
        if (dtype == DS4G_BF16)
            k_quant_mx<uint16_t><<<grid_1d(nb, 256), 256, 0, st>>>((const uint16_t*)x, nb, K, data, scales);
        else
            k_quant_mx<float><<<grid_1d(nb, 256), 256, 0, st>>>((const float*)x, nb, K, data, scales);
        return cudaGetLastError();
    }
    const int64_t nb = n / 16;
    const float* g = g_in;
    if (!g_in) {
        unsigned int* amax = reinterpret_cast<unsigned int*>(ws);
        cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(unsigned int), st);
        if (e != cudaSuccess) return e;
        if (dtype == DS4G_BF16)
            k_amax<uint16_t><<<grid_1d(n / 8, 256), 256, 0, st>>>((const uint16_t*)x, n, amax);
        else
            k_amax<float><<<grid_1d(n / 8, 256), 256, 0, st>>>((const float*)x, n, amax);
        k_g_from_amax<<<1, 1, 0, st>>>(amax, g_out);
        g = g_out;
    } else if (g_out && g_out != g_in) {
        cudaError_t e = cudaMemcpyAsync(g_out, g_in, sizeof(float), cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return e;
    }
    if (dtype == DS4G_BF16)
        k_quant_nv<uint16_t><<<grid_1d(nb, 256), 256, 0, st>>>((const uint16_t*)x, nb, g, data, scales);
    else
        k_quant_nv<float><<<grid_1d(nb, 256), 256, 0, st>>>((const float*)x, nb, g, data, scales);
    return cudaGetLastError();
}

}  // namespace ds4g
