// swiglu.cu -- SwiGLU + requantisation as its own step (the fused "SwiGLU +
// quant" pattern of "Moore Threads full-link adaptation of DeepSeek-V4",
// here requantising to FP4).  h = silu(gate) * up with silu(x) = x/(1+e^-x),
// gate = column i, up = column I + i of the FC1 output; h is quantised by the
// same MX / NV rule as the activations.  One warp handles 32 consecutive
// columns of one row (one MX block, or two NV blocks).
#include "common.cuh"
#include "kernels.cuh"

namespace ds4g {

template <int FMT>
__global__ void k_swiglu_requant(const float* __restrict__ y1, int64_t rows, int I, uint8_t* __restrict__ hd,
                                 uint8_t* __restrict__ hs, const float* __restrict__ hg, float* __restrict__ h_debug)
{
    const int lane = threadIdx.x & 31;
    const int64_t nb = (int64_t)I / 32;
    const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (wid >= rows * nb) return;
    const int64_t row = wid / nb, b = wid % nb;
    const int col = (int)(b * 32) + lane;
    const float g = y1[row * 2 * I + col];
    const float u = y1[row * 2 * I + I + col];
    const float h = swiglu_f32(g, u);
    if (h_debug) h_debug[row * I + col] = h;
    uint32_t code;
    if (FMT == DS4G_MXFP4) {
        float m = fabsf(h);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const int X = mx_shared_exp(m);
        code = e2m1_code(__fmul_rn(h, exp2i(-X)));
        if (lane == 0) hs[row * nb + b] = (uint8_t)(X + 127);
    } else {
        float m = fabsf(h);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float gh = *hg;
        const uint32_t s = ue4m3_encode(__fdiv_rn(m, __fmul_rn(6.0f, gh)));
        const float ds = ue4m3_value(s);
        code = (ds == 0.0f) ? ((__float_as_uint(h) >> 28) & 8u) : e2m1_code(__fdiv_rn(h, __fmul_rn(ds, gh)));
        if ((lane & 15) == 0) hs[row * (I / 16) + b * 2 + (lane >> 4)] = (uint8_t)s;
    }
    const uint32_t hi_code = __shfl_down_sync(0xffffffffu, code, 1);
    if ((lane & 1) == 0) hd[row * (I / 2) + b * 16 + (lane >> 1)] = (uint8_t)(code | (hi_code << 4));
}

cudaError_t launch_swiglu_requant(const float* y1, int64_t rows, int I, int fmt, uint8_t* hd, uint8_t* hs,
                                  const float* hg, float* h_debug, cudaStream_t st)
{
    const int64_t warps = rows * (I / 32);
    if (warps == 0) return cudaSuccess;
    const unsigned grid = (unsigned)ceil_div(warps, 8);
    if (fmt == DS4G_MXFP4) k_swiglu_requant<DS4G_MXFP4><<<grid, 256, 0, st>>>(y1, rows, I, hd, hs, hg, h_debug);
    else k_swiglu_requant<DS4G_NVFP4><<<grid, 256, 0, st>>>(y1, rows, I, hd, hs, hg, h_debug);
    return cudaGetLastError();
}

}  // namespace ds4g
