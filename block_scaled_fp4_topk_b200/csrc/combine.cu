// combine.cu -- MoE combine ("Moore Threads full-link adaptation of
// DeepSeek-V4": MoE routing / dispatch / combine operators): each token's
// output row is the routing-weighted sum of its k expert output rows, summed
// in j = 0..k-1 order (a gather per token, no atomics, deterministic).  A 2-D
// grid (token, 1024-column slice) keeps a few-token decode step from running
// on a handful of CTAs; 16-byte loads and stores.
#include "common.cuh"
#include "kernels.cuh"

namespace ds4g {

__global__ void k_combine(const float* __restrict__ y2, const int32_t* __restrict__ slot_to_row,
                          const float* __restrict__ w, int k, int d, float* __restrict__ out)
{
    const int64_t t = blockIdx.x;
    const int nv = d / 4;
    for (int c = blockIdx.y * blockDim.x + threadIdx.x; c < nv; c += gridDim.y * blockDim.x) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const int64_t row = slot_to_row[t * k + j];
            const float wj = w[t * k + j];
            const float4 v = reinterpret_cast<const float4*>(y2 + row * d)[c];
            acc.x = fmaf(wj, v.x, acc.x);
            acc.y = fmaf(wj, v.y, acc.y);
            acc.z = fmaf(wj, v.z, acc.z);
            acc.w = fmaf(wj, v.w, acc.w);
        }
        reinterpret_cast<float4*>(out + t * d)[c] = acc;
    }
}

cudaError_t launch_combine(const float* y2, const int32_t* slot_to_row, const float* w, int T, int k, int d,
                           float* out, cudaStream_t st)
{
    if (T == 0) return cudaSuccess;
    int threads = d / 4 < 256 ? ((d / 4 + 31) / 32) * 32 : 256;
    if (threads < 32) threads = 32;
    // few tokens: spread each row over several CTAs so enough loads are in flight
    const int slices = T >= 2 * kNumSMs ? 1 : (int)ceil_div(d / 4, threads);
    k_combine<<<dim3(T, slices), threads, 0, st>>>(y2, slot_to_row, w, k, d, out);
    return cudaGetLastError();
}

}  // namespace ds4g
