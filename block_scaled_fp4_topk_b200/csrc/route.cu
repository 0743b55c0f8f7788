// route.cu -- top-k routing.  "DGX Spark native FP4 matrix instructions ..."
// sec. 2: each token is routed to a few of the resident experts;
// "[DeepSeek V4] Triton FP4 optimisation in practice", "What is the FP4 MoE
// GEMM": 256 experts, 6 active per token.
//
// One warp per token.  Each lane keeps E/32 logits in registers; k rounds of
// a warp arg-max (largest value, lower index on ties) pick the experts in
// descending order, then the weights are the softmax over the k picks.  A NaN
// logit ranks as -inf and a pick equal to the maximum has softmax factor 1, so
// any logits give k distinct experts in [0, E) (infinities take the limit).
#include "common.cuh"
#include "kernels.cuh"

namespace ds4g {

// one token's routing by one warp: lane j < k receives the j-th pick (expert
// and softmax weight over the k picks)
template <int VPL>  // logits per lane (E <= 32 * VPL)
__device__ __forceinline__ void route_token(const float* __restrict__ l, int E, int k, int lane, int& out_e,
                                            float& out_w)
{
    float v[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        int e = i * 32 + lane;           // coalesced: lane-consecutive experts
        const float x = (e < E) ? l[e] : -INFINITY;
        v[i] = isnan(x) ? -INFINITY : x; // a NaN ranks below every number: picks stay in [0, E)
    }
    unsigned taken = 0;                  // bit i: v[i] already selected
    float sel_v = 0.f, vmax = 0.f, den = 0.f;
    int my_e = -1;
    float my_v = 0.f;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int be = 0x7FFFFFFF;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            int e = i * 32 + lane;
            bool ok = !((taken >> i) & 1u) && e < E;
            if (ok && (v[i] > bv || (v[i] == bv && e < be))) { bv = v[i]; be = e; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (j == 0) vmax = bv;
        sel_v = bv;
        float p = (sel_v == vmax) ? 1.f : expf(sel_v - vmax);   // 1 also when the maximum is +-inf
        den += p;
        if (lane == j) { my_e = be; my_v = p; }
    }
    out_e = my_e;
    out_w = __fdiv_rn(my_v, den);
}

template <int VPL>
__global__ void k_route_topk(const float* __restrict__ logits, int T, int E, int k,
                             int32_t* __restrict__ idx, float* __restrict__ w)
{
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    int e;
    float wt;
    route_token<VPL>(logits + (int64_t)t * E, E, k, lane, e, wt);
    if (lane < k) {
        idx[(int64_t)t * k + lane] = e;
        w[(int64_t)t * k + lane] = wt;
    }
}

cudaError_t launch_route_topk(const float* logits, int T, int E, int k, int32_t* idx, float* w, cudaStream_t st)
{
    if (T == 0) return cudaSuccess;
    const int threads = 256, tpb = threads / 32;
    dim3 grid((unsigned)ceil_div(T, tpb));
    if (E <= 32) k_route_topk<1><<<grid, threads, 0, st>>>(logits, T, E, k, idx, w);
    else if (E <= 64) k_route_topk<2><<<grid, threads, 0, st>>>(logits, T, E, k, idx, w);
    else if (E <= 128) k_route_topk<4><<<grid, threads, 0, st>>>(logits, T, E, k, idx, w);
    else if (E <= 256) k_route_topk<8><<<grid, threads, 0, st>>>(logits, T, E, k, idx, w);
    else if (E <= 512) k_route_topk<16><<<grid, threads, 0, st>>>(logits, T, E, k, idx, w);
    else k_route_topk<32><<<grid, threads, 0, st>>>(logits, T, E, k, idx, w);
    return cudaGetLastError();
}

}  // namespace ds4g
