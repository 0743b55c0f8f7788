// dispatch.cu -- routing, activation quantisation and the expert-contiguous
// permutation of one batch as a single call (ds4g_moe_dispatch).
//
// The three steps are the ones of route.cu ("[DeepSeek V4] Triton FP4
// optimisation in practice", "What is the FP4 MoE GEMM": top-6 of 256
// experts), quantize.cu ("DGX Spark native FP4 matrix instructions ..."
// sec. 1: E2M1 with UE8M0 per 32 / UE4M3 per 16) and permute.cu ("Step 0":
// the grouped GEMM takes each expert's rows as one contiguous segment), with
// the same per-token routing and per-block quantisation functions, so the
// results are bit-identical to calling them one after the other.
//
// Up to kDispatchSmallS slots (decode batches) one CTA does all of it:
// every warp routes tokens, the CTA counts the picks per expert, one warp
// scans and ranks them stably, and then each token row is quantised once and
// its packed blocks are written both to x_q and to the token's k permuted
// rows (no second pass that reads x_q back).  Larger batches run the
// separate calls' routing and ranking kernels, then one quantise-and-scatter
// pass.
#include "common.cuh"
#include "kernels.cuh"

namespace ds4g {

constexpr int kDispatchSmallS = 512;
constexpr int kDispatchThreads = 512;

template <int VPL, typename T, int FMT>
__global__ void __launch_bounds__(kDispatchThreads)
k_dispatch_small(const float* __restrict__ logits, const T* __restrict__ x, int Tn, int E, int k, int64_t d,
                 const float* __restrict__ g_in, int32_t* __restrict__ idx, float* __restrict__ w,
                 uint8_t* __restrict__ xd, uint8_t* __restrict__ xs, float* __restrict__ xg,
                 int32_t* __restrict__ offsets, int32_t* __restrict__ row_to_slot, int32_t* __restrict__ slot_to_row,
                 uint8_t* __restrict__ ad, uint8_t* __restrict__ as, float* __restrict__ ag)
{
    extern __shared__ int32_t sh[];
    // the next kernel on the stream (FC1) may launch now and set itself up
    // on the SMs this one-CTA kernel leaves idle; it reads nothing of ours
    // before this grid has finished
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int S = Tn * k;
    int32_t* sidx = sh;               // [S]  picked expert of each slot
    int32_t* cnt = sidx + S;          // [E]  picks per expert, then running ranks
    int32_t* off = cnt + E;           // [E + 1]
    int32_t* s2r = off + E + 1;       // [S]  slot -> permuted row
    __shared__ unsigned int s_amax;
    __shared__ float s_g;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;

    // 1. routing: one warp per token
    for (int t = warp; t < Tn; t += nwarps) {
        int e;
        float wt;
        route_token<VPL>(logits + (int64_t)t * E, E, k, lane, e, wt);
        if (lane < k) {
            idx[(int64_t)t * k + lane] = e;
            w[(int64_t)t * k + lane] = wt;
            sidx[t * k + lane] = e;
        }
    }
    for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
    if (tid == 0) s_amax = 0u;
    __syncthreads();

    // 2. picks per expert; for NVFP4 without a given tensor scale, amax |x|
    for (int s = tid; s < S; s += blockDim.x) atomicAdd(&cnt[sidx[s]], 1);
    if (FMT == DS4G_NVFP4 && g_in == nullptr) {
        float m = 0.f;
        const int64_t n = (int64_t)Tn * d;
        for (int64_t i = (int64_t)tid * 8; i < n; i += (int64_t)blockDim.x * 8) {
            float v[8];
            load_block<T>(x + i, v, 8);
#pragma unroll
            for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) atomicMax(&s_amax, __float_as_uint(m));
    }
    __syncthreads();

    // 3. offsets and stable ranks (ascending slot id inside each expert)
    if (warp == 0) {
        const int per = (E + 31) / 32;
        int32_t sum = 0;
        for (int i = 0; i < per; ++i) {
            const int e = lane * per + i;
            if (e < E) sum += cnt[e];
        }
        int32_t incl = sum;
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int32_t run = incl - sum;
        for (int i = 0; i < per; ++i) {
            const int e = lane * per + i;
            if (e < E) {
                off[e] = run;
                offsets[e] = run;
                run += cnt[e];
                cnt[e] = 0;
            }
        }
        if (lane == 31) offsets[E] = incl;
        __syncwarp();
        for (int g = 0; g < S; g += 32) {
            const int s = g + lane;
            const bool valid = s < S;
            const int e = valid ? sidx[s] : -1 - lane;
            const unsigned peers = __match_any_sync(0xffffffffu, e);
            const int rank = __popc(peers & ((1u << lane) - 1u));
            int32_t pos = 0;
            if (valid) pos = off[e] + cnt[e] + rank;
            __syncwarp();
            if (valid && rank == 0) cnt[e] += __popc(peers);
            __syncwarp();
            if (valid) {
                s2r[s] = pos;
                row_to_slot[pos] = s;
                slot_to_row[s] = pos;
            }
        }
    }
    if (FMT == DS4G_NVFP4 && tid == 32) {
        const float a = __uint_as_float(s_amax);
        const float g = g_in ? *g_in : ((a == 0.0f) ? 1.0f : __fdiv_rn(a, 2688.0f));
        s_g = g;
        *xg = g;
        *ag = g;
    }
    __syncthreads();

    // 4. quantise each token's blocks once; write x_q and the k permuted rows
    constexpr int BLK = (FMT == DS4G_MXFP4) ? 32 : 16;
    const int64_t bpr = d / BLK;
    const int64_t nb = (int64_t)Tn * bpr;
    for (int64_t b = tid; b < nb; b += blockDim.x) {
        const int t = (int)(b / bpr);
        const int64_t c = b - (int64_t)t * bpr;
        float v[BLK];
        load_block<T>(x + (int64_t)t * d + c * BLK, v, BLK);
        if (FMT == DS4G_MXFP4) {
            uint4 pk;
            uint8_t sc;
            quant_mx_block(v, pk, sc);
            *reinterpret_cast<uint4*>(xd + (int64_t)t * (d / 2) + c * 16) = pk;
            xs[(int64_t)t * bpr + c] = sc;
            for (int j = 0; j < k; ++j) {
                const int64_t r = s2r[t * k + j];
                *reinterpret_cast<uint4*>(ad + r * (d / 2) + c * 16) = pk;
                as[r * bpr + c] = sc;
            }
        } else {
            uint2 pk;
            uint8_t sc;
            quant_nv_block(v, s_g, pk, sc);
            *reinterpret_cast<uint2*>(xd + (int64_t)t * (d / 2) + c * 8) = pk;
            xs[(int64_t)t * bpr + c] = sc;
            for (int j = 0; j < k; ++j) {
                const int64_t r = s2r[t * k + j];
                *reinterpret_cast<uint2*>(ad + r * (d / 2) + c * 8) = pk;
                as[r * bpr + c] = sc;
            }
        }
    }
}

// larger batches: the permutation is ranked first, then each token row is
// quantised once and written to x_q and to its k permuted rows (the separate
// calls quantise, then gather the rows back out of x_q)
template <typename T, int FMT>
__global__ void k_quant_scatter(const T* __restrict__ x, int Tn, int64_t d, int k, const float* __restrict__ g_ptr,
                                const int32_t* __restrict__ slot_to_row, uint8_t* __restrict__ xd,
                                uint8_t* __restrict__ xs, uint8_t* __restrict__ ad, uint8_t* __restrict__ as,
                                float* __restrict__ ag)
{
    constexpr int BLK = (FMT == DS4G_MXFP4) ? 32 : 16;
    const float g = (FMT == DS4G_NVFP4) ? *g_ptr : 1.0f;
    if (FMT == DS4G_NVFP4 && blockIdx.x == 0 && threadIdx.x == 0) *ag = g;
    const int64_t bpr = d / BLK;
    const int64_t nb = (int64_t)Tn * bpr;
    for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < nb; b += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = b / bpr;
        const int64_t c = b - t * bpr;
        float v[BLK];
        load_block<T>(x + t * d + c * BLK, v, BLK);
        if (FMT == DS4G_MXFP4) {
            uint4 pk;
            uint8_t sc;
            quant_mx_block(v, pk, sc);
            reinterpret_cast<uint4*>(xd)[b] = pk;
            xs[b] = sc;
            for (int j = 0; j < k; ++j) {
                const int64_t r = slot_to_row[t * k + j];
                *reinterpret_cast<uint4*>(ad + r * (d / 2) + c * 16) = pk;
                as[r * bpr + c] = sc;
            }
        } else {
            uint2 pk;
            uint8_t sc;
            quant_nv_block(v, g, pk, sc);
            reinterpret_cast<uint2*>(xd)[b] = pk;
            xs[b] = sc;
            for (int j = 0; j < k; ++j) {
                const int64_t r = slot_to_row[t * k + j];
                *reinterpret_cast<uint2*>(ad + r * (d / 2) + c * 8) = pk;
                as[r * bpr + c] = sc;
            }
        }
    }
}

size_t dispatch_workspace_bytes(int T, int k, int E, int fmt, int has_g_in)
{
    // the multi-kernel path: the permutation's counts, then the quantiser's
    // amax word (16-byte aligned)
    const size_t pw = (permute_workspace_bytes(T, k, E) + 15) / 16 * 16;
    return pw + ((fmt == DS4G_NVFP4 && !has_g_in) ? 16 : 0);
}

template <typename T, int FMT>
static cudaError_t launch_small(const float* logits, const T* x, int Tn, int E, int k, int64_t d, const float* g_in,
                                int32_t* idx, float* w, uint8_t* xd, uint8_t* xs, float* xg, int32_t* offsets,
                                int32_t* r2s, int32_t* s2r, uint8_t* ad, uint8_t* as, float* ag, cudaStream_t st)
{
    const int S = Tn * k;
    const size_t shm = (size_t)(2 * S + 2 * E + 1) * sizeof(int32_t);
#define DS4G_DISPATCH(VPL)                                                                                           \
    k_dispatch_small<VPL, T, FMT><<<1, kDispatchThreads, shm, st>>>(logits, x, Tn, E, k, d, g_in, idx, w, xd, xs, xg, \
                                                                   offsets, r2s, s2r, ad, as, ag)
    if (E <= 32) DS4G_DISPATCH(1);
    else if (E <= 64) DS4G_DISPATCH(2);
    else if (E <= 128) DS4G_DISPATCH(4);
    else if (E <= 256) DS4G_DISPATCH(8);
    else if (E <= 512) DS4G_DISPATCH(16);
    else DS4G_DISPATCH(32);
#undef DS4G_DISPATCH
    return cudaGetLastError();
}

cudaError_t launch_dispatch(const float* logits, const void* x, int dtype, int Tn, int E, int k, int64_t d, int fmt,
                            const float* g_in, int32_t* idx, float* w, uint8_t* xd, uint8_t* xs, float* xg,
                            int32_t* offsets, int32_t* r2s, int32_t* s2r, uint8_t* ad, uint8_t* as, float* ag,
                            void* ws, cudaStream_t st)
{
    const int64_t S = (int64_t)Tn * k;
    if (S > 0 && S <= kDispatchSmallS) {
        if (fmt == DS4G_MXFP4)
            return dtype == DS4G_BF16
                       ? launch_small<uint16_t, DS4G_MXFP4>(logits, (const uint16_t*)x, Tn, E, k, d, g_in, idx, w, xd, xs,
                                                            xg, offsets, r2s, s2r, ad, as, ag, st)
                       : launch_small<float, DS4G_MXFP4>(logits, (const float*)x, Tn, E, k, d, g_in, idx, w, xd, xs, xg,
                                                         offsets, r2s, s2r, ad, as, ag, st);
        return dtype == DS4G_BF16
                   ? launch_small<uint16_t, DS4G_NVFP4>(logits, (const uint16_t*)x, Tn, E, k, d, g_in, idx, w, xd, xs,
                                                        xg, offsets, r2s, s2r, ad, as, ag, st)
                   : launch_small<float, DS4G_NVFP4>(logits, (const float*)x, Tn, E, k, d, g_in, idx, w, xd, xs, xg,
                                                     offsets, r2s, s2r, ad, as, ag, st);
    }
    // route; NVFP4 tensor scale (amax, g) unless given; counts, scan, ranks;
    // then one pass that quantises and scatters
    cudaError_t e = launch_route_topk(logits, Tn, E, k, idx, w, st);
    if (e != cudaSuccess) return e;
    const size_t pw = (permute_workspace_bytes(Tn, k, E) + 15) / 16 * 16;
    const float* g = nullptr;
    if (fmt == DS4G_NVFP4) {
        if (g_in) {
            if (g_in != xg) e = cudaMemcpyAsync(xg, g_in, sizeof(float), cudaMemcpyDeviceToDevice, st);
        } else {
            unsigned int* amax = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(ws) + pw);
            e = cudaMemsetAsync(amax, 0, sizeof(unsigned int), st);
            if (e != cudaSuccess) return e;
            const int64_t n = (int64_t)Tn * d;
            const int64_t ga0 = ceil_div(n / 8, 256);
            const int ga = (int)(ga0 < (int64_t)kNumSMs * 16 ? ga0 : (int64_t)kNumSMs * 16);
            if (dtype == DS4G_BF16) k_amax<uint16_t><<<ga, 256, 0, st>>>((const uint16_t*)x, n, amax);
            else k_amax<float><<<ga, 256, 0, st>>>((const float*)x, n, amax);
            k_g_from_amax<<<1, 1, 0, st>>>(amax, xg);
            e = cudaGetLastError();
        }
        if (e != cudaSuccess) return e;
        g = xg;
    }
    int32_t* pws = reinterpret_cast<int32_t*>(ws);
    const int B = (int)ceil_div(S, kChunk);
    const size_t shm = (size_t)E * sizeof(int32_t);
    k_perm_hist<<<B, 256, shm, st>>>(idx, S, E, B, pws);
    k_perm_scan<<<1, 1024, 0, st>>>(pws, E * B, E, B, S, offsets);
    k_perm_rank<<<B, 32, shm, st>>>(idx, S, E, B, pws, r2s, s2r);
    const int64_t nb = (int64_t)Tn * (d / (fmt == DS4G_MXFP4 ? 32 : 16));
    const int64_t gq0 = ceil_div(nb, 256);
    const int gq = (int)(gq0 < (int64_t)kNumSMs * 16 ? gq0 : (int64_t)kNumSMs * 16);
#define DS4G_QS(TT, F) k_quant_scatter<TT, F><<<gq, 256, 0, st>>>((const TT*)x, Tn, d, k, g, s2r, xd, xs, ad, as, ag)
    if (fmt == DS4G_MXFP4) {
        if (dtype == DS4G_BF16) DS4G_QS(uint16_t, DS4G_MXFP4);
        else DS4G_QS(float, DS4G_MXFP4);
    } else {
        if (dtype == DS4G_BF16) DS4G_QS(uint16_t, DS4G_NVFP4);
        else DS4G_QS(float, DS4G_NVFP4);
    }
#undef DS4G_QS
    return cudaGetLastError();
}

}  // namespace ds4g
