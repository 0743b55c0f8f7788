// permute.cu -- expert-contiguous permutation of the routed slots and the
// gather of the quantised rows ("[DeepSeek V4] Triton FP4 optimisation in
// practice", "Step 0": the grouped GEMM takes the rows of each expert as one
// contiguous segment).
//
// Slots s = t*k + j are split into chunks of kChunk.  Three small kernels:
//   hist     per-chunk expert histogram          -> ws[e * B + b]
//   scan     exclusive scan of ws in (e, b) order -> segment bases, offsets
//   rank     per chunk, one warp walks its slots in order; __match_any_sync
//            ranks equal experts inside each group of 32 and a shared
//            running count carries the rank across groups, so the order
//            inside an expert is ascending slot id (stable)
// and a gather that copies each permuted row's packed data and scales with
// 16-byte loads, one warp per row.
#include "common.cuh"
#include "kernels.cuh"

namespace ds4g {

constexpr int kChunk = 256;       // slots per rank warp (more warps in flight than 1024-slot chunks)

size_t permute_workspace_bytes(int T, int k, int E)
{
    int64_t S = (int64_t)T * k;
    int64_t B = ceil_div(S, kChunk);
    if (B < 1) B = 1;
    return (size_t)(E * B) * sizeof(int32_t);
}

__global__ void k_perm_hist(const int32_t* __restrict__ idx, int64_t S, int E, int B, int32_t* __restrict__ ws)
{
    extern __shared__ int32_t h[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    __syncthreads();
    const int64_t s0 = (int64_t)blockIdx.x * kChunk;
    const int64_t s1 = min(s0 + kChunk, S);
    for (int64_t s = s0 + threadIdx.x; s < s1; s += blockDim.x) atomicAdd(&h[idx[s]], 1);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) ws[(int64_t)e * B + blockIdx.x] = h[e];
}

// exclusive scan of n = E*B ints in place (one block of 1024 threads); also
// offsets[e] = scanned[e*B], offsets[E] = S.  Tiles of 4096 ints: each thread
// takes 4 adjacent ones (a warp reads 512 contiguous bytes), scans them, then
// warp and block scans of the thread totals and a carry across tiles.
__global__ void __launch_bounds__(1024) k_perm_scan(int32_t* __restrict__ ws, int n, int E, int B, int64_t S,
                                                    int32_t* __restrict__ offsets)
{
    __shared__ int32_t wsum[32];
    __shared__ int32_t carry_s;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) carry_s = 0;
    __syncthreads();
    for (int base = 0; base < n; base += 4 * 1024) {
        const int i0 = base + 4 * tid;
        int32_t v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = (i0 + j < n) ? ws[i0 + j] : 0;
        const int32_t tsum = v[0] + v[1] + v[2] + v[3];
        int32_t incl = tsum;                               // inclusive scan of thread totals in the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const int32_t x = wsum[lane];
            int32_t wi = x;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, wi, o);
                if (lane >= o) wi += y;
            }
            wsum[lane] = wi - x;                           // exclusive base of each warp
        }
        __syncthreads();
        const int32_t carry = carry_s;
        int32_t run = carry + wsum[warp] + incl - tsum;    // exclusive base of this thread
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (i0 + j < n) ws[i0 + j] = run;
            run += v[j];
        }
        __syncthreads();                                   // every thread has read carry_s and wsum
        if (tid == 1023) carry_s = run;                    // the tile's total, carried on
        __syncthreads();
    }
    for (int e = tid; e < E; e += blockDim.x) offsets[e] = ws[(int64_t)e * B];
    if (tid == 0) offsets[E] = (int32_t)S;
}

__global__ void k_perm_rank(const int32_t* __restrict__ idx, int64_t S, int E, int B,
                            const int32_t* __restrict__ base, int32_t* __restrict__ row_to_slot,
                            int32_t* __restrict__ slot_to_row)
{
    extern __shared__ int32_t cnt[];
    const int lane = threadIdx.x;
    for (int e = lane; e < E; e += 32) cnt[e] = 0;
    __syncwarp();
    const int64_t s0 = (int64_t)blockIdx.x * kChunk;
    const int64_t s1 = min(s0 + kChunk, S);
    for (int64_t g = s0; g < s1; g += 32) {
        const int64_t s = g + lane;
        const bool valid = s < s1;
        const int e = valid ? idx[s] : -1 - lane;     // invalid lanes never match a real expert
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        int32_t pos = 0;
        if (valid) pos = base[(int64_t)e * B + blockIdx.x] + cnt[e] + rank;
        __syncwarp();
        if (valid && rank == 0) cnt[e] += __popc(peers);
        __syncwarp();
        if (valid) {
            row_to_slot[pos] = (int32_t)s;
            slot_to_row[s] = pos;
        }
    }
}

// one warp per permuted row: copy data (rb bytes per row -- K/2 for FP4, K
// for MXFP8 -- in 16-byte pieces) and the ns scale bytes (even)
__global__ void k_perm_gather(const uint8_t* __restrict__ xd, const uint8_t* __restrict__ xs,
                              const float* __restrict__ xg, int64_t S, int k, int64_t rb, int64_t ns,
                              const int32_t* __restrict__ row_to_slot, uint8_t* __restrict__ ad,
                              uint8_t* __restrict__ as, float* __restrict__ ag)
{
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (ag && r == 0 && lane == 0) *ag = *xg;
    if (r >= S) return;
    const int64_t t = row_to_slot[r] / k;
    const int64_t nvec = rb / 16;
    const uint4* src = reinterpret_cast<const uint4*>(xd + t * rb);
    uint4* dst = reinterpret_cast<uint4*>(ad + r * rb);
    for (int64_t i = lane; i < nvec; i += 32) dst[i] = src[i];
    const uint16_t* ss = reinterpret_cast<const uint16_t*>(xs + t * ns);
    uint16_t* sd = reinterpret_cast<uint16_t*>(as + r * ns);
    for (int64_t i = lane; i < ns / 2; i += 32) sd[i] = ss[i];
}

// Small slot counts (decode): the whole permutation in one CTA -- counts,
// scan, stable ranks and the row gather -- so a decode step pays one launch.
constexpr int kSmallS = 512;

__global__ void __launch_bounds__(512)
k_perm_small(const int32_t* __restrict__ idx, int S, int E, int k, int64_t rb, int64_t ns,
             const uint8_t* __restrict__ xd, const uint8_t* __restrict__ xs, const float* __restrict__ xg,
             int32_t* __restrict__ offsets, int32_t* __restrict__ row_to_slot, int32_t* __restrict__ slot_to_row,
             uint8_t* __restrict__ ad, uint8_t* __restrict__ as, float* __restrict__ ag)
{
    extern __shared__ int32_t sh[];
    int32_t* cnt = sh;                 // [E]
    int32_t* off = sh + E;             // [E + 1]
    int32_t* r2s = off + E + 1;        // [S]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (ag && tid == 0) *ag = *xg;
    for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    for (int s = tid; s < S; s += blockDim.x) atomicAdd(&cnt[idx[s]], 1);
    __syncthreads();
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
                cnt[e] = 0;            // reused as the running rank of each expert
            }
        }
        if (lane == 31) {
            off[E] = incl;
            offsets[E] = incl;
        }
        __syncwarp();
        for (int g = 0; g < S; g += 32) {
            const int s = g + lane;
            const bool valid = s < S;
            const int e = valid ? idx[s] : -1 - lane;
            const unsigned peers = __match_any_sync(0xffffffffu, e);
            const int rank = __popc(peers & ((1u << lane) - 1u));
            int32_t pos = 0;
            if (valid) pos = off[e] + cnt[e] + rank;
            __syncwarp();
            if (valid && rank == 0) cnt[e] += __popc(peers);
            __syncwarp();
            if (valid) {
                r2s[pos] = s;
                row_to_slot[pos] = s;
                slot_to_row[s] = pos;
            }
        }
    }
    __syncthreads();
    // gather: one warp per permuted row
    const int64_t nvec = rb / 16;
    for (int r = warp; r < S; r += blockDim.x / 32) {
        const int64_t t = r2s[r] / k;
        const uint4* src = reinterpret_cast<const uint4*>(xd + t * rb);
        uint4* dst = reinterpret_cast<uint4*>(ad + (int64_t)r * rb);
        for (int64_t i = lane; i < nvec; i += 32) dst[i] = src[i];
        const uint16_t* ss = reinterpret_cast<const uint16_t*>(xs + t * ns);
        uint16_t* sd = reinterpret_cast<uint16_t*>(as + (int64_t)r * ns);
        for (int64_t i = lane; i < ns / 2; i += 32) sd[i] = ss[i];
    }
}

// segment ids: row r of [0, rows) lies in segment s when offsets[s] - offsets[0]
// <= r < offsets[s + 1] - offsets[0]; out[r] = s % modulo (binary search per row)
__global__ void k_segment_ids(const int32_t* __restrict__ offsets, int nseg, int modulo, int64_t rows,
                              int32_t* __restrict__ out)
{
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    const int64_t v = r + offsets[0];
    int lo = 0, hi = nseg - 1;          // largest s with offsets[s] <= v
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offsets[mid] <= v) lo = mid; else hi = mid - 1;
    }
    out[r] = lo % modulo;
}

cudaError_t launch_segment_ids(const int32_t* offsets, int nseg, int modulo, int64_t rows, int32_t* out,
                               cudaStream_t st)
{
    if (rows == 0) return cudaSuccess;
    k_segment_ids<<<(unsigned)ceil_div(rows, 256), 256, 0, st>>>(offsets, nseg, modulo, rows, out);
    return cudaGetLastError();
}

cudaError_t launch_permute(const int32_t* idx, int T, int k, int E, const uint8_t* xd, const uint8_t* xs,
                           const float* xg, int64_t K, int fmt, int32_t* offsets, int32_t* row_to_slot,
                           int32_t* slot_to_row, uint8_t* ad, uint8_t* as, float* ag, void* ws_,
                           cudaStream_t st)
{
    const int64_t S = (int64_t)T * k;
    int32_t* ws = reinterpret_cast<int32_t*>(ws_);
    const int B = (int)(S > 0 ? ceil_div(S, kChunk) : 1);
    const size_t shm = (size_t)E * sizeof(int32_t);
    if (S == 0) {
        cudaError_t e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), st);
        if (e != cudaSuccess) return e;
        if (fmt == DS4G_NVFP4 && ag) return cudaMemcpyAsync(ag, xg, sizeof(float), cudaMemcpyDeviceToDevice, st);
        return cudaSuccess;
    }
    const int64_t rb = (fmt == DS4G_MXFP8) ? K : K / 2;          // data bytes per row
    const int64_t ns = K / (fmt == DS4G_NVFP4 ? 16 : 32);          // scale bytes per row
    if (S <= kSmallS) {
        const size_t shs = (size_t)(2 * E + 1 + S) * sizeof(int32_t);
        k_perm_small<<<1, 512, shs, st>>>(idx, (int)S, E, k, rb, ns, xd, xs, xg, offsets, row_to_slot, slot_to_row,
                                          ad, as, fmt == DS4G_NVFP4 ? ag : nullptr);
        return cudaGetLastError();
    }
    k_perm_hist<<<B, 256, shm, st>>>(idx, S, E, B, ws);
    k_perm_scan<<<1, 1024, 0, st>>>(ws, E * B, E, B, S, offsets);
    k_perm_rank<<<B, 32, shm, st>>>(idx, S, E, B, ws, row_to_slot, slot_to_row);
    k_perm_gather<<<(unsigned)ceil_div(S, 8), 256, 0, st>>>(xd, xs, xg, S, k, rb, ns, row_to_slot, ad, as,
                                                          fmt == DS4G_NVFP4 ? ag : nullptr);
    return cudaGetLastError();
}

}  // namespace ds4g
