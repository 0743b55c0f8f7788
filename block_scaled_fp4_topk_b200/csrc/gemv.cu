// gemv.cu -- decode-sized grouped FP4 GEMM (at most a few rows per expert).
//
// The work is bound by streaming the touched experts' packed weights from
// HBM ("[DeepSeek V4] Triton FP4 optimisation in practice", lesson 3: moving
// fewer bytes beats faster math), so the kernel is built around 128-bit
// coalesced weight loads: a lane owns one 32-element block (16 bytes + its
// scale) per step, a warp streams 512 contiguous bytes of a weight row.
//
// Decode: each E2M1 code becomes the int8 value 2*E2M1 through a 16-entry
// lookup done with `prmt` (the FP4 -> 16-entry-table equivalence of "ik_llama
// PR #454 ..." sec. 5).  `prmt`'s sign-replicate selector bit is the E2M1
// sign bit, so one lookup on the codes yields the positive terms and one on
// the sign-flipped codes yields the negative terms; two dp4a accumulators
// give the exact integer dot product of a block, which is then scaled by the
// two block scales (exact: powers of two for MX, 4-bit mantissas for NV) and
// accumulated in fp32.  The few activation rows are decoded to int8 once per
// CTA into shared memory.
//
// Grid: (column tiles, S).  blockIdx.y = permuted row r; only the CTA whose r
// starts an expert segment works, so each touched expert's weights are read
// once per column tile and empty experts cost nothing.
#include "common.cuh"
#include "kernels.cuh"

namespace ds4g {

template <int FMT>
struct BlockScale;

template <>
struct BlockScale<DS4G_MXFP4> {
    // activation side carries the 1/4 of the two doubled int8 operands
    static __device__ __forceinline__ float a(uint32_t b) { return exp2i((int)b - 129); }
    static __device__ __forceinline__ float w(uint32_t b) { return exp2i((int)b - 127); }
};

template <>
struct BlockScale<DS4G_NVFP4> {
    static __device__ __forceinline__ float a(uint32_t b) { return ue4m3_value(b) * 0.25f; }
    static __device__ __forceinline__ float w(uint32_t b) { return ue4m3_value(b); }
};

// int8 (2 * E2M1) of 8 codes in one word -> two words of 4 int8, in order
__device__ __forceinline__ void decode_word_signed(uint32_t x, uint32_t& lo, uint32_t& hi)
{
    // used only for the activation rows (once per CTA): magnitude lookup on
    // the codes with the sign bit cleared, then negate the bytes whose code
    // had the sign bit set
    uint32_t m = x & 0x77777777u;
    uint32_t mlo = prmt(kLutLo, kLutHi, m);
    uint32_t mhi = prmt(kLutLo, kLutHi, m >> 16);
    uint32_t r[2] = {mlo, mhi};
    uint32_t out[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t v = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int code = (x >> (4 * (4 * h + i))) & 0xF;
            int mag = (r[h] >> (8 * i)) & 0xFF;
            int val = (code & 8) ? -mag : mag;
            v |= ((uint32_t)val & 0xFFu) << (8 * i);
        }
        out[h] = v;
    }
    lo = out[0];
    hi = out[1];
}

// NW warps per CTA, NR weight rows per warp, activation rows handled MAXR at a
// time (rows beyond the segment are skipped at run time, CTA-uniformly).
// FC1 with the fused epilogue: a CTA owns 32 gate columns and the matching 32
// up rows (NW * NR == 64), each warp NR/2 gate + NR/2 up rows.
template <int FMT, int EPI, int MAXR, int NW, int NR>
__global__ void __launch_bounds__(NW * 32)
k_gemv(const GemmArgs p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    constexpr int BLK = (FMT == DS4G_MXFP4) ? 32 : 16;
    constexpr int NSB = 32 / BLK;                       // scales per 32-element chunk
    constexpr int NT = NW * 32;
    constexpr bool kSwiGLU = (EPI == DS4G_EPI_SWIGLU_REQUANT);
    const int64_t K = p.K;
    const int64_t nchunk = K / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- leader check: does permuted row r start an expert segment?
    const int64_t r = blockIdx.y;
    int lo = 0, hi = p.E - 1;                          // largest e with offsets[e] <= r
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (p.offsets[mid] <= r) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    if (p.offsets[e] != r || p.offsets[e + 1] <= r) return;
    const int64_t seg_end = p.offsets[e + 1];

    int8_t* a8 = reinterpret_cast<int8_t*>(smem);                       // [MAXR][K]
    float* asc = reinterpret_cast<float*>(smem + (size_t)MAXR * K);     // [MAXR][K/BLK]
    float* red = asc + (size_t)MAXR * (K / BLK);                        // [2][MAXR][32]

    const float gscale = (FMT == DS4G_NVFP4) ? __fmul_rn(p.a_g[0], p.w_g[e]) : 1.0f;   // per-expert weight scale
    const int I = p.N / 2;

    // this warp's weight rows
    int64_t wrow[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) {
        int n;
        if (kSwiGLU) {
            constexpr int H = NR / 2;
            n = (i < H) ? (blockIdx.x * 32 + warp * H + i) : (I + blockIdx.x * 32 + warp * H + (i - H));
        } else {
            n = blockIdx.x * (NW * NR) + warp * NR + i;
        }
        wrow[i] = (int64_t)e * p.N + n;
    }

    for (int64_t rg = r; rg < seg_end; rg += MAXR) {
        const int nr = (int)min((int64_t)MAXR, seg_end - rg);
        __syncthreads();
        // ---- activation rows -> int8 + float scales in shared memory
        for (int64_t i = threadIdx.x; i < (int64_t)nr * (K / 8); i += NT) {
            const int rr = (int)(i / (K / 8));
            const int64_t wd = i % (K / 8);
            uint32_t lo8, hi8;
            const uint32_t x = reinterpret_cast<const uint32_t*>(p.a_data + (rg + rr) * (K / 2))[wd];
            decode_word_signed(x, lo8, hi8);
            reinterpret_cast<uint2*>(a8)[i] = make_uint2(lo8, hi8);
        }
        for (int64_t i = threadIdx.x; i < (int64_t)nr * (K / BLK); i += NT) {
            const int rr = (int)(i / (K / BLK));
            asc[i] = BlockScale<FMT>::a(p.a_scales[(rg + rr) * (K / BLK) + i % (K / BLK)]);
        }
        __syncthreads();

        float acc[NR][MAXR];
#pragma unroll
        for (int i = 0; i < NR; ++i)
#pragma unroll
            for (int j = 0; j < MAXR; ++j) acc[i][j] = 0.f;

        uint4 wv[NR];
        uint32_t ws[NR];
        auto load = [&](int64_t c) {
#pragma unroll
            for (int i = 0; i < NR; ++i) {
                if (c < nchunk) {
                    wv[i] = __ldg(reinterpret_cast<const uint4*>(p.w_data + wrow[i] * (K / 2)) + c);
                    if (NSB == 1) ws[i] = __ldg(p.w_scales + wrow[i] * (K / BLK) + c);
                    else ws[i] = __ldg(reinterpret_cast<const uint16_t*>(p.w_scales + wrow[i] * (K / BLK)) + c);
                }
            }
        };

        int64_t c = lane;
        load(c);
        for (; c < nchunk; c += 32) {
            uint4 cv[NR];
            uint32_t cs[NR];
#pragma unroll
            for (int i = 0; i < NR; ++i) { cv[i] = wv[i]; cs[i] = ws[i]; }
            load(c + 32);                                  // prefetch the next step
#pragma unroll
            for (int i = 0; i < NR; ++i) {
                uint32_t pp[8], pn[8];
                const uint32_t xw[4] = {cv[i].x, cv[i].y, cv[i].z, cv[i].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t x = xw[q], xs = x ^ 0x88888888u;
                    pp[2 * q] = prmt(kLutLo, kLutHi, x);
                    pp[2 * q + 1] = prmt(kLutLo, kLutHi, x >> 16);
                    pn[2 * q] = prmt(kLutLo, kLutHi, xs);
                    pn[2 * q + 1] = prmt(kLutLo, kLutHi, xs >> 16);
                }
#pragma unroll
                for (int rr = 0; rr < MAXR; ++rr) {
                    if (rr < nr) {
                        const uint4* ap = reinterpret_cast<const uint4*>(a8 + (size_t)rr * K + c * 32);
                        const uint4 a0 = ap[0], a1 = ap[1];
                        const uint32_t av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                        if (FMT == DS4G_MXFP4) {
                            int dp = 0, dn = 0;
#pragma unroll
                            for (int m = 0; m < 8; ++m) {
                                dp = __dp4a((int)pp[m], (int)av[m], dp);
                                dn = __dp4a((int)pn[m], (int)av[m], dn);
                            }
                            const float sa = asc[(size_t)rr * (K / BLK) + c];
                            acc[i][rr] += ((float)(dp - dn) * sa) * BlockScale<FMT>::w(cs[i]);
                        } else {
                            int dp0 = 0, dn0 = 0, dp1 = 0, dn1 = 0;
#pragma unroll
                            for (int m = 0; m < 4; ++m) {
                                dp0 = __dp4a((int)pp[m], (int)av[m], dp0);
                                dn0 = __dp4a((int)pn[m], (int)av[m], dn0);
                                dp1 = __dp4a((int)pp[m + 4], (int)av[m + 4], dp1);
                                dn1 = __dp4a((int)pn[m + 4], (int)av[m + 4], dn1);
                            }
                            const float sa0 = asc[(size_t)rr * (K / BLK) + 2 * c];
                            const float sa1 = asc[(size_t)rr * (K / BLK) + 2 * c + 1];
                            acc[i][rr] += ((float)(dp0 - dn0) * sa0) * BlockScale<FMT>::w(cs[i] & 0xFF);
                            acc[i][rr] += ((float)(dp1 - dn1) * sa1) * BlockScale<FMT>::w(cs[i] >> 8);
                        }
                    }
                }
            }
        }

        // ---- warp reduction of every (weight row, activation row) pair
#pragma unroll
        for (int i = 0; i < NR; ++i)
#pragma unroll
            for (int rr = 0; rr < MAXR; ++rr) {
                if (rr < nr) {
                    float v = acc[i][rr];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                    acc[i][rr] = v * gscale;
                }
            }

        if (!kSwiGLU) {
#pragma unroll
            for (int rr = 0; rr < MAXR; ++rr) {
                if (rr == lane && rr < nr) {
#pragma unroll
                    for (int i = 0; i < NR; ++i) {
                        const int64_t n = blockIdx.x * (NW * NR) + warp * NR + i;
                        if (EPI == kEpiCombine) {
                            const int32_t s = p.r2s[rg + rr];
                            atomicAdd(p.out + (int64_t)(s / p.topk) * p.N + n, acc[i][rr] * p.route_w[s]);
                        } else {
                            p.out[(rg + rr) * p.N + n] = acc[i][rr];
                        }
                    }
                }
            }
        } else {
            // gate / up results of this CTA's 32 columns -> shared, then one
            // warp per activation row computes h and quantises its block(s)
            constexpr int H = NR / 2;
            if (lane == 0) {
#pragma unroll
                for (int rr = 0; rr < MAXR; ++rr)
#pragma unroll
                    for (int i = 0; i < H; ++i) {
                        red[(0 * MAXR + rr) * 32 + warp * H + i] = acc[i][rr];
                        red[(1 * MAXR + rr) * 32 + warp * H + i] = acc[i + H][rr];
                    }
            }
            __syncthreads();
            for (int rr = warp; rr < nr; rr += NW) {
                const float g = red[(0 * MAXR + rr) * 32 + lane];
                const float u = red[(1 * MAXR + rr) * 32 + lane];
                const float h = swiglu_f32(g, u);
                const int64_t row = rg + rr;
                const int col = blockIdx.x * 32 + lane;
                if (p.h_debug) p.h_debug[row * I + col] = h;
                uint32_t code;
                if (FMT == DS4G_MXFP4) {
                    float m = fabsf(h);
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                    const int X = mx_shared_exp(m);
                    code = e2m1_code(__fmul_rn(h, exp2i(-X)));
                    if (lane == 0) p.oq_scales[row * (I / 32) + blockIdx.x] = (uint8_t)(X + 127);
                } else {
                    float m = fabsf(h);
#pragma unroll
                    for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                    const float gh = *p.oq_g;
                    const uint32_t s = ue4m3_encode(__fdiv_rn(m, __fmul_rn(6.0f, gh)));
                    const float ds = ue4m3_value(s);
                    code = (ds == 0.0f) ? ((__float_as_uint(h) >> 28) & 8u)
                                        : e2m1_code(__fdiv_rn(h, __fmul_rn(ds, gh)));
                    if ((lane & 15) == 0) p.oq_scales[row * (I / 16) + blockIdx.x * 2 + (lane >> 4)] = (uint8_t)s;
                }
                const uint32_t hi_code = __shfl_down_sync(0xffffffffu, code, 1);
                if ((lane & 1) == 0)
                    p.oq_data[row * (I / 2) + blockIdx.x * 16 + (lane >> 1)] = (uint8_t)(code | (hi_code << 4));
            }
        }
    }
}

template <int FMT, int EPI, int MAXR, int NW, int NR>
static cudaError_t run(const GemmArgs& a, int gx, cudaStream_t st)
{
    constexpr int BLK = (FMT == DS4G_MXFP4) ? 32 : 16;
    const size_t shm = (size_t)MAXR * a.K + (size_t)MAXR * (a.K / BLK) * 4 + 2 * MAXR * 32 * 4;
    auto kern = k_gemv<FMT, EPI, MAXR, NW, NR>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)gx, (unsigned)a.S);
    kern<<<grid, NW * 32, shm, st>>>(a);
    return cudaGetLastError();
}

template <int FMT, int EPI, int MAXR>
static cudaError_t pick_shape(const GemmArgs& a, cudaStream_t st)
{
    constexpr int NRMAX = MAXR >= 4 ? 4 : 8;     // keeps the accumulators in registers
    if (EPI == DS4G_EPI_SWIGLU_REQUANT) return run<FMT, EPI, MAXR, 64 / NRMAX, NRMAX>(a, a.N / 2 / 32, st);
    // enough CTAs in flight: aim for >= 4 CTAs per SM over the touched experts
    const int64_t experts = a.S < a.E ? a.S : a.E;
    int rpw = NRMAX;
    while (rpw > 1 && (int64_t)(a.N / (8 * rpw)) * experts < 4 * kNumSMs) rpw >>= 1;
    switch (rpw) {
    case 8: return run<FMT, EPI, MAXR, 8, (NRMAX >= 8 ? 8 : 4)>(a, a.N / (8 * (NRMAX >= 8 ? 8 : 4)), st);
    case 4: return run<FMT, EPI, MAXR, 8, 4>(a, a.N / 32, st);
    case 2: return run<FMT, EPI, MAXR, 8, 2>(a, a.N / 16, st);
    default: return run<FMT, EPI, MAXR, 8, 1>(a, a.N / 8, st);
    }
}

template <int FMT, int EPI>
static cudaError_t pick_rows(const GemmArgs& a, cudaStream_t st)
{
    if (a.max_rows <= 1) return pick_shape<FMT, EPI, 1>(a, st);
    if (a.max_rows <= 2) return pick_shape<FMT, EPI, 2>(a, st);
    if (a.max_rows <= 4) return pick_shape<FMT, EPI, 4>(a, st);
    return pick_shape<FMT, EPI, 8>(a, st);
}

cudaError_t launch_gemv(const GemmArgs& a, cudaStream_t st)
{
    if (a.S == 0) return cudaSuccess;
    if (a.fmt == DS4G_MXFP4)
        return a.epilogue == DS4G_EPI_NONE ? pick_rows<DS4G_MXFP4, DS4G_EPI_NONE>(a, st)
             : a.epilogue == kEpiCombine   ? pick_rows<DS4G_MXFP4, kEpiCombine>(a, st)
                                           : pick_rows<DS4G_MXFP4, DS4G_EPI_SWIGLU_REQUANT>(a, st);
    return a.epilogue == DS4G_EPI_NONE ? pick_rows<DS4G_NVFP4, DS4G_EPI_NONE>(a, st)
         : a.epilogue == kEpiCombine   ? pick_rows<DS4G_NVFP4, kEpiCombine>(a, st)
                                       : pick_rows<DS4G_NVFP4, DS4G_EPI_SWIGLU_REQUANT>(a, st);
}

}  // namespace ds4g
