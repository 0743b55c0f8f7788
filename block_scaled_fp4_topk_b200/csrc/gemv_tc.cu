// gemv_tc.cu -- decode-sized grouped block-scaled FP4 GEMM on the tensor
// cores, operands swapped: the 128 weight rows of a tile are the MMA's M side
// and the (at most 16) activation rows of the expert are its N side.
//
// At decode sizes ("[DeepSeek V4] Triton FP4 optimisation in practice":
// moving fewer bytes beats faster math) the work is streaming the touched
// experts' packed weights from HBM once.  Doing the dot products on the tensor
// cores (tcgen05.mma kind::mxf4 / kind::mxf4nvf4, M128 N16 K64, the same
// block-scaled MMA as the prefill kernel) leaves the SMs nothing to do but
// keep TMA copies in flight, so the kernel runs at the rate weights arrive.
//
// Roles (one persistent CTA per SM, 288 threads):
//   warps 0, 8  TMA producers, alternate scale stages: weight tile (128 rows
//           x 256 K) and the expert's activation rows (16 rows x 256 K), 10
//           stages; row-major scale boxes of both (512 K per scale stage, 5
//           scale stages for MXFP4, 4 for NVFP4)
//   warps 1, 3  MMA issuers, alternate scale stages: scales -> TMEM
//           (tcgen05.cp), 4 MMAs per data stage, double-buffered 16-column
//           accumulators each (the epilogue adds the two); warp 3 also
//           allocates TMEM
//   warp 2  scale transposer (weights in place; activations into zeroed
//           128-line chunks of which lines 0..15 carry the 16 rows)
//   warps 4-7  epilogue: thread = weight row, 16 token columns; the plain
//           fp32 store is coalesced along the weight rows; FC1 exchanges the up
//           rows through shared memory and quantises h along 32-column blocks
// Items (expert, group of 16 activation rows, weight tile) come from the
// expert offsets on the device; empty experts have none.  Every mbarrier
// wait is bounded.  Launches use programmatic stream serialization: the
// set-up overlaps the previous kernel, and no input is read before
// griddepcontrol.wait (a chained FC2 reads its offsets first and waits only
// before its activation rows).  A launch releases the next kernel on the
// stream only after its own wait has returned.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.cuh"

namespace ds4g {

namespace dtc {

using namespace tc;   // PTX wrappers and the scale transposer of gemm_tc.cu

constexpr int BMW = 128;           // weight rows per tile (MMA M)
constexpr int BNT = 16;            // activation rows per tile (MMA N)
constexpr int BKB = 128;
constexpr int BK = 256;
constexpr int kThreads = 288;
constexpr int W_BYTES = BMW * BKB;   // 16 KB
constexpr int X_BYTES = BNT * BKB;   // 2 KB
constexpr int kTmemCols = 128;
constexpr int kColAcc = 0;         // [issuer][buffer] 16-column accumulators: 64 columns
constexpr int kColSF = 64;         // [issuer] 16 weight-scale then 16 activation-scale columns
constexpr int kMaxE = 512;        // experts whose offsets and item counts fit in shared memory

// SPLIT: 1 = one CTA per item; 2 = a CTA pair shares each item, each CTA
// taking half of its K range (few items: decode FC1 at T = 1)
template <int FMT, int SPLIT = 1>
struct Cfg {
    // ring depths: as many 18 KB data stages as shared memory holds next to
    // the scale stages (each scale stage covers two data stages); a split
    // NVFP4 kernel gives one stage to the partial-sum exchange rows
    static constexpr int STAGES = (SPLIT == 2 && FMT == DS4G_NVFP4) ? 9 : 10;
    static constexpr int SF_STAGES = (FMT == DS4G_MXFP4) ? 5 : 4;
    static constexpr int WPS = (FMT == DS4G_MXFP4) ? 2 : 4;    // 4-scale words per row per K stage
    static constexpr int SF_ROW = 2 * WPS * 4;                  // scale bytes per row per scale stage
    static constexpr int SFW_BYTES = BMW * SF_ROW;              // weights, transposed in place
    static constexpr int SFXR_BYTES = BNT * SF_ROW;             // activations, as loaded
    static constexpr int SFXC_BYTES = 2 * WPS * 512;            // activations, chunk order
    static constexpr int DATA_BYTES = STAGES * (W_BYTES + X_BYTES);
    static constexpr int SF_BYTES = SF_STAGES * (SFW_BYTES + SFXR_BYTES + SFXC_BYTES);
    static constexpr int EARR_BYTES = ((kMaxE + 1) * 4 + 15) / 16 * 16;   // one [E + 1] int32 array
    static constexpr int XRED_BYTES = (SPLIT == 2) ? BMW * BNT * 4 : 0;   // the follower's partial sums
    // data, scales, barriers, the SwiGLU exchange, item prefix and offsets,
    // partial-sum rows
    static constexpr size_t SMEM =
        1024 + (size_t)DATA_BYTES + SF_BYTES + 512 + 64 * 16 * 4 + 2 * EARR_BYTES + XRED_BYTES;
    static_assert((2 * STAGES + 3 * SF_STAGES + 6) * 8 + 16 <= 512, "barrier block");
    static_assert(SMEM <= 232448, "shared memory per CTA");
};

struct Item {
    int e;
    int wt;        // weight tile
    int64_t x0;    // first activation row
    int nr;        // activation rows in the group (<= 16)
};

__device__ __forceinline__ Item item_of(int64_t it, const int32_t* prefix, const int32_t* offsets, int E, int wtiles)
{
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= it) lo = mid; else hi = mid - 1;
    }
    Item r;
    r.e = lo;
    const int64_t local = it - prefix[lo];
    r.wt = (int)(local % wtiles);
    r.x0 = offsets[lo] + (local / wtiles) * BNT;
    r.nr = (int)min((int64_t)BNT, (int64_t)offsets[lo + 1] - r.x0);
    return r;
}

template <int EPI>
__device__ __forceinline__ void w_rows(const Item& itm, int N, int I, int64_t& y0, int64_t& y1)
{
    const int64_t wbase = (int64_t)itm.e * N;
    if (EPI == DS4G_EPI_SWIGLU_REQUANT) {
        y0 = wbase + (int64_t)itm.wt * 64;
        y1 = wbase + I + (int64_t)itm.wt * 64;
    } else {
        y0 = wbase + (int64_t)itm.wt * BMW;
        y1 = y0;
    }
}

// activation scales: 16 row-major rows of SF_ROW bytes -> zeroed 128-line
// chunks (one per word) whose line l < 16 holds word c of row l in its first
// 4 bytes (rows 32.. of the chunk do not exist at N = 16)
template <int WORDS>
__device__ __forceinline__ void sfx_transpose(const uint8_t* raw, uint8_t* chunks, int lane)
{
#pragma unroll
    for (int c = 0; c < WORDS; ++c) {
        uint32_t w0 = 0;
        if (lane < BNT) w0 = reinterpret_cast<const uint32_t*>(raw + lane * WORDS * 4)[c];
        *reinterpret_cast<uint4*>(chunks + c * 512 + lane * 16) = make_uint4(w0, 0u, 0u, 0u);
    }
    __syncwarp();
}

// the follower's partial sums into the leader's shared memory, counted on the
// leader's mbarrier
__device__ __forceinline__ void st_async_v4(uint32_t cluster_addr, float a, float b, float c, float d,
                                            uint32_t mbar_cluster)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];"
                 ::"r"(cluster_addr), "f"(a), "f"(b), "f"(c), "f"(d), "r"(mbar_cluster)
                 : "memory");
}

template <int FMT, int EPI, int SPLIT>
__global__ void __launch_bounds__(kThreads, 1)
k_gemv_tc(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
          const __grid_constant__ CUtensorMap map_sfw, const __grid_constant__ CUtensorMap map_sfx, const GemmArgs p)
{
    using C = Cfg<FMT, SPLIT>;
    constexpr int STAGES = C::STAGES;
    constexpr int SF_STAGES = C::SF_STAGES;
    constexpr bool kSwiGLU = (EPI == DS4G_EPI_SWIGLU_REQUANT);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sW = smem;
    uint8_t* sX = sW + STAGES * W_BYTES;
    uint8_t* sSFW = sX + STAGES * X_BYTES;                    // [SF_STAGES][SFW_BYTES]
    uint8_t* sSFXC = sSFW + SF_STAGES * C::SFW_BYTES;         // [SF_STAGES][SFXC_BYTES]
    uint8_t* sSFXR = sSFXC + SF_STAGES * C::SFXC_BYTES;       // [SF_STAGES][SFXR_BYTES]
    uint64_t* bars = reinterpret_cast<uint64_t*>(sSFXR + SF_STAGES * C::SFXR_BYTES);
    uint64_t* full = bars;
    uint64_t* empty = full + STAGES;
    uint64_t* sf_full = empty + STAGES;
    uint64_t* sf_ready = sf_full + SF_STAGES;
    uint64_t* sf_empty = sf_ready + SF_STAGES;
    uint64_t* tmem_full = sf_empty + SF_STAGES;
    uint64_t* tmem_empty = tmem_full + 2;
    uint64_t* red_full = tmem_empty + 2;                      // split: the leader's exchange rows landed
    uint64_t* red_empty = red_full + 1;                       // split: the follower may send the next item
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red_empty + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int32_t* total_items = reinterpret_cast<int32_t*>(tmem_slot + 2);
    float* xch = reinterpret_cast<float*>(smem + C::DATA_BYTES + C::SF_BYTES + 512);   // [64][16] up rows
    int32_t* prefix = reinterpret_cast<int32_t*>(xch + 64 * 16);
    int32_t* soff = prefix + C::EARR_BYTES / 4;      // the expert offsets, staged once
    float* xred = reinterpret_cast<float*>(soff + C::EARR_BYTES / 4);   // split: [128][16] partial sums

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;
    const int64_t K = p.K;
    const int nks = (int)ceil_div(K, BK);
    const int npairs = (nks + 1) / 2;
    const int I = p.N / 2;
    // a split pair: rank r takes scale stages [jb, jb + np_loc) of every item
    // (the leader the first half); both walk the items of their cluster
    const uint32_t rank = (SPLIT == 2) ? cluster_ctarank() : 0u;
    const int np_lo = (SPLIT == 2) ? (npairs + 1) / 2 : npairs;
    const int jb = (rank == 1) ? np_lo : 0;
    const int np_loc = (SPLIT == 2) ? (rank == 0 ? np_lo : npairs - np_lo) : npairs;
    const int nks_loc = min(nks, 2 * (jb + np_loc)) - 2 * jb;
    const int64_t t_first = (SPLIT == 2) ? (int64_t)cluster_id_x() : (int64_t)blockIdx.x;
    const int64_t t_step = (SPLIT == 2) ? (int64_t)nclusters_x() : (int64_t)gridDim.x;
    const int wtiles = kSwiGLU ? (I / 64) : (p.N / BMW);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int r = 0; r < SF_STAGES; ++r) {
            mbar_init(smem_u32(&sf_full[r]), 1);
            mbar_init(smem_u32(&sf_ready[r]), 1);
            mbar_init(smem_u32(&sf_empty[r]), 1);
        }
        for (int b2 = 0; b2 < 2; ++b2) {
            mbar_init(smem_u32(&tmem_full[b2]), 2);
            mbar_init(smem_u32(&tmem_empty[b2]), 128);
        }
        mbar_init(smem_u32(red_full), 1);      // the leader's expect-tx arrival + the follower's bytes
        mbar_init(smem_u32(red_empty), 4);     // one arrival per leader epilogue warp
        *abort_flag = 0;
        fence_barrier_init();
    }
    // Every launch may begin while the previous kernel on the stream ends
    // (programmatic serialization): the set-up above touches no input, and
    // this wait holds every read of one until that kernel has finished.
    // The next kernel on the stream is released only after this wait has
    // returned, so when any kernel of a chain starts, every kernel before
    // its immediate predecessor has completed.
    // A chained FC2 (p.chained) reads its offsets now (written before its
    // predecessor, FC1, started: complete by the rule above); its producers
    // wait only before its activation rows, its other threads once the
    // set-up below is done.
    if (!p.chained) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    }
    // the expert offsets -> shared memory in one parallel pass (a loop of
    // dependent global loads here cost about 2 us per launch); L2 loads, so
    // that a chained launch, which may start before its predecessor ends,
    // never reads a line its SM cached earlier
    for (int e = threadIdx.x; e <= E; e += kThreads) soff[e] = __ldcg(p.offsets + e);
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_w) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_x) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_sfw) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_sfx) : "memory");
    }
    if (warp == 3) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    __syncthreads();
    if (warp == 0) {
        // items per expert, exclusive scan by one warp
        const int per = (E + 31) / 32;
        int32_t sum = 0;
        for (int i = 0; i < per; ++i) {
            const int e = lane * per + i;
            if (e < E) sum += (int32_t)(ceil_div((int64_t)soff[e + 1] - soff[e], BNT) * wtiles);
        }
        int32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int32_t run = incl - sum;
        for (int i = 0; i < per; ++i) {
            const int e = lane * per + i;
            if (e < E) {
                prefix[e] = run;
                run += (int32_t)(ceil_div((int64_t)soff[e + 1] - soff[e], BNT) * wtiles);
            }
        }
        if (lane == 31) {
            prefix[E] = incl;
            int32_t tot = incl;
            if ((int64_t)soff[E] > p.S) {
                raise_error(kErrBadOffsets);
                tot = 0;
            }
            *total_items = tot;
        }
    }
    tc_fence_before();
    // a pair: the peer's barriers must be initialised before anything arrives on them
    if (SPLIT == 2) cluster_sync_all(); else __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int64_t nitems = *total_items;
    if (p.chained && !((warp == 0 || warp == 8) && lane == 0)) {
        // a chained launch: every thread but the two producers (which load
        // weights first) waits for the previous kernel here, before any role
        // reads an input it writes
        asm volatile("griddepcontrol.wait;" ::: "memory");
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    }

    // A thread that has issued asynchronous work (TMA copies, tensor-core
    // instructions) and then waits on a barrier, or branches on anything it
    // reads, first waits for that work to drain.  So producers and MMA
    // issuers come in pairs that take alternate scale stages (each with its
    // one or two data stages), and each waits for all the barriers of a scale
    // stage before issuing any of its work: one drain per scale stage, while
    // the other thread of the pair keeps the copy engine or the tensor pipe
    // busy.
    if (warp == 0 || warp == 8) {
        // ================= TMA producers =================
        if (lane == 0) {
            const int pi = (warp == 0) ? 0 : 1;
            uint32_t tcount = 0, it_next = 0, sit_next = 0;
            bool ok = true;
            // a chained launch may start while the previous kernel on the
            // stream (the producer of the activations) still runs: the first
            // SF_STAGES scale stages (whose ring slots are free at the start)
            // load their weights at once and their activation rows only after
            // griddepcontrol.wait; ndef counts this thread's deferred stages
            // (scale stages pi, pi + 2, ...)
            bool waited = (p.chained == 0);
            uint32_t ndef = 0;
            auto load_x = [&](uint32_t sit) {
                const uint32_t n = sit / (uint32_t)np_loc, jl = sit % (uint32_t)np_loc;
                const Item it = item_of(t_first + (int64_t)n * t_step, prefix, soff, E, wtiles);
                const int j = jb + (int)jl;
                const uint32_t ita = n * (uint32_t)nks_loc + 2 * jl;
                const int nd = min(2, nks - 2 * j);
                const int r = sit % SF_STAGES;
                tma_load_2d(smem_u32(sSFXR + r * C::SFXR_BYTES), &map_sfx, smem_u32(&sf_full[r]), j * C::SF_ROW,
                            (int)it.x0);
                for (int d = 0; d < nd; ++d) {
                    const int s = (ita + d) % STAGES;
                    tma_load_2d(smem_u32(sX + s * X_BYTES), &map_x, smem_u32(&full[s]), (2 * j + d) * BKB, (int)it.x0);
                }
            };
            auto release_deferred = [&]() {
                asm volatile("griddepcontrol.wait;" ::: "memory");
                asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
                for (uint32_t i = 0; i < ndef; ++i) load_x((uint32_t)pi + 2 * i);
                waited = true;
            };
            for (int64_t t = t_first; t < nitems && ok; t += t_step, ++tcount) {
                const Item itm = item_of(t, prefix, soff, E, wtiles);
                int64_t y0, y1;
                w_rows<EPI>(itm, p.N, I, y0, y1);
                const uint32_t it0 = tcount * (uint32_t)nks_loc, sit0 = tcount * (uint32_t)np_loc;
                for (int jl = pi ^ (int)(sit0 & 1); jl < np_loc; jl += 2) {
                    const int j = jb + jl;                        // scale stage within the item's K
                    const uint32_t sit = sit0 + jl, ita = it0 + 2 * jl;
                    const int nd = min(2, nks - 2 * j);
                    const int r = sit % SF_STAGES;
                    // deferred stages never wait for a slot; the first other
                    // stage releases them before it waits (its slot frees
                    // only once a deferred stage has been consumed)
                    const bool defer = !waited && sit < (uint32_t)SF_STAGES;
                    if (!waited && !defer) release_deferred();
                    if (!mbar_wait(smem_u32(&sf_empty[r]), ((sit / SF_STAGES) & 1) ^ 1, abort_flag)) { ok = false; break; }
                    for (int d = 0; d < nd && ok; ++d)
                        ok = mbar_wait(smem_u32(&empty[(ita + d) % STAGES]), (((ita + d) / STAGES) & 1) ^ 1, abort_flag);
                    if (!ok) break;
                    const uint32_t sfb = smem_u32(&sf_full[r]);
                    mbar_arrive_tx(sfb, C::SFW_BYTES + C::SFXR_BYTES);
                    const int x = j * C::SF_ROW;
                    tma_load_2d(smem_u32(sSFW + r * C::SFW_BYTES), &map_sfw, sfb, x, (int)y0);
                    if (kSwiGLU) tma_load_2d(smem_u32(sSFW + r * C::SFW_BYTES + C::SFW_BYTES / 2), &map_sfw, sfb, x, (int)y1);
                    if (!defer) tma_load_2d(smem_u32(sSFXR + r * C::SFXR_BYTES), &map_sfx, sfb, x, (int)itm.x0);
                    for (int d = 0; d < nd; ++d) {
                        const int s = (ita + d) % STAGES;
                        const int ks = 2 * j + d;
                        const uint32_t fb = smem_u32(&full[s]);
                        mbar_arrive_tx(fb, W_BYTES + X_BYTES);
                        tma_load_2d(smem_u32(sW + s * W_BYTES), &map_w, fb, ks * BKB, (int)y0);
                        if (kSwiGLU) tma_load_2d(smem_u32(sW + s * W_BYTES + W_BYTES / 2), &map_w, fb, ks * BKB, (int)y1);
                        if (!defer) tma_load_2d(smem_u32(sX + s * X_BYTES), &map_x, fb, ks * BKB, (int)itm.x0);
                    }
                    if (defer) ++ndef;
                    it_next = ita + nd;
                    sit_next = sit + 1;
                }
            }
            // every armed stage gets its activation rows, also on an early exit
            if (!waited) release_deferred();
            if (!ok) {
                // let this thread's copies in flight land before the CTA goes
                // away (stop at the first wait that gives up)
                volatile int never = 0;
                bool go = true;
                for (uint32_t j = (it_next > STAGES + 2 ? it_next - STAGES - 2 : 0); j < it_next && go; ++j) {
                    const uint32_t owner = ((j / nks_loc) * np_loc + (j % nks_loc) / 2) & 1;
                    if ((int)owner == pi) go = mbar_wait(smem_u32(&full[j % STAGES]), (j / STAGES) & 1, &never);
                }
                for (uint32_t j = (sit_next > SF_STAGES + 1 ? sit_next - SF_STAGES - 1 : 0); j < sit_next && go; ++j)
                    if ((int)(j & 1) == pi) go = mbar_wait(smem_u32(&sf_full[j % SF_STAGES]), (j / SF_STAGES) & 1, &never);
            }
        }
        __syncwarp();
    } else if (warp == 1 || warp == 3) {
        // ================= MMA issuers =================
        // each with its own accumulators and scale columns; the epilogue adds
        // the two partial sums
        if (lane == 0) {
            const int pi = (warp == 1) ? 0 : 1;
            const uint32_t ibase = (1u << 7) | (1u << 10) | ((uint32_t)(BNT >> 3) << 17) |
                                   ((FMT == DS4G_MXFP4 ? 1u : 0u) << 23) | ((uint32_t)(BMW >> 4) << 24);
            const uint32_t col_sfw = tmem + kColSF + pi * 32, col_sfx = col_sfw + 16;
            uint32_t tcount = 0;
            bool ok = true;
            for (int64_t t = t_first; t < nitems && ok; t += t_step, ++tcount) {
                const int buf = tcount & 1;
                if (!mbar_wait(smem_u32(&tmem_empty[buf]), ((tcount >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t acc = tmem + kColAcc + pi * 32 + buf * BNT;
                const uint32_t it0 = tcount * (uint32_t)nks_loc, sit0 = tcount * (uint32_t)np_loc;
                bool first = true;
                for (int jl = pi ^ (int)(sit0 & 1); jl < np_loc; jl += 2) {
                    const int j = jb + jl;                        // scale stage within the item's K
                    const uint32_t sit = sit0 + jl, ita = it0 + 2 * jl;
                    const int nd = min(2, nks - 2 * j);
                    const int r = sit % SF_STAGES;
                    if (!mbar_wait(smem_u32(&sf_ready[r]), (sit / SF_STAGES) & 1, abort_flag)) { ok = false; break; }
                    for (int d = 0; d < nd && ok; ++d)
                        ok = mbar_wait(smem_u32(&full[(ita + d) % STAGES]), ((ita + d) / STAGES) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t sfw_s = smem_u32(sSFW + r * C::SFW_BYTES);
                    const uint32_t sfx_s = smem_u32(sSFXC + r * C::SFXC_BYTES);
                    for (int d = 0; d < nd; ++d) {
                        const int s = (ita + d) % STAGES;
                        const int ks = 2 * j + d;
                        const int w0 = d * C::WPS;
#pragma unroll
                        for (int c = 0; c < C::WPS; ++c) {
                            utccp(col_sfw + 4 * c, desc_sf(sfw_s + (w0 + c) * 512));
                            utccp(col_sfx + 4 * c, desc_sf(sfx_s + (w0 + c) * 512));
                        }
                        const int64_t krem = K - (int64_t)ks * BK;
                        const int nmma = krem >= BK ? 4 : (int)(krem / 64);
                        const uint32_t w_s = smem_u32(sW + s * W_BYTES);
                        const uint32_t x_s = smem_u32(sX + s * X_BYTES);
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) {
                            if (jj < nmma) {
                                const int c = (FMT == DS4G_MXFP4) ? (jj >> 1) : jj;
                                const uint32_t sfid = (FMT == DS4G_MXFP4) ? (uint32_t)((jj & 1) * 2) : 0u;
                                const uint32_t idesc = ibase | (sfid << 4) | (sfid << 29);
                                mma<FMT>(acc, desc_sw128(w_s + 32 * jj), desc_sw128(x_s + 32 * jj), idesc,
                                         (!first || jj > 0) ? 1u : 0u, col_sfw + 4 * c, col_sfx + 4 * c);
                            }
                        }
                        first = false;
                        tc_commit(smem_u32(&empty[s]));
                    }
                    tc_commit(smem_u32(&sf_empty[r]));
                }
                if (!ok) break;
                tc_commit(smem_u32(&tmem_full[buf]));             // also when this issuer had no stage
            }
        }
        __syncwarp();
    } else if (warp == 2) {
        // ================= scale transposer =================
        uint32_t sit = 0;
        for (int64_t t = t_first; t < nitems; t += t_step) {
            bool ok = true;
            for (int pr = 0; pr < np_loc; ++pr, ++sit) {
                const int r = sit % SF_STAGES;
                bool w_ok = true;
                if (lane == 0) w_ok = mbar_wait(smem_u32(&sf_full[r]), (sit / SF_STAGES) & 1, abort_flag);
                if (!__shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0)) { ok = false; break; }
                sf_transpose<2 * C::WPS, 1>(sSFW + r * C::SFW_BYTES, lane);
                sfx_transpose<2 * C::WPS>(sSFXR + r * C::SFXR_BYTES, sSFXC + r * C::SFXC_BYTES, lane);
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&sf_ready[r]));
            }
            if (!ok) break;
        }
    } else if (warp >= 4) {
        // ================= epilogue =================
        const int q = warp & 3;                  // weight rows 32q .. 32q + 31 of the tile
        uint32_t tcount = 0;
        const float gh = (FMT == DS4G_NVFP4 && kSwiGLU) ? *p.oq_g : 1.0f;
        for (int64_t t = t_first; t < nitems; t += t_step, ++tcount) {
            const int buf = tcount & 1;
            const bool got = mbar_wait(smem_u32(&tmem_full[buf]), (tcount >> 1) & 1, abort_flag);
            // a pair's teardown is a warp-aligned cluster barrier: the whole
            // warp leaves the loop together
            if (SPLIT == 2 ? !__all_sync(0xffffffffu, got) : !got) break;
            tc_fence_after();
            const Item itm = item_of(t, prefix, soff, E, wtiles);
            const float gscale = (FMT == DS4G_NVFP4) ? __fmul_rn(p.a_g[0], p.w_g[itm.e]) : 1.0f;
            // issuer i holds the sum over the scale stages of parity i
            const uint32_t sit0 = tcount * (uint32_t)np_loc;
            const uint32_t lanes = (uint32_t)(32 * q) << 16;
            float v[16];
            if (np_loc >= 2) {
                float v1[16];
                tmem_ld16(tmem + kColAcc + buf * BNT + lanes, v);
                tmem_ld16(tmem + kColAcc + 32 + buf * BNT + lanes, v1);
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] += v1[i];
            } else {
                tmem_ld16(tmem + kColAcc + (sit0 & 1) * 32 + buf * BNT + lanes, v);
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&tmem_empty[buf]));          // accumulator drained into registers
            if (SPLIT == 2) {
                // the follower sends its K half's sums for this item to the
                // leader, which adds them and runs the epilogue
                const int i = 32 * q + lane;                  // weight row of the tile
                if (rank == 1) {
                    const bool free_ = mbar_wait(smem_u32(red_empty), (tcount & 1) ^ 1, abort_flag);
                    if (!__all_sync(0xffffffffu, free_)) break;
                    const uint32_t dst = mapa_shared(smem_u32(xred + i * BNT), 0);
                    const uint32_t mb = mapa_shared(smem_u32(red_full), 0);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        st_async_v4(dst + 16u * c, v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3], mb);
                    continue;
                }
                if (threadIdx.x == 128) mbar_arrive_tx(smem_u32(red_full), BMW * BNT * 4);
                const bool landed = mbar_wait(smem_u32(red_full), tcount & 1, abort_flag);
                if (!__all_sync(0xffffffffu, landed)) break;
                const float4* src = reinterpret_cast<const float4*>(xred + i * BNT);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float4 u4 = src[c];
                    v[4 * c] += u4.x;
                    v[4 * c + 1] += u4.y;
                    v[4 * c + 2] += u4.z;
                    v[4 * c + 3] += u4.w;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(red_empty), 1));
            }
            if (!kSwiGLU) {
                const int64_t n = (int64_t)itm.wt * BMW + 32 * q + lane;
#pragma unroll
                for (int tt = 0; tt < BNT; ++tt) {
                    if (tt < itm.nr) {
                        if (EPI == kEpiCombine) {
                            // add w * row into its token's output (coalesced along n)
                            const int32_t s = p.r2s[itm.x0 + tt];
                            atomicAdd(p.out + (int64_t)(s / p.topk) * p.N + n, v[tt] * gscale * p.route_w[s]);
                        } else {
                            p.out[(itm.x0 + tt) * p.N + n] = v[tt] * gscale;
                        }
                    }
                }
            } else {
                // up rows (warps with q >= 2) -> shared; gate rows compute h
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (q >= 2) {
#pragma unroll
                    for (int tt = 0; tt < BNT; ++tt) xch[((q - 2) * 32 + lane) * BNT + tt] = v[tt];
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (q < 2) {
                    const int col = itm.wt * 64 + 32 * q + lane;    // h column (gate row within I)
#pragma unroll 1
                    for (int tt = 0; tt < itm.nr; ++tt) {
                        const float h = swiglu_f32(__fmul_rn(v[tt], gscale),
                                                   __fmul_rn(xch[(q * 32 + lane) * BNT + tt], gscale));
                        const int64_t row = itm.x0 + tt;
                        if (p.h_debug) p.h_debug[row * I + col] = h;
                        uint32_t code;
                        if (FMT == DS4G_MXFP4) {
                            float m = fabsf(h);
#pragma unroll
                            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                            const int X = mx_shared_exp(m);
                            code = e2m1_code(__fmul_rn(h, exp2i(-X)));
                            if (lane == 0) p.oq_scales[row * (I / 32) + col / 32] = (uint8_t)(X + 127);
                        } else {
                            float m = fabsf(h);
#pragma unroll
                            for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                            const uint32_t s = ue4m3_encode(__fdiv_rn(m, __fmul_rn(6.0f, gh)));
                            const float ds = ue4m3_value(s);
                            code = (ds == 0.0f) ? ((__float_as_uint(h) >> 28) & 8u)
                                                : e2m1_code(__fmul_rn(h, __frcp_rn(__fmul_rn(ds, gh))));
                            if ((lane & 15) == 0) p.oq_scales[row * (I / 16) + col / 16] = (uint8_t)s;
                        }
                        const uint32_t hi_code = __shfl_down_sync(0xffffffffu, code, 1);
                        if ((lane & 1) == 0) p.oq_data[row * (I / 2) + col / 2] = (uint8_t)(code | (hi_code << 4));
                    }
                }
            }
        }
    }

    tc_fence_before();
    // a pair: neither CTA leaves while the other may still reach its shared memory
    if (SPLIT == 2) cluster_sync_all(); else __syncthreads();
    tc_fence_after();
    if (warp == 3) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

}  // namespace dtc

template <int FMT, int EPI, int SPLIT = 1>
static cudaError_t run_dtc(const GemmArgs& a, cudaStream_t st)
{
    using C = dtc::Cfg<FMT, SPLIT>;
    const int blk = (FMT == DS4G_MXFP4) ? 32 : 16;
    const uint32_t wbox = (EPI == DS4G_EPI_SWIGLU_REQUANT) ? 64 : 128;
    CUtensorMap mw, mx, msw, msx;
    if (!make_map(&mw, a.w_data, (int64_t)a.E * a.N, a.K / 2, 128, wbox, true) ||
        !make_map(&mx, a.a_data, a.S, a.K / 2, 128, dtc::BNT, true) ||
        !make_map(&msw, a.w_scales, (int64_t)a.E * a.N, a.K / blk, C::SF_ROW, wbox, false) ||
        !make_map(&msx, a.a_scales, a.S, a.K / blk, C::SF_ROW, dtc::BNT, false))
        return cudaErrorInvalidValue;
    auto kern = dtc::k_gemv_tc<FMT, EPI, SPLIT>;
    const size_t shm = C::SMEM;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = kNumSMs;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (SPLIT == 1) {
        // may start while the previous kernel on the stream runs (the kernel
        // waits for it before reading any input; a chained FC2 before its
        // activation rows)
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.gridDim = dim3((unsigned)sms);
        cfg.blockDim = dim3(dtc::kThreads);
        cfg.dynamicSmemBytes = shm;
        cfg.stream = st;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kern, mw, mx, msw, msx, a);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    // CTA pairs: clusters of two, as many as can be resident at once; may
    // start while the previous kernel runs, as above
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)(sms & ~1));
    cfg.blockDim = dim3(dtc::kThreads);
    cfg.dynamicSmemBytes = shm;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;                          // the occupancy query sees the cluster shape only
    int nclusters = 0;
    e = cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg);
    if (e != cudaSuccess) return e;
    if (nclusters < 1) return cudaErrorInvalidConfiguration;
    cfg.gridDim = dim3((unsigned)(2 * (nclusters < sms / 2 ? nclusters : sms / 2)));
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, kern, mw, mx, msw, msx, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// FC1 with few items (at most about two per SM: decode T = 1) splits each
// item's K range over a CTA pair, so that no SM streams two whole items while
// others idle.  Chosen from the shape alone.
static bool use_split(const GemmArgs& a)
{
    const int64_t K = a.K;
    const int npairs = (int)((ceil_div(K, 256) + 1) / 2);
    if (a.epilogue != DS4G_EPI_SWIGLU_REQUANT || npairs < 2) return false;
    const int64_t wtiles = (a.N / 2) / 64;
    const int64_t experts = a.E < a.S ? a.E : a.S;       // experts that can hold rows
    return experts * wtiles <= 2 * kNumSMs;
}

bool gemv_tc_supports(int fmt, int64_t K, int N, int epilogue, int E)
{
    if (E < 1 || E > dtc::kMaxE || !gemm_tc_supports(fmt, K)) return false;
    return epilogue != DS4G_EPI_SWIGLU_REQUANT ? (N % 128 == 0) : (N % 2 == 0 && (N / 2) % 64 == 0);
}

cudaError_t launch_gemv_tc(const GemmArgs& a, cudaStream_t st)
{
    if (a.S == 0) return cudaSuccess;
    if (!gemv_tc_supports(a.fmt, a.K, a.N, a.epilogue, a.E)) return cudaErrorInvalidValue;
    const bool split = use_split(a);
    if (a.fmt == DS4G_MXFP4)
        return a.epilogue == DS4G_EPI_NONE ? run_dtc<DS4G_MXFP4, DS4G_EPI_NONE>(a, st)
             : a.epilogue == kEpiCombine   ? run_dtc<DS4G_MXFP4, kEpiCombine>(a, st)
             : split                       ? run_dtc<DS4G_MXFP4, DS4G_EPI_SWIGLU_REQUANT, 2>(a, st)
                                           : run_dtc<DS4G_MXFP4, DS4G_EPI_SWIGLU_REQUANT>(a, st);
    return a.epilogue == DS4G_EPI_NONE ? run_dtc<DS4G_NVFP4, DS4G_EPI_NONE>(a, st)
         : a.epilogue == kEpiCombine   ? run_dtc<DS4G_NVFP4, kEpiCombine>(a, st)
         : split                       ? run_dtc<DS4G_NVFP4, DS4G_EPI_SWIGLU_REQUANT, 2>(a, st)
                                       : run_dtc<DS4G_NVFP4, DS4G_EPI_SWIGLU_REQUANT>(a, st);
}

}  // namespace ds4g
