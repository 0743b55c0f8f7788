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
//           stages; row-major scale boxes of both (512 K per scale stage, 6
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
    // an even count: scale slot r belongs to the pair that takes the scale
    // stages of parity r & 1 (see the kernel)
    static constexpr int SF_STAGES = (FMT == DS4G_MXFP4) ? 6 : 4;
    static constexpr int WPS = (FMT == DS4G_MXFP4) ? 2 : 4;    // 4-scale words per row per K stage
    static constexpr int SF_ROW = 2 * WPS * 4;                  // scale bytes per row per scale stage
    static constexpr int SFW_BYTES = BMW * SF_ROW;              // weights, transposed in place
    static constexpr int SFXR_BYTES = BNT * SF_ROW;             // activations, as loaded
    static constexpr int SFXC_BYTES = 2 * WPS * 512;            // activations, chunk order
    static constexpr int DATA_BYTES = STAGES * (W_BYTES + X_BYTES);
    static constexpr int SF_BYTES = SF_STAGES * (SFW_BYTES + SFXR_BYTES + SFXC_BYTES);
    static constexpr int EARR_BYTES = ((kMaxE + 1) * 4 + 15) / 16 * 16;   // one [E + 1] int32 array
    static constexpr int XRED_BYTES = (SPLIT == 2) ? BMW * BNT * 4 : 0;   // the follower's partial sums
    // data, scales, barriers, the SwiGLU exchange, the item prefixes (one
    // per GEMM) and the offsets, partial-sum rows
    static constexpr size_t SMEM =
        1024 + (size_t)DATA_BYTES + SF_BYTES + 512 + 64 * 16 * 4 + 3 * EARR_BYTES + XRED_BYTES;
    static_assert((2 * STAGES + 3 * SF_STAGES + 8) * 8 + 32 <= 512, "barrier block");
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

// the four tensor maps of one GEMM: weights, activation rows, their scales
struct Maps {
    CUtensorMap w, x, sfw, sfx;
};

// one GEMM's tiling as this CTA sees it
struct Geo {
    int64_t K;
    int N, I, nks, np_loc, jb_rank, wtiles;
    bool sw;      // SwiGLU pairs of 64 gate + 64 up weight rows per tile
};

// counter published by another CTA: bounded wait until *addr >= target (acquire)
__device__ __forceinline__ bool wait_count(const int32_t* addr, int32_t target, volatile int* abort_flag)
{
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        int32_t v;
        asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(addr) : "memory");
        if (v >= target) return true;
        if (it == 0) {
            t0 = globaltimer();
        } else if ((it & 15u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > kWaitNs) {
                *abort_flag = 1;
                raise_error(kErrWaitTimeout);
                return false;
            }
        }
        __nanosleep(32);
    }
}

// EPI: DS4G_EPI_NONE, DS4G_EPI_SWIGLU_REQUANT or kEpiCombine (one GEMM: args
// p, maps m0), or kEpiFfn: the decode FFN in one launch, FC1 with SwiGLU +
// requantisation (p, m0) and then FC2 with the weighted combine (p2, m1).
// In the FFN every CTA (pair) takes its FC1 items, then its FC2 items in
// reverse unit order (units with one FC1 item more take fewer FC2 items).
// An FC1 item publishes its h columns on ctr[e] (release) once they are
// stored; an FC2 item of expert e loads h only after ctr[e] has counted all
// of e's FC1 items (acquire, then a proxy fence for the TMA loads).  The last
// CTA to finish (ctr[E] counts finished CTAs) sets ctr[0..E] back to zero.
template <int FMT, int EPI, int SPLIT>
__global__ void __launch_bounds__(kThreads, 1)
k_gemv_tc(const __grid_constant__ Maps m0, const __grid_constant__ Maps m1, const GemmArgs p, const GemmArgs p2,
          int32_t* __restrict__ ctr)
{
    using C = Cfg<FMT, SPLIT>;
    constexpr int STAGES = C::STAGES;
    constexpr int SF_STAGES = C::SF_STAGES;
    constexpr bool kFfn = (EPI == kEpiFfn);
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
    uint64_t* drain = red_empty + 1;                          // [2] each issuer's tensor-core work finished
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int32_t* total_items = reinterpret_cast<int32_t*>(tmem_slot + 2);   // [2]: items of each GEMM
    volatile int* last_cta = reinterpret_cast<volatile int*>(tmem_slot + 4);
    float* xch = reinterpret_cast<float*>(smem + C::DATA_BYTES + C::SF_BYTES + 512);   // [64][16] up rows
    int32_t* prefix = reinterpret_cast<int32_t*>(xch + 64 * 16);
    int32_t* prefix2 = prefix + C::EARR_BYTES / 4;   // the FFN's FC2 items per expert
    int32_t* soff = prefix2 + C::EARR_BYTES / 4;     // the expert offsets, staged once
    float* xred = reinterpret_cast<float*>(soff + C::EARR_BYTES / 4);   // split: [128][16] partial sums

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;
    // a split pair: rank r takes scale stages [jb, jb + np_loc) of every item
    // (the leader the first half); both walk the items of their cluster.
    // Split K (plain epilogue, few items): every item comes ksplit times,
    // part q taking scale stages [q np_loc, (q + 1) np_loc) and adding its
    // partial sums into the zeroed output (the host splits only a K of whole
    // scale stages into equal parts)
    const int ksplit = (SPLIT == 1 && EPI == DS4G_EPI_NONE && p.ksplit > 1 && !p.chained) ? p.ksplit : 1;
    const uint32_t rank = (SPLIT == 2) ? cluster_ctarank() : 0u;
    auto geo_of = [&](const GemmArgs& a, bool sw, int ks) {
        Geo g;
        g.K = a.K;
        g.N = a.N;
        g.I = a.N / 2;
        g.nks = (int)ceil_div(a.K, BK);
        const int npairs = (g.nks + 1) / 2;
        const int np_lo = (SPLIT == 2) ? (npairs + 1) / 2 : npairs / ks;
        g.jb_rank = (rank == 1) ? np_lo : 0;
        g.np_loc = (SPLIT == 2) ? (rank == 0 ? np_lo : npairs - np_lo) : np_lo;
        g.wtiles = sw ? (g.I / 64) : (a.N / BMW);
        g.sw = sw;
        return g;
    };
    const Geo G0 = geo_of(p, EPI == DS4G_EPI_SWIGLU_REQUANT || kFfn, ksplit);
    const Geo G1 = kFfn ? geo_of(p2, false, 1) : G0;
    // first scale stage of phase-0 item t's K range
    auto jb_of = [&](int64_t t) { return ksplit > 1 ? (int)(t % ksplit) * G0.np_loc : G0.jb_rank; };
    const int64_t t_first = (SPLIT == 2) ? (int64_t)cluster_id_x() : (int64_t)blockIdx.x;
    const int64_t t_step = (SPLIT == 2) ? (int64_t)nclusters_x() : (int64_t)gridDim.x;

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
        mbar_init(smem_u32(&drain[0]), 1);
        mbar_init(smem_u32(&drain[1]), 1);
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
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&m0.w) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&m0.x) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&m0.sfw) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&m0.sfx) : "memory");
        if (kFfn) {
            asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&m1.w) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&m1.x) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&m1.sfw) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&m1.sfx) : "memory");
        }
    }
    if (warp == 3) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    __syncthreads();
    if (warp == 0 || (kFfn && warp == 1)) {
        // items per expert, exclusive scan by one warp (warp 1: the FFN's FC2)
        const int wt = (warp == 0) ? G0.wtiles : G1.wtiles;
        int32_t* pre = (warp == 0) ? prefix : prefix2;
        const int per = (E + 31) / 32;
        int32_t sum = 0;
        for (int i = 0; i < per; ++i) {
            const int e = lane * per + i;
            if (e < E) sum += (int32_t)(ceil_div((int64_t)soff[e + 1] - soff[e], BNT) * wt);
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
                pre[e] = run;
                run += (int32_t)(ceil_div((int64_t)soff[e + 1] - soff[e], BNT) * wt);
            }
        }
        if (lane == 31) {
            pre[E] = incl;
            int32_t tot = incl;
            if ((int64_t)soff[E] > p.S) {
                if (warp == 0) raise_error(kErrBadOffsets);
                tot = 0;
            }
            total_items[warp] = tot;
        }
    }
    tc_fence_before();
    // a pair: the peer's barriers must be initialised before anything arrives on them
    if (SPLIT == 2) cluster_sync_all(); else __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int64_t nitems0 = (int64_t)total_items[0] * ksplit;
    const int64_t nitems1 = kFfn ? (int64_t)total_items[1] : 0;
    // this unit's phase-0 items: t_first, t_first + t_step, ...
    const int64_t n0 = nitems0 > t_first ? (nitems0 - t_first + t_step - 1) / t_step : 0;
    // item n of this unit (its phase, its index in that phase); false past the last
    auto item_at = [&](int64_t n, int& ph, int64_t& t) {
        if (n < n0) {
            ph = 0;
            t = t_first + n * t_step;
            return true;
        }
        if (!kFfn) return false;
        ph = 1;
        t = (t_step - 1 - t_first) + (n - n0) * t_step;
        return t < nitems1;
    };
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
    //
    // Scale stage sit (counted over this CTA's items) uses scale slot
    // sit % SF_STAGES and data stages 2 sit and 2 sit + 1 of a ring of
    // STAGES, so that up to min(SF_STAGES, STAGES / 2) scale stages are in
    // flight in the order they are needed (a scale stage with one data
    // stage, at the end of an odd K stage count, still passes its second
    // data slot's barriers, without bytes).  A parity wait cannot tell "the
    // previous use is done" from "the use before it is not", so every slot's
    // previous-but-one use must be consumed before anyone waits on the slot.
    // With an even SF_STAGES a scale slot belongs to one pair (slot parity =
    // stage parity), so a producer's scale-slot wait at sit finds its own
    // stage sit - SF_STAGES consumed, and by induction its earlier ones.  A
    // data slot alternates between the pairs; its previous-but-one use is
    // STAGES scale stages back: the pair's own stage sit - 10 (consumed, as
    // SF_STAGES <= 10), or with 9 data slots the other pair's stage sit - 9,
    // consumed before its stage sit - 7, which this pair's data slot waits at
    // sit - 2 had found consumed.  (An odd scale ring, shared by the pairs,
    // lets a producer whose issuer fell two uses behind pass early: measured
    // on a CPU simulation of this protocol.)
    static_assert(SF_STAGES % 2 == 0 && SF_STAGES <= 10 && (STAGES == 9 || STAGES == 10), "ring ownership");

    if (warp == 0 || warp == 8) {
        // ================= TMA producers =================
        if (lane == 0) {
            const int pi = (warp == 0) ? 0 : 1;
            uint32_t it_next = 0, sit_next = 0, sit_base = 0;
            bool ok = true;
            // a chained launch may start while the previous kernel on the
            // stream (the producer of the activations) still runs: the first
            // kDeferStages scale stages (whose scale and data slots are both
            // free at the start) load their weights at once and their
            // activation rows only after griddepcontrol.wait; ndef counts
            // this thread's deferred stages (scale stages pi, pi + 2, ...; a
            // chained launch has one phase)
            constexpr int kDeferStages = SF_STAGES < STAGES / 2 ? SF_STAGES : STAGES / 2;
            bool waited = (p.chained == 0);
            uint32_t ndef = 0;
            auto load_x = [&](uint32_t sit) {
                const uint32_t n = sit / (uint32_t)G0.np_loc, jl = sit % (uint32_t)G0.np_loc;
                const int64_t tn = t_first + (int64_t)n * t_step;
                const Item it = item_of(tn / ksplit, prefix, soff, E, G0.wtiles);
                const int j = jb_of(tn) + (int)jl;
                const uint32_t ita = 2 * sit;
                const int nd = min(2, G0.nks - 2 * j);
                const int r = sit % SF_STAGES;
                tma_load_2d(smem_u32(sSFXR + r * C::SFXR_BYTES), &m0.sfx, smem_u32(&sf_full[r]), j * C::SF_ROW,
                            (int)it.x0);
                for (int d = 0; d < nd; ++d) {
                    const int s = (ita + d) % STAGES;
                    tma_load_2d(smem_u32(sX + s * X_BYTES), &m0.x, smem_u32(&full[s]), (2 * j + d) * BKB, (int)it.x0);
                }
            };
            auto release_deferred = [&]() {
                asm volatile("griddepcontrol.wait;" ::: "memory");
                asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
                for (uint32_t i = 0; i < ndef; ++i) load_x((uint32_t)pi + 2 * i);
                waited = true;
            };
            int ph = 0;
            int64_t t = 0;
            for (int64_t n = 0; ok && item_at(n, ph, t); ++n) {
                const Geo g = ph ? G1 : G0;
                const Maps& mp = ph ? m1 : m0;
                const Item itm = item_of(ph ? t : t / ksplit, ph ? prefix2 : prefix, soff, E, g.wtiles);
                int64_t y0, y1;
                if (g.sw) w_rows<DS4G_EPI_SWIGLU_REQUANT>(itm, g.N, g.I, y0, y1);
                else w_rows<DS4G_EPI_NONE>(itm, g.N, g.I, y0, y1);
                const int jb = ph ? g.jb_rank : jb_of(t);
                const uint32_t sit0 = sit_base;
                sit_base += (uint32_t)g.np_loc;
                bool h_ready = !(kFfn && ph == 1);
                for (int jl = pi ^ (int)(sit0 & 1); jl < g.np_loc; jl += 2) {
                    const int j = jb + jl;                        // scale stage within the item's K
                    const uint32_t sit = sit0 + jl, ita = 2 * sit;
                    const int nd = min(2, g.nks - 2 * j);
                    const int r = sit % SF_STAGES;
                    // deferred stages never wait for a slot; the first other
                    // stage releases them before it waits (its slot frees
                    // only once a deferred stage has been consumed)
                    const bool defer = !waited && ph == 0 && sit < (uint32_t)kDeferStages;
                    if (!waited && !defer) release_deferred();
                    if (!h_ready) {
                        // the FFN's FC2: every FC1 item of this expert has
                        // stored its h columns
                        if (!wait_count(ctr + itm.e, prefix[itm.e + 1] - prefix[itm.e], abort_flag)) { ok = false; break; }
                        asm volatile("fence.proxy.async.global;" ::: "memory");
                        h_ready = true;
                    }
                    if (!mbar_wait(smem_u32(&sf_empty[r]), ((sit / SF_STAGES) & 1) ^ 1, abort_flag)) { ok = false; break; }
                    for (int d = 0; d < 2 && ok; ++d)
                        ok = mbar_wait(smem_u32(&empty[(ita + d) % STAGES]), (((ita + d) / STAGES) & 1) ^ 1, abort_flag);
                    if (!ok) break;
                    const uint32_t sfb = smem_u32(&sf_full[r]);
                    mbar_arrive_tx(sfb, C::SFW_BYTES + C::SFXR_BYTES);
                    const int x = j * C::SF_ROW;
                    tma_load_2d(smem_u32(sSFW + r * C::SFW_BYTES), &mp.sfw, sfb, x, (int)y0);
                    if (g.sw) tma_load_2d(smem_u32(sSFW + r * C::SFW_BYTES + C::SFW_BYTES / 2), &mp.sfw, sfb, x, (int)y1);
                    if (!defer) tma_load_2d(smem_u32(sSFXR + r * C::SFXR_BYTES), &mp.sfx, sfb, x, (int)itm.x0);
                    for (int d = 0; d < 2; ++d) {
                        const int s = (ita + d) % STAGES;
                        const int ks = 2 * j + d;
                        const uint32_t fb = smem_u32(&full[s]);
                        if (d >= nd) {
                            mbar_arrive(fb);                      // no second data stage: a use without bytes
                            continue;
                        }
                        mbar_arrive_tx(fb, W_BYTES + X_BYTES);
                        tma_load_2d(smem_u32(sW + s * W_BYTES), &mp.w, fb, ks * BKB, (int)y0);
                        if (g.sw) tma_load_2d(smem_u32(sW + s * W_BYTES + W_BYTES / 2), &mp.w, fb, ks * BKB, (int)y1);
                        if (!defer) tma_load_2d(smem_u32(sX + s * X_BYTES), &mp.x, fb, ks * BKB, (int)itm.x0);
                    }
                    if (defer) ++ndef;
                    it_next = ita + 2;
                    sit_next = sit + 1;
                }
            }
            // every armed stage gets its activation rows, also on an early exit
            if (!waited) release_deferred();
            if (!ok) {
                // let this thread's copies in flight land before the CTA goes
                // away: its stages among the last ring's worth.  Each wait has
                // its own bound; one that runs out means the slot has moved
                // on, i.e. that stage landed and was consumed long ago.
                for (uint32_t j = (it_next > STAGES ? it_next - STAGES : 0); j < it_next; ++j) {
                    volatile int never = 0;
                    if ((int)((j >> 1) & 1) == pi) mbar_wait(smem_u32(&full[j % STAGES]), (j / STAGES) & 1, &never);
                }
                for (uint32_t j = (sit_next > SF_STAGES ? sit_next - SF_STAGES : 0); j < sit_next; ++j) {
                    volatile int never = 0;
                    if ((int)(j & 1) == pi) mbar_wait(smem_u32(&sf_full[j % SF_STAGES]), (j / SF_STAGES) & 1, &never);
                }
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
            uint32_t sit_base = 0;
            bool ok = true;
            int ph = 0;
            int64_t t = 0;
            for (int64_t n = 0; ok && item_at(n, ph, t); ++n) {
                const Geo g = ph ? G1 : G0;
                const uint32_t tcount = (uint32_t)n;
                const int buf = tcount & 1;
                if (!mbar_wait(smem_u32(&tmem_empty[buf]), ((tcount >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t acc = tmem + kColAcc + pi * 32 + buf * BNT;
                const uint32_t sit0 = sit_base;
                sit_base += (uint32_t)g.np_loc;
                const int jb = ph ? g.jb_rank : jb_of(t);
                bool first = true;
                for (int jl = pi ^ (int)(sit0 & 1); jl < g.np_loc; jl += 2) {
                    const int j = jb + jl;                        // scale stage within the item's K
                    const uint32_t sit = sit0 + jl, ita = 2 * sit;
                    const int nd = min(2, g.nks - 2 * j);
                    const int r = sit % SF_STAGES;
                    if (!mbar_wait(smem_u32(&sf_ready[r]), (sit / SF_STAGES) & 1, abort_flag)) { ok = false; break; }
                    for (int d = 0; d < 2 && ok; ++d)
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
                        const int64_t krem = g.K - (int64_t)ks * BK;
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
                    if (nd < 2) mbar_arrive(smem_u32(&empty[(ita + 1) % STAGES]));   // the use without bytes
                    tc_commit(smem_u32(&sf_empty[r]));
                }
                if (!ok) break;
                tc_commit(smem_u32(&tmem_full[buf]));             // also when this issuer had no stage
            }
            // no tensor-core work of this thread may be in flight when the CTA
            // releases its tensor memory (an early exit leaves some)
            tc_commit(smem_u32(&drain[pi]));
            volatile int never = 0;
            mbar_wait(smem_u32(&drain[pi]), 0, &never);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ================= scale transposer =================
        uint32_t sit = 0;
        int ph = 0;
        int64_t t = 0;
        bool ok = true;
        for (int64_t n = 0; ok && item_at(n, ph, t); ++n) {
            const int np_loc = ph ? G1.np_loc : G0.np_loc;
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
        }
    } else if (warp >= 4) {
        // ================= epilogue =================
        const int q = warp & 3;                  // weight rows 32q .. 32q + 31 of the tile
        uint32_t sit_base = 0;
        const float gh = (FMT == DS4G_NVFP4 && (EPI == DS4G_EPI_SWIGLU_REQUANT || kFfn)) ? *p.oq_g : 1.0f;
        int ph = 0;
        int64_t t = 0;
        for (int64_t n = 0; item_at(n, ph, t); ++n) {
            const uint32_t tcount = (uint32_t)n;
            const Geo g = ph ? G1 : G0;
            const GemmArgs& a = ph ? p2 : p;
            // this item's epilogue: SwiGLU + requantisation, the combine or
            // the plain store
            const int epi = kFfn ? (ph ? kEpiCombine : DS4G_EPI_SWIGLU_REQUANT) : EPI;
            const int buf = tcount & 1;
            const uint32_t sit0 = sit_base;
            sit_base += (uint32_t)g.np_loc;
            const bool got = mbar_wait(smem_u32(&tmem_full[buf]), (tcount >> 1) & 1, abort_flag);
            // a pair's teardown is a warp-aligned cluster barrier: the whole
            // warp leaves the loop together
            if (SPLIT == 2 ? !__all_sync(0xffffffffu, got) : !got) break;
            tc_fence_after();
            const Item itm = item_of(ph ? t : t / ksplit, ph ? prefix2 : prefix, soff, E, g.wtiles);
            const float gscale = (FMT == DS4G_NVFP4) ? __fmul_rn(a.a_g[0], a.w_g[itm.e]) : 1.0f;
            // issuer i holds the sum over the scale stages of parity i; a
            // CTA of a pair may have none of an item's scale stages (the
            // FFN's FC2 with one scale stage per item): it adds nothing
            const uint32_t lanes = (uint32_t)(32 * q) << 16;
            float v[16];
            if (g.np_loc == 0) {
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = 0.0f;
            } else if (g.np_loc >= 2) {
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
            if (SPLIT == 2 && ph == 0) {
                // the follower sends its K half's sums for this item to the
                // leader, which adds them and runs the epilogue (the FFN's
                // FC2 items need no exchange: each half adds into out)
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
            if (epi != DS4G_EPI_SWIGLU_REQUANT) {
                if (g.np_loc == 0) continue;
                const int64_t nn = (int64_t)itm.wt * BMW + 32 * q + lane;
#pragma unroll
                for (int tt = 0; tt < BNT; ++tt) {
                    if (tt < itm.nr) {
                        if (epi == kEpiCombine) {
                            // add w * row into its token's output (coalesced along n)
                            const int32_t s = a.r2s[itm.x0 + tt];
                            atomicAdd(a.out + (int64_t)(s / a.topk) * a.N + nn, v[tt] * gscale * a.route_w[s]);
                        } else if (ksplit > 1) {
                            atomicAdd(a.out + (itm.x0 + tt) * a.N + nn, v[tt] * gscale);   // one K part of the sum
                        } else {
                            a.out[(itm.x0 + tt) * a.N + nn] = v[tt] * gscale;
                        }
                    }
                }
            } else {
                const int I = g.I;
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
                        if (a.h_debug) a.h_debug[row * I + col] = h;
                        uint32_t code;
                        if (FMT == DS4G_MXFP4) {
                            float m = fabsf(h);
#pragma unroll
                            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                            const int X = mx_shared_exp(m);
                            code = e2m1_code(__fmul_rn(h, exp2i(-X)));
                            if (lane == 0) a.oq_scales[row * (I / 32) + col / 32] = (uint8_t)(X + 127);
                        } else {
                            float m = fabsf(h);
#pragma unroll
                            for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                            const uint32_t s = ue4m3_encode(__fdiv_rn(m, __fmul_rn(6.0f, gh)));
                            const float ds = ue4m3_value(s);
                            code = (ds == 0.0f) ? ((__float_as_uint(h) >> 28) & 8u)
                                                : e2m1_code(__fmul_rn(h, __frcp_rn(__fmul_rn(ds, gh))));
                            if ((lane & 15) == 0) a.oq_scales[row * (I / 16) + col / 16] = (uint8_t)s;
                        }
                        const uint32_t hi_code = __shfl_down_sync(0xffffffffu, code, 1);
                        if ((lane & 1) == 0) a.oq_data[row * (I / 2) + col / 2] = (uint8_t)(code | (hi_code << 4));
                    }
                }
                if (kFfn) {
                    // this item's h columns are stored: count them for expert
                    // e's FC2 items (all epilogue threads' stores before the
                    // release)
                    asm volatile("bar.sync 1, 128;" ::: "memory");
                    if (threadIdx.x == 128)
                        asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(ctr + itm.e) : "memory");
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
    if (kFfn) {
        // the last CTA to finish sets the counters back to zero for the next
        // launch (every other CTA has read and published all it will)
        if (threadIdx.x == 0) {
            int32_t old;
            asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(ctr + E) : "memory");
            *last_cta = (old == (int32_t)gridDim.x - 1) ? 1 : 0;
        }
        __syncthreads();
        if (*last_cta)
            for (int e = threadIdx.x; e <= E; e += kThreads) ctr[e] = 0;
    }
}

}  // namespace dtc

// a2, ctr: the FFN's FC2 (EPI kEpiFfn) and its counters
template <int FMT, int EPI, int SPLIT = 1>
static cudaError_t run_dtc(const GemmArgs& a, cudaStream_t st, const GemmArgs* a2 = nullptr, int32_t* ctr = nullptr)
{
    using C = dtc::Cfg<FMT, SPLIT>;
    const int blk = (FMT == DS4G_MXFP4) ? 32 : 16;
    auto maps_of = [&](const GemmArgs& g, bool sw, dtc::Maps& m) {
        const uint32_t wbox = sw ? 64 : 128;
        return make_map(&m.w, g.w_data, (int64_t)g.E * g.N, g.K / 2, 128, wbox, true) &&
               make_map(&m.x, g.a_data, g.S, g.K / 2, 128, dtc::BNT, true) &&
               make_map(&m.sfw, g.w_scales, (int64_t)g.E * g.N, g.K / blk, C::SF_ROW, wbox, false) &&
               make_map(&m.sfx, g.a_scales, g.S, g.K / blk, C::SF_ROW, dtc::BNT, false);
    };
    constexpr bool kFfn = (EPI == kEpiFfn);
    dtc::Maps m0, m1;
    if (!maps_of(a, EPI == DS4G_EPI_SWIGLU_REQUANT || kFfn, m0)) return cudaErrorInvalidValue;
    if (kFfn) {
        if (!a2 || !ctr || !maps_of(*a2, false, m1)) return cudaErrorInvalidValue;
    } else {
        m1 = m0;
    }
    const GemmArgs b2 = kFfn ? *a2 : a;
    auto kern = dtc::k_gemv_tc<FMT, EPI, SPLIT>;
    const size_t shm = C::SMEM;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = kNumSMs;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (SPLIT == 1) {
        // may start while the previous kernel on the stream runs (the kernel
        // waits for it before reading any input; a chained FC2 before its
        // activation rows).  One CTA per SM: every CTA of the FFN is resident
        // once the previous kernel has left, as its FC2 items wait on FC1
        // items of other CTAs.
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
        e = cudaLaunchKernelEx(&cfg, kern, m0, m1, a, b2, ctr);
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
    e = cudaLaunchKernelEx(&cfg, kern, m0, m1, a, b2, ctr);
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

// Plain epilogue with few items (a dense GEMM of a few rows: 4096 weight rows
// are 32 items for 148 SMs): each item's K range in ksplit equal parts of
// whole scale stages, the largest divisor of the scale-stage count that keeps
// the items within two per SM, each part adding into the output (zeroed
// first).  1 = no split.
static int plain_ksplit(const GemmArgs& a, int sms)
{
    if (a.epilogue != DS4G_EPI_NONE || a.chained) return 1;
    const int nks = (int)ceil_div(a.K, 256);
    if (nks % 2 != 0) return 1;
    const int npairs = nks / 2;
    const int64_t est = (a.E < a.S ? a.E : a.S) * (int64_t)(a.N / 128);   // upper bound on the items
    if (est * 2 > sms) return 1;
    int best = 1;
    for (int q = 2; q <= npairs; ++q)
        if (npairs % q == 0 && est * q <= 2 * sms) best = q;
    return best;
}

cudaError_t launch_gemv_tc(const GemmArgs& a_in, cudaStream_t st)
{
    if (a_in.S == 0) return cudaSuccess;
    if (!gemv_tc_supports(a_in.fmt, a_in.K, a_in.N, a_in.epilogue, a_in.E)) return cudaErrorInvalidValue;
    GemmArgs a = a_in;
    int dev = 0, sms = kNumSMs;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    a.ksplit = plain_ksplit(a, sms);
    if (a.ksplit > 1) {
        cudaError_t e = cudaMemsetAsync(a.out, 0, sizeof(float) * (size_t)a.S * a.N, st);
        if (e != cudaSuccess) return e;
    }
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

bool ffn_dtc_supports(int fmt, int64_t d, int I, int E)
{
    return (fmt == DS4G_MXFP4 || fmt == DS4G_NVFP4) && gemv_tc_supports(fmt, d, 2 * I, DS4G_EPI_SWIGLU_REQUANT, E) &&
           gemv_tc_supports(fmt, I, (int)d, DS4G_EPI_NONE, E);
}

cudaError_t launch_ffn_dtc(const GemmArgs& fc1, const GemmArgs& fc2, int32_t* ctr, cudaStream_t st)
{
    if (fc1.S == 0) return cudaSuccess;
    if (!ffn_dtc_supports(fc1.fmt, fc1.K, fc1.N / 2, fc1.E) || fc2.K != fc1.N / 2 || fc2.fmt != fc1.fmt)
        return cudaErrorInvalidValue;
    // one CTA per SM, FC1 items not split over CTA pairs: the CTAs with one
    // FC1 item fewer start on FC2 items at once, which balances the SMs
    // better than halving every FC1 item (decode T = 1: 54.7 -> 51.1 us per
    // step, measured)
    if (fc1.fmt == DS4G_MXFP4) return run_dtc<DS4G_MXFP4, kEpiFfn>(fc1, st, &fc2, ctr);
    return run_dtc<DS4G_NVFP4, kEpiFfn>(fc1, st, &fc2, ctr);
}

}  // namespace ds4g
