// gemm_tc.cu -- prefill-sized grouped block-scaled FP4 GEMM on the 5th
// generation tensor cores (tcgen05), sm_100a.
//
// What it computes: "DGX Spark native FP4 matrix instructions: how DwarfStar
// uses Blackwell", sec. 1-2 (one block-scaled FP4 MMA consumes E2M1 operands
// and their UE8M0 / UE4M3 block scales directly, no dequantisation) and the
// grouped "contiguous" GEMM of "[DeepSeek V4] Triton FP4 optimisation in
// practice", "Step 0" (each expert's rows form one segment).  The page's
// kernel is the warp-level mma.sync m16n8k64 form of sm_12x; on sm_100a the
// same math is tcgen05.mma kind::mxf4 (.block32, UE8M0) / kind::mxf4nvf4
// (.block16, UE4M3) with the accumulator in tensor memory.  FP8 activations
// (MXFP8: E4M3 + UE8M0 per 32, the FP8 x FP4 GEMM of the same page's "Step
// 0") run the same kernel with kind::mxf8f6f4, against MXFP4 weights (loaded
// unpacked, one byte per element) or MXFP8 weights (a shared expert's).
//
// Design (one persistent CTA per SM, 384 threads, 448 with two MMA issuers,
// warp-specialised):
//   warp 0   TMA producer: tiles of A (128 rows x 128 bytes of K) and W
//            (up to 256 rows x 128 bytes) into 128B-swizzled shared memory
//            (4 stages), and the row-major scale bytes of two (FP4) or four
//            (FP8) K stages of both as 16 / 32-byte row boxes
//   warp 1   MMA issuer: the stage's scale words shared -> TMEM with
//            tcgen05.cp (32x128b.warpx4), 4 x tcgen05.mma (M128, K64 FP4 or
//            K32 FP8), tcgen05.commit releases the stage / publishes the
//            accumulator
//   warp 2   scale transposer: rewrites each scale stage in place from row
//            order into the 32-line x 16-byte chunks tcgen05.cp expects
//            (with two issuers warp 13 does the second issuer's stages)
//   warp 3   TMEM allocator (and, with two accumulators, the second issuer)
//   warps 4-11  epilogue: two warps per TMEM lane quarter, each reading half
//            of the tile's columns with tcgen05.ld (thread = tile row), then
//            the fp32 store or SwiGLU + requantisation
// Tiles (expert, n-tile, m-tile) are enumerated on the device from the
// expert offsets (no host read-back); every CTA walks tile t, t + #CTAs, ...
// Every mbarrier wait is bounded: past ~4 s it records kErrWaitTimeout in
// the device error word and the CTA winds down.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdlib.h>

#include "common.cuh"
#include "kernels.cuh"

namespace ds4g {

namespace tc {

constexpr int BM = 128;            // tile rows (tokens)
constexpr int BKB = 128;           // bytes of K per stage per row (256 FP4)
constexpr int STAGES = 4;
constexpr int kEpiWarps = 8;
constexpr int kProducer2Warp = 4 + kEpiWarps;   // the second TMA producer (two MMA issuers)
constexpr int kTransposer2Warp = 5 + kEpiWarps; // the second scale transposer (two MMA issuers)
constexpr int A_BYTES = BM * BKB;  // 16 KB
constexpr int kTmemCols = 512;
constexpr int kColAcc = 0;
constexpr int kMaxE = 1024;
constexpr unsigned long long kWaitNs = 4000000000ull;

// TBN: tile columns (weight rows).  256 with one accumulator; 224 (for N a
// multiple of 224, e.g. FC2 with N = 7168) with two, so that the epilogue of
// one tile overlaps the MMAs of the next: 2 x 224 accumulator columns plus
// the scale columns fit the 512 TMEM columns, 2 x 256 do not.
template <int FMT, int TBN, int NISS>
struct Cfg {
    static_assert(TBN == 256 || TBN == 224 || TBN == 192, "tile width");
    static_assert(NISS == 1 || (NISS == 2 && TBN < 256), "two issuers need two accumulators");
    static constexpr int NACC = (TBN == 256) ? 1 : 2;               // accumulator buffers
    static constexpr int HALF = TBN / 2;                             // weight rows per TMA box
    static constexpr int B_BYTES = TBN * BKB;                        // weight bytes per stage
    // bytes the weight loads of a stage count on its barrier: the shared
    // memory they fill, except for FP4 weights unpacked next to FP8
    // activations, whose loads write only the packed half of each 16-byte
    // chunk (the other half is a gap they leave untouched)
    static constexpr int B_TX = (FMT == DS4G_MXFP8) ? B_BYTES / 2 : B_BYTES;
    // K elements per K stage: 128 bytes of each operand row in shared
    // memory, i.e. 256 FP4 elements, or 128 for FP8 activations (their FP4
    // weight rows are unpacked to one byte per element on the way in)
    static constexpr int KE = fp8_act(FMT) ? 128 : 256;
    // 4-scale words per row per K stage (MX: 8 scales of 32, NV: 16 of 16,
    // FP8 activations: 4 of 32)
    static constexpr int WPS = (FMT == DS4G_MXFP4) ? 2 : (FMT == DS4G_NVFP4 ? 4 : 1);
    // K stages per scale stage, so that a row's scale box is at least the
    // 16 bytes a TMA copy moves
    static constexpr int KPS = fp8_act(FMT) ? 4 : 2;
    // TMEM scale columns per issuer: A (4 per word) then W (8 per word)
    static constexpr int SF_COLS = 12 * WPS;
    // scale stages in shared memory, each covering KPS K stages: two per issuer
    static constexpr int SF_STAGES = 2 * NISS;
    static constexpr int COL_SFA = NACC * TBN;
    static_assert(COL_SFA + NISS * SF_COLS <= 512, "TMEM columns");
    static constexpr int THREADS = 32 * (4 + kEpiWarps + (NISS == 2 ? 2 : 0));
    static constexpr int SF_ROW = KPS * WPS * 4;                     // scale bytes per row per scale stage
    static constexpr int SFA_BYTES = BM * SF_ROW;                    // one scale stage of A
    static constexpr int SFB_BYTES = 256 * SF_ROW;                   // one scale stage of W (two 128-row groups)
    static constexpr int SF_BYTES = SF_STAGES * (SFA_BYTES + SFB_BYTES);
    // 224-column tiles with one MMA issuer stage their fp32 epilogue through
    // shared memory, 16 rows x 32 columns per warp (rows padded to 33
    // floats), so that each store / reduction instruction covers 4 rows x 128
    // contiguous bytes.  With two issuers the mainloop is already bound by
    // shared-memory bandwidth and the staging traffic slows it more than the
    // wider reductions gain (measured: FC2 0.389 -> 0.448 ms at T = 2048), so
    // that configuration stores straight from registers.
    static constexpr bool STAGED = (TBN == 224 && NISS == 1);
    static constexpr int BAR_BYTES = 256;                            // barriers + TMEM slot + flags
    static constexpr int PREFIX_BYTES = ((kMaxE + 1) * 4 + 15) / 16 * 16;
    static constexpr int STAGE_BYTES = STAGED ? kEpiWarps * 16 * 33 * 4 : 0;
    static constexpr int NST = STAGES;                               // data ring
    static constexpr int DATA_BYTES = NST * (A_BYTES + B_BYTES);
    // tile prefix, then the expert offsets staged once ([E + 1] int32 each)
    static constexpr int STAGE_OFF = DATA_BYTES + SF_BYTES + BAR_BYTES + 2 * PREFIX_BYTES;
    static constexpr size_t SMEM = 1024 + (size_t)STAGE_OFF + STAGE_BYTES;
    static_assert(SMEM <= 232448, "shared memory per CTA");
    static_assert((2 * NST + 3 * SF_STAGES + 6) * 8 + 16 <= BAR_BYTES, "barrier block");
};

// ---- PTX wrappers ----------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ uint64_t globaltimer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t a, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint32_t a, uint32_t tx)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(a), "r"(tx) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t a)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(a) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t a, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    return ok != 0;
}

// bounded wait; false when it gave up (or another role already gave up).
// Spins without touching the timer first, so a wait that completes within a
// few thousand polls costs nothing extra.
__device__ __forceinline__ bool mbar_wait(uint32_t a, uint32_t parity, volatile int* abort_flag)
{
#pragma unroll 1
    for (int i = 0; i < 4096; ++i)
        if (mbar_try(a, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try(a, parity)) return true;
        if ((it & 255u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > kWaitNs) {
                *abort_flag = 1;
                raise_error(kErrWaitTimeout);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void fence_barrier_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t mbar, int x, int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(dst), "l"((uint64_t)map), "r"(mbar), "r"(x), "r"(y)
        : "memory");
}

// ---- cluster (CTA pair) wrappers, used by the decode kernel's split mode
__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id_x()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t nclusters_x()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
// all threads of both CTAs of the cluster
__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// shared::cluster address of the object at shared::cta address `a` in CTA `rank`
__device__ __forceinline__ uint32_t mapa_shared(uint32_t a, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}
// arrive on an mbarrier of either CTA of the cluster.  Default (CTA-scope)
// release: a cluster-scope release made the leader see each arrival about
// 2,000 cycles late (measured), stalling the MMA issuer at every scale stage.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// shared-memory matrix descriptor (tcgen05): K-major, 128-byte swizzle,
// 8-row core groups 1024 bytes apart
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)(1024 >> 4) << 32;     // stride byte offset
    d |= (uint64_t)1 << 46;               // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;               // SWIZZLE_128B
    return d;
}

// descriptor of one 32 x 16-byte scale-factor chunk (no swizzle, 8-row core
// matrices 128 bytes apart)
__device__ __forceinline__ uint64_t desc_sf(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)(128 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    return d;
}

// instruction descriptor: fp32 accumulate, K-major A and B, M = 128,
// N = TBN.  FP4 formats (kind::mxf4 / mxf4nvf4): E2M1 x E2M1 (type code 1),
// scale format UE8M0 (MX) or UE4M3 (NV).  FP8 activations (kind::mxf8f6f4):
// A E4M3 (code 0) x B E2M1 (code 5) or, with FP8 weights, E4M3 (code 0);
// UE8M0.
template <int FMT, int TBN>
__device__ __forceinline__ uint32_t idesc_base()
{
    const uint32_t at = fp8_act(FMT) ? 0u : 1u;
    const uint32_t bt = (FMT == DS4G_MXFP8) ? 5u : (FMT == kFmtFp8Fp8 ? 0u : 1u);
    return (at << 7) | (bt << 10) | ((uint32_t)(TBN >> 3) << 17) | ((FMT == DS4G_NVFP4 ? 0u : 1u) << 23) |
           ((uint32_t)(BM >> 4) << 24);
}

template <int FMT>
__device__ __forceinline__ void mma(uint32_t d_tmem, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t acc,
                                    uint32_t sfa, uint32_t sfb)
{
    if (fp8_act(FMT)) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
            ::"r"(d_tmem), "l"(ad), "l"(bd), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
            : "memory");
    } else if (FMT == DS4G_MXFP4) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
            ::"r"(d_tmem), "l"(ad), "l"(bd), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
            ::"r"(d_tmem), "l"(ad), "l"(bd), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
            : "memory");
    }
}

// shared -> tensor memory copy of one 32 x 16-byte scale chunk into all four
// lane quarters
__device__ __forceinline__ void utccp(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// arrive on `mbar` once the thread's earlier tensor-core operations are done
__device__ __forceinline__ void tc_commit(uint32_t mbar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}

// 16 TMEM lanes x 16 columns: thread t gets lanes t/4 and t/4 + 8, columns
// 2(t%4), 2(t%4)+1 (r0, r1 / r2, r3) and 8 + 2(t%4), +1 (r4, r5 / r6, r7)
__device__ __forceinline__ void tmem_ld_16x256b_x2(uint32_t taddr, uint32_t* r)
{
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// G consecutive 16-column chunks of the same 16x256b.x2 shape, one wait for
// all of them; the empty asm statements after the wait make every later use
// of the registers depend on it
template <int G>
__device__ __forceinline__ void tmem_ld_16x256b_x2_batch(uint32_t taddr, uint32_t (&r)[G][8])
{
#pragma unroll
    for (int g = 0; g < G; ++g)
        asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=r"(r[g][0]), "=r"(r[g][1]), "=r"(r[g][2]), "=r"(r[g][3]), "=r"(r[g][4]), "=r"(r[g][5]),
                       "=r"(r[g][6]), "=r"(r[g][7])
                     : "r"(taddr + 16u * g)
                     : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int g = 0; g < G; ++g)
        asm volatile(""
                     : "+r"(r[g][0]), "+r"(r[g][1]), "+r"(r[g][2]), "+r"(r[g][3]), "+r"(r[g][4]), "+r"(r[g][5]),
                       "+r"(r[g][6]), "+r"(r[g][7]));
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v)
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v)
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// in-place transposition of one scale stage of `rows` rows (multiple of 128)
// from row order [rows][words * 4 bytes] to the tcgen05.cp chunk order: for
// 128-row group g and word c, a 512-byte chunk at ((c * groups) + g) * 512
// whose 16-byte line l holds word c of rows l, l + 32, l + 64, l + 96.
template <int WORDS, int GROUPS>
__device__ __forceinline__ void sf_transpose(uint8_t* base, int lane)
{
    uint32_t v[GROUPS][4][WORDS];
#pragma unroll
    for (int g = 0; g < GROUPS; ++g)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t* row = reinterpret_cast<const uint32_t*>(base + (size_t)(g * 128 + q * 32 + lane) * WORDS * 4);
#pragma unroll
            for (int c = 0; c < WORDS; c += 4) {
                const uint4 x = *reinterpret_cast<const uint4*>(row + c);
                v[g][q][c] = x.x; v[g][q][c + 1] = x.y; v[g][q][c + 2] = x.z; v[g][q][c + 3] = x.w;
            }
        }
    __syncwarp();
#pragma unroll
    for (int g = 0; g < GROUPS; ++g)
#pragma unroll
        for (int c = 0; c < WORDS; ++c)
            *reinterpret_cast<uint4*>(base + (size_t)((c * GROUPS + g) * 512 + lane * 16)) =
                make_uint4(v[g][0][c], v[g][1][c], v[g][2][c], v[g][3][c]);
    __syncwarp();
}

// ---- tile enumeration --------------------------------------------------------
struct Tile {
    int e;        // expert
    int nt;       // column tile
    int64_t m0;   // first row of the tile
    int64_t end;  // end of the expert's segment
};

// Tiles are numbered band by band: a band is nb consecutive column tiles
// (the last band may be narrower), and within a band expert by expert, then
// column tile, then row tile.  prefix[e] counts the row tiles of the experts
// before e (prefix[E] of all of them).  With one band (nb = n_tiles) this is
// expert-major order.  The combine epilogue uses several bands when the
// output is larger than L2: the reductions of all experts into one band's
// columns of the output then happen while those columns are in L2.
__device__ __forceinline__ Tile tile_of(int64_t t, const int32_t* prefix, const int32_t* offsets, int E,
                                        int n_tiles, int nb)
{
    const int64_t U = prefix[E];
    const int nbands = (n_tiles + nb - 1) / nb;
    int64_t band = t / (U * nb);
    if (band > nbands - 1) band = nbands - 1;
    const int nbb = min(nb, n_tiles - (int)band * nb);          // column tiles of this band
    const int64_t local = t - band * U * nb;
    int lo = 0, hi = E - 1;   // largest e with prefix[e] * nbb <= local (prefix non-decreasing)
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if ((int64_t)prefix[mid] * nbb <= local) lo = mid; else hi = mid - 1;
    }
    Tile r;
    r.e = lo;
    const int64_t beg = offsets[lo];
    r.end = offsets[lo + 1];
    const int64_t mt_cnt = ceil_div(r.end - beg, BM);
    const int64_t le = local - (int64_t)prefix[lo] * nbb;
    r.nt = (int)(band * nb + le / mt_cnt);
    r.m0 = beg + (le % mt_cnt) * BM;
    return r;
}

// first weight rows of the two halves of the W tile
template <int EPI, int TBN>
__device__ __forceinline__ void w_rows(const Tile& tl, int N, int I, int64_t& y0, int64_t& y1)
{
    const int64_t wbase = (int64_t)tl.e * N;
    if (EPI == DS4G_EPI_SWIGLU_REQUANT) {
        y0 = wbase + (int64_t)tl.nt * (TBN / 2);          // gate rows
        y1 = wbase + I + (int64_t)tl.nt * (TBN / 2);      // up rows
    } else {
        y0 = wbase + (int64_t)tl.nt * TBN;
        y1 = y0 + TBN / 2;
    }
}

template <int FMT, int EPI, int TBN, int NISS>
__global__ void __launch_bounds__(Cfg<FMT, TBN, NISS>::THREADS, 1)
k_gemm_tc(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
          const __grid_constant__ CUtensorMap map_sfa, const __grid_constant__ CUtensorMap map_sfb, const GemmArgs p)
{
    using C = Cfg<FMT, TBN, NISS>;
    constexpr int STAGES = C::NST;
    constexpr int SF_STAGES = C::SF_STAGES;
    static_assert(EPI != DS4G_EPI_SWIGLU_REQUANT || TBN == 256 || TBN == 192,
                  "SwiGLU tiles pair TBN/2 gate and TBN/2 up rows, a multiple of 32 each");
    constexpr int NACC = C::NACC;
    constexpr int B_BYTES = C::B_BYTES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + STAGES * A_BYTES;
    uint8_t* sSFA = sB + STAGES * B_BYTES;                 // [SF_STAGES][SFA_BYTES]
    uint8_t* sSFB = sSFA + SF_STAGES * C::SFA_BYTES;       // [SF_STAGES][SFB_BYTES]
    uint64_t* bars = reinterpret_cast<uint64_t*>(sSFB + SF_STAGES * C::SFB_BYTES);
    uint64_t* full = bars;                                 // [STAGES]  TMA data landed
    uint64_t* empty = full + STAGES;                       // [STAGES]  MMAs done with the data
    uint64_t* sf_full = empty + STAGES;                    // [SF_STAGES] TMA scales landed
    uint64_t* sf_ready = sf_full + SF_STAGES;              // [SF_STAGES] scales transposed
    uint64_t* sf_empty = sf_ready + SF_STAGES;             // [SF_STAGES] MMAs done with the scales
    uint64_t* tmem_full = sf_empty + SF_STAGES;            // [NACC] accumulator complete
    uint64_t* tmem_empty = tmem_full + 2;                  // [NACC] accumulator drained
    uint64_t* drain = tmem_empty + 2;                      // [NISS] each issuer's tensor-core work finished
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int32_t* total_tiles = reinterpret_cast<int32_t*>(tmem_slot + 2);
    int32_t* prefix = reinterpret_cast<int32_t*>(smem + C::DATA_BYTES + C::SF_BYTES + C::BAR_BYTES);
    int32_t* soff = prefix + C::PREFIX_BYTES / 4;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;
    const int64_t K = p.K;
    constexpr int KPS = C::KPS;
    // split K (plain epilogue, few tiles): every tile comes ksplit times,
    // part q taking K stages [q nks, (q + 1) nks) and adding its partial sums
    // into the zeroed output (the host splits only into equal parts of whole
    // scale stages)
    const int ksplit = (EPI == DS4G_EPI_NONE && p.ksplit > 1) ? p.ksplit : 1;
    const int nks = (int)ceil_div(K, C::KE) / ksplit;   // K stages per tile (part)
    const int nsfs = (nks + KPS - 1) / KPS;              // scale stages per tile (part)
    const int I = p.N / 2;
    // SwiGLU: the last tile may be ragged (I % (TBN/2) != 0); its columns past
    // I are computed from other rows and never stored
    const int n_tiles = (EPI == DS4G_EPI_SWIGLU_REQUANT) ? (int)ceil_div(I, TBN / 2) : (int)ceil_div(p.N, TBN);
    // column tiles per band of the tile order (see tile_of)
    const int nb = (EPI == kEpiCombine && p.band_tiles > 0 && p.band_tiles < n_tiles) ? p.band_tiles : n_tiles;
    const int64_t tile0 = blockIdx.x;
    const int64_t tstride = gridDim.x;

    // ---- prologue
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
        for (int b2 = 0; b2 < NACC; ++b2) {
            mbar_init(smem_u32(&tmem_full[b2]), 1);
            mbar_init(smem_u32(&tmem_empty[b2]), 32 * kEpiWarps);
        }
        mbar_init(smem_u32(&drain[0]), 1);
        mbar_init(smem_u32(&drain[1]), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    // the expert offsets -> shared memory in one parallel pass (a loop of
    // dependent global loads here cost about 2 us per launch)
    for (int e = threadIdx.x; e <= E; e += C::THREADS) soff[e] = p.offsets[e];
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_a) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_b) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_sfa) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&map_sfb) : "memory");
    }
    if (warp == 3) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    __syncthreads();
    if (warp == 0) {
        // row tiles per expert, exclusive scan by one warp
        const int per = (E + 31) / 32;
        int32_t sum = 0;
        for (int i = 0; i < per; ++i) {
            const int e = lane * per + i;
            if (e < E) sum += (int32_t)ceil_div((int64_t)soff[e + 1] - soff[e], BM);
        }
        int32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int32_t run = incl - sum;
        for (int i = 0; i < per; ++i) {
            const int e = lane * per + i;
            if (e < E) {
                prefix[e] = run;
                run += (int32_t)ceil_div((int64_t)soff[e + 1] - soff[e], BM);
            }
        }
        if (lane == 31) {
            prefix[E] = incl;
            int32_t tot = incl * n_tiles * ksplit;
            if ((int64_t)soff[E] > p.S) {   // inconsistent offsets: do nothing
                raise_error(kErrBadOffsets);
                tot = 0;
            }
            *total_tiles = tot;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int64_t ntiles = *total_tiles;

    // Ring slots belong to tile group members: member m of a group (issuer m,
    // producer m) uses data slots m, m + NISS, ... and scale slots m, m +
    // NISS, counting its own uses l = 0, 1, ... (slot NISS (l % depth) + m,
    // phase (l / depth) & 1).  Each slot then has one producer and one
    // consumer taking its uses in order, which the parity waits require.
    constexpr int DPM = STAGES / NISS;       // data slots per member
    constexpr int SPM = SF_STAGES / NISS;    // scale slots per member
    static_assert(DPM * NISS == STAGES && SPM * NISS == SF_STAGES && SPM == 2, "ring split");

    if (warp == 0 || (NISS == 2 && warp == kProducer2Warp)) {
        // ================= TMA producer(s) =================
        // This CTA's tiles come in groups of NISS consecutive ones.  Producer
        // pp (warp 0, and warp 12 with two issuers) loads the data and scale
        // stages of member pp of each group, the ones issuer pp consumes.  A
        // thread that has issued copies and then waits on a barrier first
        // waits for its copies to land; with two producers one's copies are
        // in flight while the other waits for a free slot.
        if (lane == 0) {
            const int pp = (warp == 0) ? 0 : 1;
            uint32_t ld = 0, ls = 0;           // this member's data / scale uses issued
            bool ok = true;
            for (int64_t j0 = 0; ok; j0 += NISS) {
                const int64_t t0 = tile0 + j0 * tstride;
                if (t0 >= ntiles) break;
                const int gsz = (NISS == 2 && t0 + tstride < ntiles) ? 2 : 1;
                if (pp >= gsz) break;                                   // the CTA's last group has one member
                const int64_t t = t0 + pp * tstride;
                const Tile tl = tile_of(t / ksplit, prefix, soff, E, n_tiles, nb);
                const int kb = (int)(t % ksplit) * nks;                  // first K stage of this part
                int64_t y0, y1;
                w_rows<EPI, TBN>(tl, p.N, I, y0, y1);
                for (int ks = 0; ks < nks; ++ks) {
                    if ((ks % KPS) == 0) {
                        const int r = NISS * (int)(ls % SPM) + pp;
                        if (!mbar_wait(smem_u32(&sf_empty[r]), ((ls / SPM) & 1) ^ 1, abort_flag)) { ok = false; break; }
                        const uint32_t fb = smem_u32(&sf_full[r]);
                        mbar_arrive_tx(fb, C::SFA_BYTES + TBN * C::SF_ROW);
                        const int x = ((kb + ks) / KPS) * C::SF_ROW;
                        tma_load_2d(smem_u32(sSFA + r * C::SFA_BYTES), &map_sfa, fb, x, (int)tl.m0);
                        tma_load_2d(smem_u32(sSFB + r * C::SFB_BYTES), &map_sfb, fb, x, (int)y0);
                        tma_load_2d(smem_u32(sSFB + r * C::SFB_BYTES + C::HALF * C::SF_ROW), &map_sfb, fb, x, (int)y1);
                        ++ls;
                    }
                    const int s = NISS * (int)(ld % DPM) + pp;
                    if (!mbar_wait(smem_u32(&empty[s]), ((ld / DPM) & 1) ^ 1, abort_flag)) { ok = false; break; }
                    const uint32_t fb = smem_u32(&full[s]);
                    mbar_arrive_tx(fb, A_BYTES + C::B_TX);
                    const int kx = (kb + ks) * BKB;
                    tma_load_2d(smem_u32(sA + s * A_BYTES), &map_a, fb, kx, (int)tl.m0);
                    tma_load_2d(smem_u32(sB + s * B_BYTES), &map_b, fb, kx, (int)y0);
                    tma_load_2d(smem_u32(sB + s * B_BYTES + B_BYTES / 2), &map_b, fb, kx, (int)y1);
                    ++ld;
                }
            }
            if (!ok) {
                // let this member's copies in flight land before the CTA goes
                // away: its latest uses of each slot (earlier ones completed
                // before their slot was refilled)
                for (uint32_t l = (ld > (uint32_t)DPM ? ld - DPM : 0u); l < ld; ++l) {
                    volatile int never = 0;
                    mbar_wait(smem_u32(&full[NISS * (int)(l % DPM) + pp]), (l / DPM) & 1, &never);
                }
                for (uint32_t l = (ls > (uint32_t)SPM ? ls - SPM : 0u); l < ls; ++l) {
                    volatile int never = 0;
                    mbar_wait(smem_u32(&sf_full[NISS * (int)(l % SPM) + pp]), (l / SPM) & 1, &never);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1 || (NISS == 2 && warp == 3)) {
        // ================= MMA issuer(s) =================
        // Issuer pi takes member pi of each tile group, accumulating into
        // accumulator pi (two issuers) with its own scale columns.  An issuing
        // thread that waits on a barrier first drains its own tensor-core
        // work; with two issuers the other one's MMAs fill that gap.
        if (lane == 0) {
            const int pi = (warp == 1) ? 0 : 1;
            const uint32_t ibase = idesc_base<FMT, TBN>();
            const uint32_t col_sfa = tmem + C::COL_SFA + pi * C::SF_COLS;
            const uint32_t col_sfb = col_sfa + 4 * C::WPS;
            uint32_t ld = 0, ls = 0;           // this member's data / scale uses consumed
            bool ok = true;
            for (int64_t j0 = 0; ok; j0 += NISS) {
                const int64_t t0 = tile0 + j0 * tstride;
                if (t0 >= ntiles) break;
                const int gsz = (NISS == 2 && t0 + tstride < ntiles) ? 2 : 1;
                if (pi >= gsz) break;
                const int64_t jt = j0 + pi;                        // this CTA's local tile index
                const int buf = (NISS == 2) ? pi : (int)(jt % NACC);
                const uint32_t use = (NISS == 2) ? (uint32_t)(j0 / 2) : (uint32_t)(jt / NACC);
                if (!mbar_wait(smem_u32(&tmem_empty[buf]), (use & 1) ^ 1, abort_flag)) break;
                const uint32_t acc = tmem + kColAcc + buf * TBN;
                const int kb = (int)((t0 + pi * tstride) % ksplit) * nks;   // first K stage of this part
                tc_fence_after();
                int r = 0;
                for (int ks = 0; ks < nks; ++ks) {
                    if ((ks % KPS) == 0) {
                        r = NISS * (int)(ls % SPM) + pi;
                        if (!mbar_wait(smem_u32(&sf_ready[r]), (ls / SPM) & 1, abort_flag)) { ok = false; break; }
                        ++ls;
                    }
                    const int s = NISS * (int)(ld % DPM) + pi;
                    if (!mbar_wait(smem_u32(&full[s]), (ld / DPM) & 1, abort_flag)) { ok = false; break; }
                    ++ld;
                    tc_fence_after();
                    // this K stage's scale words -> TMEM
                    const int w0 = (ks % KPS) * C::WPS;
                    const uint32_t sfa_s = smem_u32(sSFA + r * C::SFA_BYTES);
                    const uint32_t sfb_s = smem_u32(sSFB + r * C::SFB_BYTES);
#pragma unroll
                    for (int c = 0; c < C::WPS; ++c) {
                        utccp(col_sfa + 4 * c, desc_sf(sfa_s + (w0 + c) * 512));
                        utccp(col_sfb + 8 * c, desc_sf(sfb_s + ((w0 + c) * 2 + 0) * 512));
                        utccp(col_sfb + 8 * c + 4, desc_sf(sfb_s + ((w0 + c) * 2 + 1) * 512));
                    }
                    const int64_t krem = K - (int64_t)(kb + ks) * C::KE;
                    const int nmma = krem >= C::KE ? 4 : (int)(krem / (C::KE / 4));
                    const uint32_t a_s = smem_u32(sA + s * A_BYTES);
                    const uint32_t b_s = smem_u32(sB + s * B_BYTES);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        if (j < nmma) {
                            // scale word (4 TMEM columns) and byte of MMA j:
                            // MX K = 64 takes 2 scales (bytes 0-1 / 2-3 of
                            // word j / 2), NV K = 64 all 4 of word j, MXFP8
                            // K = 32 byte j of the stage's one word
                            const int c = (FMT == DS4G_MXFP4) ? (j >> 1) : (FMT == DS4G_NVFP4 ? j : 0);
                            const uint32_t sfid = (FMT == DS4G_MXFP4) ? (uint32_t)((j & 1) * 2)
                                                                     : (FMT == DS4G_NVFP4 ? 0u : (uint32_t)j);
                            const uint32_t idesc = ibase | (sfid << 4) | (sfid << 29);
                            mma<FMT>(acc, desc_sw128(a_s + 32 * j), desc_sw128(b_s + 32 * j), idesc,
                                     (ks > 0 || j > 0) ? 1u : 0u, col_sfa + 4 * c, col_sfb + 8 * c);
                        }
                    }
                    tc_commit(smem_u32(&empty[s]));
                    if ((ks % KPS) == KPS - 1 || ks == nks - 1) tc_commit(smem_u32(&sf_empty[r]));
                }
                if (!ok) break;
                tc_commit(smem_u32(&tmem_full[buf]));
            }
            // no tensor-core work of this thread may be in flight when the CTA
            // releases its tensor memory (an early exit leaves some)
            tc_commit(smem_u32(&drain[pi]));
            volatile int never = 0;
            mbar_wait(smem_u32(&drain[pi]), 0, &never);
        }
        __syncwarp();
    } else if (warp == 2 || (NISS == 2 && warp == kTransposer2Warp)) {
        // ================= scale transposer(s) =================
        // one per tile group member (warp 2, and warp 13 with two issuers),
        // taking that member's scale stages in order, so that neither
        // issuer's scales wait behind the other's (with one warp for both,
        // the issuers waited 14-23% of their time for transposed scales)
        const int m = (warp == 2) ? 0 : 1;
        uint32_t ls = 0;
        bool ok = true;
        for (int64_t j0 = 0; ok; j0 += NISS) {
            const int64_t t0 = tile0 + j0 * tstride;
            if (t0 >= ntiles) break;
            const int gsz = (NISS == 2 && t0 + tstride < ntiles) ? 2 : 1;
            if (m >= gsz) break;                                    // the CTA's last group has one member
            for (int pr = 0; pr < nsfs && ok; ++pr) {
                const int r = NISS * (int)(ls % SPM) + m;
                bool w_ok = true;
                if (lane == 0) w_ok = mbar_wait(smem_u32(&sf_full[r]), (ls / SPM) & 1, abort_flag);
                if (!__shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0)) { ok = false; break; }
                ++ls;
                sf_transpose<KPS * C::WPS, 1>(sSFA + r * C::SFA_BYTES, lane);
                sf_transpose<KPS * C::WPS, 2>(sSFB + r * C::SFB_BYTES, lane);
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&sf_ready[r]));
            }
        }
    } else if (warp >= 4 && warp < 4 + kEpiWarps) {
        // ================= epilogue =================
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        const int half = (warp - 4) >> 2;       // which half of the tile's columns
        uint32_t tcount = 0;
        const float gh = (FMT == DS4G_NVFP4 && EPI == DS4G_EPI_SWIGLU_REQUANT) ? *p.oq_g : 1.0f;
        for (int64_t t = tile0; t < ntiles; t += tstride, ++tcount) {
            const int buf = (int)(tcount % NACC);
            // the tile, its scale and (register-direct plain / combine
            // epilogue) the output rows of this thread's four tile rows are
            // looked up before waiting for the accumulator, so that their
            // global loads overlap the tile's mainloop
            const Tile tl = tile_of(t / ksplit, prefix, soff, E, n_tiles, nb);
            const float gscale = (FMT == DS4G_NVFP4) ? __fmul_rn(p.a_g[0], p.w_g[tl.e]) : 1.0f;
            constexpr bool kDirect = (EPI != DS4G_EPI_SWIGLU_REQUANT) && !C::STAGED;
            float* dk[2][2];
            float wk[2][2];
            if (kDirect) {
                // rows 16 hh + rsub + 8 k of the warp's 32: four threads hold
                // 32 contiguous bytes of one row in the 16-lane TMEM loads
                const int rsub = lane >> 2;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const int64_t rk = tl.m0 + 32 * q + 16 * hh + rsub + 8 * k;
                        dk[hh][k] = nullptr;
                        wk[hh][k] = gscale;
                        if (rk < tl.end) {
                            if (EPI == kEpiCombine) {
                                const int32_t s = p.r2s[rk];
                                dk[hh][k] = p.out + (int64_t)(s / p.topk) * p.N + (int64_t)tl.nt * TBN;
                                wk[hh][k] = p.route_w[s] * gscale;
                            } else {
                                dk[hh][k] = p.out + rk * p.N + (int64_t)tl.nt * TBN;
                            }
                        }
                    }
            }
            if (!mbar_wait(smem_u32(&tmem_full[buf]), (tcount / NACC) & 1, abort_flag)) break;
            tc_fence_after();
            const int64_t row = tl.m0 + 32 * q + lane;
            const bool valid = row < tl.end;
            const uint32_t tbase = tmem + kColAcc + buf * TBN + ((uint32_t)(32 * q) << 16);
            if (EPI != DS4G_EPI_SWIGLU_REQUANT) {
                // plain: store the row; combine: add w * row into its token's output
                if (C::STAGED) {
                    float* dst_row = p.out + row * p.N;
                    float wr = gscale;
                    if (EPI == kEpiCombine && valid) {
                        const int32_t s = p.r2s[row];
                        dst_row = p.out + (int64_t)(s / p.topk) * p.N;
                        wr = p.route_w[s] * gscale;
                    }
                    // 32-column pieces of this warp's half (the last one 16 wide),
                    // each as two 16-row blocks through the warp's staging area
                    float* stg = reinterpret_cast<float*>(smem + C::STAGE_OFF) + (warp - 4) * (16 * 33);
                    const unsigned long long my_dst =
                        valid ? reinterpret_cast<unsigned long long>(dst_row + (int64_t)tl.nt * TBN) : 0ull;
#pragma unroll 1
                    for (int c8 = 0; c8 < (C::HALF + 31) / 32; ++c8) {
                        const int col = half * C::HALF + 32 * c8;
                        const int ncol = min(32, C::HALF - 32 * c8);
                        float v[32];
                        if (ncol == 32) tmem_ld32(tbase + col, v);
                        else tmem_ld16(tbase + col, v);
#pragma unroll 1
                        for (int hh = 0; hh < 2; ++hh) {
                            if ((lane >> 4) == hh) {
                                float* srow = stg + (lane & 15) * 33;
#pragma unroll
                                for (int i = 0; i < 32; ++i)
                                    if (i < ncol) srow[i] = v[i] * wr;
                            }
                            __syncwarp();
#pragma unroll
                            for (int i4 = 0; i4 < 4; ++i4) {
                                const int rl = 4 * i4 + (lane >> 3);       // staged row
                                const unsigned long long d = __shfl_sync(0xffffffffu, my_dst, 16 * hh + rl);
                                const int cc = (lane & 7) * 4;
                                if (d != 0ull && cc < ncol) {
                                    const float* sr = stg + rl * 33 + cc;
                                    float* g = reinterpret_cast<float*>(d) + col + cc;
                                    if (EPI == kEpiCombine || ksplit > 1)     // combine, or one K part of the sum
                                        red_add_v4(g, sr[0], sr[1], sr[2], sr[3]);
                                    else
                                        *reinterpret_cast<float4*>(g) = make_float4(sr[0], sr[1], sr[2], sr[3]);
                                }
                            }
                            __syncwarp();
                        }
                    }
                } else {
                    // 16-lane x 16-column TMEM loads: four threads hold 32
                    // contiguous bytes of one row, so a store / reduction
                    // instruction writes 8 rows x 32 bytes (full sectors).
                    // All of a row half's loads are issued before one wait.
                    constexpr int G = C::HALF / 16;
                    const int sub = lane & 3;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const uint32_t tb = tmem + kColAcc + buf * TBN + ((uint32_t)(32 * q + 16 * hh) << 16) +
                                            half * C::HALF;
                        uint32_t r[G][8];
                        tmem_ld_16x256b_x2_batch<G>(tb, r);
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            const int col = half * C::HALF + 16 * g;
                            if ((int64_t)tl.nt * TBN + col >= p.N) break;      // ragged last tile
#pragma unroll
                            for (int k = 0; k < 2; ++k) {
                                if (dk[hh][k] == nullptr) continue;
                                float* g0 = dk[hh][k] + col + 2 * sub;
                                const float w = wk[hh][k];
                                const float a0 = __uint_as_float(r[g][2 * k]) * w;
                                const float a1 = __uint_as_float(r[g][2 * k + 1]) * w;
                                const float b0 = __uint_as_float(r[g][4 + 2 * k]) * w;
                                const float b1 = __uint_as_float(r[g][4 + 2 * k + 1]) * w;
                                if (EPI == kEpiCombine || ksplit > 1) {   // combine, or one K part of the sum
                                    red_add_v2(g0, a0, a1);
                                    red_add_v2(g0 + 8, b0, b1);
                                } else {
                                    *reinterpret_cast<float2*>(g0) = make_float2(a0, a1);
                                    *reinterpret_cast<float2*>(g0 + 8) = make_float2(b0, b1);
                                }
                            }
                        }
                    }
                }
            } else {
#pragma unroll 1
                for (int j = half; j < C::HALF / 32; j += 2) {       // 32-column blocks of h
                    const int gcol = 32 * j;                         // gate column within the tile
                    const int64_t col0 = (int64_t)tl.nt * C::HALF + gcol;
                    if (col0 >= I) break;                            // ragged last tile
                    float gv[32], uv[32];
                    tmem_ld32(tbase + gcol, gv);
                    tmem_ld32(tbase + C::HALF + gcol, uv);
                    float h[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        h[i] = swiglu_f32(__fmul_rn(gv[i], gscale), __fmul_rn(uv[i], gscale));
                    }
                    if (valid) {
                        if (p.h_debug) {
                            float4* hd = reinterpret_cast<float4*>(p.h_debug + row * I + col0);
#pragma unroll
                            for (int i = 0; i < 8; ++i) hd[i] = make_float4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
                        }
                        uint32_t wq[4] = {0, 0, 0, 0};
                        if (fp8_act(FMT)) {
                            // "SwiGLU + FP8 quant": h -> E4M3 with a UE8M0
                            // scale per 32 (OCP MX rule, largest exponent 8)
                            float m = 0.f;
#pragma unroll
                            for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(h[i]));
                            const int X = mx_shared_exp<8>(m);
                            const float inv = exp2i(-X);
                            uint32_t w8[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                w8[i] = e4m3x2(__fmul_rn(h[4 * i], inv), __fmul_rn(h[4 * i + 1], inv)) |
                                        (e4m3x2(__fmul_rn(h[4 * i + 2], inv), __fmul_rn(h[4 * i + 3], inv)) << 16);
                            p.oq_scales[row * (I / 32) + col0 / 32] = (uint8_t)(X + 127);
                            uint4* dq = reinterpret_cast<uint4*>(p.oq_data + row * I + col0);
                            dq[0] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
                            dq[1] = make_uint4(w8[4], w8[5], w8[6], w8[7]);
                        } else if (FMT == DS4G_MXFP4) {
                            float m = 0.f;
#pragma unroll
                            for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(h[i]));
                            const int X = mx_shared_exp(m);
                            const float inv = exp2i(-X);
#pragma unroll
                            for (int i = 0; i < 32; i += 2)
                                wq[i >> 3] |= e2m1x2(__fmul_rn(h[i], inv), __fmul_rn(h[i + 1], inv)) << (4 * (i & 7));
                            p.oq_scales[row * (I / 32) + col0 / 32] = (uint8_t)(X + 127);
                        } else {
                            uint32_t sb[2];
#pragma unroll
                            for (int hb = 0; hb < 2; ++hb) {
                                float m = 0.f;
#pragma unroll
                                for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(h[16 * hb + i]));
                                const uint32_t s = ue4m3_encode(__fdiv_rn(m, __fmul_rn(6.0f, gh)));
                                const float ds = ue4m3_value(s);
                                if (ds == 0.0f) {
#pragma unroll
                                    for (int i = 0; i < 16; ++i)
                                        wq[2 * hb + (i >> 3)] |= ((__float_as_uint(h[16 * hb + i]) >> 28) & 8u) << (4 * (i & 7));
                                } else {
                                    // h / (dec(s) g_h) as h times the correctly
                                    // rounded reciprocal (within 1.5 ulp of the
                                    // quotient; a code can then differ from the
                                    // divided one only for a quotient that close
                                    // to a rounding boundary of the E2M1 grid)
                                    const float rcp = __frcp_rn(__fmul_rn(ds, gh));
#pragma unroll
                                    for (int i = 0; i < 16; i += 2)
                                        wq[2 * hb + (i >> 3)] |= e2m1x2(__fmul_rn(h[16 * hb + i], rcp),
                                                                        __fmul_rn(h[16 * hb + i + 1], rcp))
                                                                 << (4 * (i & 7));
                                }
                                sb[hb] = s;
                            }
                            *reinterpret_cast<uint16_t*>(p.oq_scales + row * (I / 16) + col0 / 16) =
                                (uint16_t)(sb[0] | (sb[1] << 8));
                        }
                        if (!fp8_act(FMT))
                            *reinterpret_cast<uint4*>(p.oq_data + row * (I / 2) + col0 / 2) =
                                make_uint4(wq[0], wq[1], wq[2], wq[3]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&tmem_empty[buf]));
        }
    }

    // ---- teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 3)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

}  // namespace tc

// ---- host side -----------------------------------------------------------------
typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static PFN_encodeTiled get_encode()
{
    static PFN_encodeTiled fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_encodeTiled>(ptr);
    }
    return fn;
}

// 2-D map over [rows][K] packed E2M1 codes (K / 2 bytes per row) that lands
// each 128-element box row in shared memory as the 8-bit-per-element layout
// kind::mxf8f6f4 reads for FP4 operands: every 16 codes (8 bytes) followed by
// an 8-byte gap, so 128 elements fill a 128-byte row (CUDA's
// CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B; needs K % 128 == 0, a 32-byte
// aligned base and a row pitch that is a multiple of 32 bytes), 128-byte
// swizzle, box 128 elements x box_h rows
static bool make_map_fp4_unpacked(CUtensorMap* m, const uint8_t* base, int64_t rows, int64_t K, uint32_t box_h)
{
    PFN_encodeTiled enc = get_encode();
    if (!enc || (reinterpret_cast<uintptr_t>(base) & 31) != 0 || K % 128 != 0 || (K / 2) % 32 != 0) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    cuuint32_t box[2] = {128, box_h};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<uint8_t*>(base), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D byte map over [rows][width] bytes with a box of box_w bytes x box_h rows
static bool make_map(CUtensorMap* m, const uint8_t* base, int64_t rows, int64_t width, uint32_t box_w,
                     uint32_t box_h, bool swizzle)
{
    PFN_encodeTiled enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)width, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)width};
    cuuint32_t box[2] = {box_w, box_h};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int FMT, int EPI, int TBN, int NISS>
static cudaError_t run_tc(const GemmArgs& a, cudaStream_t st)
{
    using C = tc::Cfg<FMT, TBN, NISS>;
    const int blk = (FMT == DS4G_NVFP4) ? 16 : 32;
    const bool fp8 = fp8_act(FMT);
    CUtensorMap ma, mb, msa, msb;
    // activations: 128 bytes of K per box row (256 FP4 or 128 FP8 elements);
    // weights: 256 packed FP4 elements, 128 unpacked FP4 elements next to FP8
    // activations, or 128 FP8 elements
    if (!make_map(&ma, a.a_data, a.S, fp8 ? a.K : a.K / 2, 128, 128, true) ||
        !(FMT == DS4G_MXFP8 ? make_map_fp4_unpacked(&mb, a.w_data, (int64_t)a.E * a.N, a.K, C::HALF)
                            : make_map(&mb, a.w_data, (int64_t)a.E * a.N, FMT == kFmtFp8Fp8 ? a.K : a.K / 2, 128,
                                       C::HALF, true)) ||
        !make_map(&msa, a.a_scales, a.S, a.K / blk, C::SF_ROW, 128, false) ||
        !make_map(&msb, a.w_scales, (int64_t)a.E * a.N, a.K / blk, C::SF_ROW, C::HALF, false))
        return cudaErrorInvalidValue;
    auto kern = tc::k_gemm_tc<FMT, EPI, TBN, NISS>;
    const size_t shm = C::SMEM;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = kNumSMs;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    kern<<<sms, C::THREADS, shm, st>>>(ma, mb, msa, msb, a);
    return cudaGetLastError();
}

// plain and combine epilogues, N % 224 == 0 (FC2, N = 7168): 224-column
// tiles with two accumulators; MXFP4 and FP8 activations with two MMA
// issuers, NVFP4 (whose scale columns do not fit beside them twice) with one
// issuer and the staged epilogue.  Other N: 256-column tiles, one accumulator.
template <int FMT, int EPI>
static cudaError_t run_tc_plain(const GemmArgs& a, cudaStream_t st)
{
    if (a.N % 224 != 0) return run_tc<FMT, EPI, 256, 1>(a, st);
    if constexpr (FMT != DS4G_NVFP4) return run_tc<FMT, EPI, 224, 2>(a, st);
    else return run_tc<FMT, EPI, 224, 1>(a, st);
}

// FC1 + SwiGLU: 96 gate + 96 up columns per tile, two accumulators, two issuers
template <int FMT>
static cudaError_t run_tc_swiglu(const GemmArgs& a, cudaStream_t st)
{
    return run_tc<FMT, DS4G_EPI_SWIGLU_REQUANT, 192, 2>(a, st);
}

bool gemm_tc_supports(int fmt, int64_t K)
{
    // the scale rows are loaded by TMA in 16 (MX, FP8) / 32 (NV) byte boxes,
    // whose row pitch K / block must be a multiple of 16 bytes
    return fmt == DS4G_NVFP4 ? (K % 256 == 0) : (K % 512 == 0);
}

// Column tiles per band of the combine epilogue's tile order: as many as keep
// one band's columns of the fp32 output (T rows) within about 60 MB, half of
// L2, so that a token's k reductions into those columns find them in L2.
// An output that fits in L2 (decode, T = 2048) is one band: expert-major order.
static int combine_band_tiles(const GemmArgs& a, int tbn)
{
    const int64_t T = a.topk > 0 ? a.S / a.topk : a.S;
    const int64_t n_tiles = ceil_div(a.N, tbn);
    const int64_t per_tile = T * tbn * 4;                 // output bytes of one column tile
    int64_t nb = per_tile > 0 ? (int64_t)60000000 / per_tile : n_tiles;
    if (nb < 1) nb = 1;
    return (int)(nb < n_tiles ? nb : n_tiles);
}

// Plain epilogue with few tiles (a dense GEMM of 64 rows: 16 tiles for 148
// SMs): each tile's K range in ksplit equal parts of whole scale stages, the
// largest divisor that keeps the tiles within about one per SM, each part
// adding into the output (zeroed first).  The tile count is bounded from the
// host's row bound (max_rows_per_expert).  1 = no split.
static int plain_ksplit_tc(const GemmArgs& a, int tbn, int sms)
{
    if (a.epilogue != DS4G_EPI_NONE) return 1;
    const int ke = fp8_act(a.fmt) ? 128 : 256, kps = fp8_act(a.fmt) ? 4 : 2;
    const int nks = (int)ceil_div(a.K, ke);
    if (nks % kps != 0) return 1;
    const int64_t rows = a.max_rows > 0 ? a.max_rows : a.S;
    const int64_t est = (a.E < a.S ? a.E : a.S) * ceil_div(rows, tc::BM) * ceil_div(a.N, tbn);
    if (est * 2 > sms) return 1;
    int best = 1;
    for (int q = 2; q <= nks / kps; ++q)
        if ((nks / kps) % q == 0 && est * q <= sms) best = q;
    return best;
}

cudaError_t launch_gemm_tc(const GemmArgs& a_in, cudaStream_t st)
{
    if (a_in.S == 0) return cudaSuccess;
    if (a_in.E > tc::kMaxE || !gemm_tc_supports(a_in.fmt, a_in.K)) return cudaErrorInvalidValue;
    GemmArgs a = a_in;
    const int tbn = a.N % 224 == 0 ? 224 : 256;
    if (a.epilogue == kEpiCombine) a.band_tiles = combine_band_tiles(a, tbn);
    int dev = 0, sms = kNumSMs;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    a.ksplit = plain_ksplit_tc(a, tbn, sms);
    if (a.ksplit > 1) {
        cudaError_t e = cudaMemsetAsync(a.out, 0, sizeof(float) * (size_t)a.S * a.N, st);
        if (e != cudaSuccess) return e;
    }
    if (a.fmt == DS4G_MXFP8)
        return a.epilogue == DS4G_EPI_NONE ? run_tc_plain<DS4G_MXFP8, DS4G_EPI_NONE>(a, st)
             : a.epilogue == kEpiCombine   ? run_tc_plain<DS4G_MXFP8, kEpiCombine>(a, st)
                                           : run_tc_swiglu<DS4G_MXFP8>(a, st);
    if (a.fmt == kFmtFp8Fp8)
        return a.epilogue == DS4G_EPI_NONE ? run_tc_plain<kFmtFp8Fp8, DS4G_EPI_NONE>(a, st)
             : a.epilogue == kEpiCombine   ? run_tc_plain<kFmtFp8Fp8, kEpiCombine>(a, st)
                                           : run_tc_swiglu<kFmtFp8Fp8>(a, st);
    if (a.fmt == DS4G_MXFP4)
        return a.epilogue == DS4G_EPI_NONE ? run_tc_plain<DS4G_MXFP4, DS4G_EPI_NONE>(a, st)
             : a.epilogue == kEpiCombine   ? run_tc_plain<DS4G_MXFP4, kEpiCombine>(a, st)
                                           : run_tc_swiglu<DS4G_MXFP4>(a, st);
    return a.epilogue == DS4G_EPI_NONE ? run_tc_plain<DS4G_NVFP4, DS4G_EPI_NONE>(a, st)
         : a.epilogue == kEpiCombine   ? run_tc_plain<DS4G_NVFP4, kEpiCombine>(a, st)
                                       : run_tc_swiglu<DS4G_NVFP4>(a, st);
}

}  // namespace ds4g
