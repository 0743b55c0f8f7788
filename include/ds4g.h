/*
 * ds4g.h -- C ABI of the block-scaled FP4 routed-expert MoE FFN library
 * (libds4g.so, sm_100a only).
 *
 * One MoE layer is, in order:
 *   ds4g_route_topk       top-k routing of each token over E experts
 *   ds4g_quantize_mx      activations -> MXFP4 / NVFP4 (on the fly)
 *   ds4g_moe_permute      expert-contiguous reordering of the quantised rows
 *     (ds4g_moe_dispatch does these three in one call)
 *   ds4g_grouped_gemm_fp4 FC1 (gate+up), optionally with the SwiGLU +
 *                         requantisation epilogue fused
 *   ds4g_swiglu_requant   the same epilogue as a separate step
 *   ds4g_grouped_gemm_fp4 FC2
 *   ds4g_moe_combine      routing-weighted sum of each token's k expert rows
 *     (ds4g_grouped_gemm_fp4_combine does FC2 and the combine in one call;
 *      ds4g_grouped_gemm_fp4_combine_chained does it overlapping FC1's end)
 *
 * Sources: "DGX Spark native FP4 matrix instructions: how DwarfStar uses
 * Blackwell" (sec. 1 FP4 formats and the block-scaled MMA, sec. 2 MoE
 * routing and batched expert GEMM with FP4 weights and activations, sec. 3
 * the K % 64 shape check with an error instead of a silent fallback);
 * "[DeepSeek V4] Triton FP4 optimisation in practice" ("What is the FP4 MoE
 * GEMM": 256 experts, 6 active, 2 FC per expert; "Step 0": the grouped
 * contiguous GEMM; "Step 2": packed FP4, even column = low nibble);
 * "Moore Threads full-link adaptation of DeepSeek-V4" (fused SwiGLU +
 * quantisation; MoE routing / combine).
 *
 * Conventions (every entry point):
 *   - All pointers are DEVICE pointers unless stated otherwise; the caller
 *     allocates and owns all memory.  The library never allocates device
 *     memory; scratch space comes from a caller-provided workspace whose size
 *     the matching *_workspace_bytes() call returns.
 *   - Calls are asynchronous on the given stream (cudaStream_t passed as
 *     void*; NULL = the legacy default stream).
 *   - Arguments and shapes are validated on the host before any launch; a bad
 *     argument returns an error status and launches nothing.  There is no
 *     silent fallback and no CPU path.
 *   - Launch failures return DS4G_ERR_CUDA.  A device-side wait that gives up
 *     (a bounded spin in a persistent kernel) records an error word that
 *     ds4g_check_device() turns into DS4G_ERR_DEVICE.
 *   - Activations and weights must be finite (no NaN / Inf).  Router logits
 *     may hold any value (see ds4g_route_topk).
 */
#ifndef DS4G_H
#define DS4G_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DS4G_OK = 0,
    DS4G_ERR_INVALID_ARG = 1,   /* null pointer, bad enum, misaligned pointer, k > E ... */
    DS4G_ERR_SHAPE = 2,         /* K % 64 != 0 and other shape rules below */
    DS4G_ERR_UNSUPPORTED = 3,   /* device is not sm_100 */
    DS4G_ERR_CUDA = 4,          /* a CUDA runtime / launch error */
    DS4G_ERR_DEVICE = 5,        /* a device-side bounded wait gave up */
    DS4G_ERR_WORKSPACE = 6      /* workspace missing or too small */
} ds4g_status;

typedef enum { DS4G_MXFP4 = 0, DS4G_NVFP4 = 1, DS4G_MXFP8 = 2 } ds4g_fmt;
typedef enum { DS4G_BF16 = 0, DS4G_F32 = 1 } ds4g_dtype;
typedef enum { DS4G_EPI_NONE = 0, DS4G_EPI_SWIGLU_REQUANT = 1 } ds4g_epilogue;

/* A block-scaled tensor of `rows` x `K` elements (row-major along K).
 *   data   MXFP4 / NVFP4: [rows][K/2] bytes of E2M1 codes (sign, 2 exponent,
 *          1 mantissa bit), element 2i in the low nibble of byte i, 2i+1 in
 *          the high nibble.  MXFP8 (FP8 activations of the FP8 x FP4
 *          variant): [rows][K] bytes of E4M3 codes (sign, 4 exponent bits
 *          with bias 7, 3 mantissa bits; max 448, no infinities).
 *   scales [rows][K/32] UE8M0 bytes (MXFP4, MXFP8: value 2^(b-127)) or
 *          [rows][K/16] UE4M3 bytes (NVFP4: unsigned E4M3, max 448).
 *   g      NVFP4 only: one fp32 tensor scale (device); element value =
 *          E2M1 * UE4M3 * g.  Ignored (may be NULL) otherwise.
 *   data and scales must be 16-byte aligned. */
typedef struct {
    uint8_t* data;
    uint8_t* scales;
    float* g;
    int64_t rows;
    int64_t K;
    int32_t fmt;   /* ds4g_fmt */
    int32_t reserved;
} ds4g_fp4;

/* Human-readable name of a status code (static string). */
const char* ds4g_status_str(ds4g_status s);

/* DS4G_OK when the current device is sm_100 (B200 class). */
ds4g_status ds4g_device_supported(void);

/* Synchronises `stream`, then reports (and clears) the device error word:
 * DS4G_ERR_DEVICE if a bounded device wait gave up since the last check. */
ds4g_status ds4g_check_device(void* stream);

/* ---------------------------------------------------------------------------
 * Quantise rows of x (bf16 or fp32, [rows][K]) to MXFP4 or NVFP4.
 *   MXFP4 ("DGX Spark native FP4 ..." sec. 1, E2M1 + UE8M0 per 32): per
 *     block, X = floor(log2(amax)) - 2 clamped to [-127, 127] (the OCP MX
 *     rule), scale byte X + 127, code = E2M1 round-to-nearest-even of
 *     v * 2^-X, saturating at 6, sign bit kept.
 *   MXFP8 (the FP8 activations of "[DeepSeek V4] Triton FP4 ..." "Step 0",
 *     m_grouped_fp8_fp4_gemm_nt_contiguous): per block of 32, X =
 *     floor(log2(amax)) - 8 clamped to [-127, 127], scale byte X + 127, code
 *     = E4M3 round-to-nearest-even of v * 2^-X, saturating at 448, sign kept.
 *   NVFP4 (sec. 1, kind::mxf4nvf4: E2M1 + UE4M3 per 16) with a tensor scale
 *     g: g = *g_in if g_in != NULL, else amax(x) / 2688 computed on the
 *     device (1 if amax is 0) and written to out->g; per block
 *     s = E4M3_RNE(amax_b / fp32(6 g)) saturating at 448, code =
 *     E2M1_RNE(v / fp32(dec(s) g)); all fp32, IEEE rounding.
 * K % 64 == 0 (DS4G_ERR_SHAPE otherwise).  out->rows/K/fmt must match.
 * Workspace: ds4g_quantize_workspace_bytes(fmt, g_in != NULL) bytes (16 for
 * NVFP4 without g_in, else 0). */
size_t ds4g_quantize_workspace_bytes(int fmt, int has_g_in);
ds4g_status ds4g_quantize_mx(const void* x, int dtype, int64_t rows, int64_t K, int fmt,
                             const float* g_in, ds4g_fp4* out,
                             void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Top-k routing ("DGX Spark native FP4 ..." sec. 2; "[DeepSeek V4] Triton
 * FP4 ..." "What is the FP4 MoE GEMM").  For each token t of logits [T][E]
 * (fp32): the k largest logits, ties to the lower expert index, written in
 * descending order to idx [T][k] (int32); weights w [T][k] (fp32) are the
 * softmax over the k selected logits (they sum to 1).  1 <= k <= min(E, 32),
 * E <= 1024.  Non-finite logits: a NaN ranks below every number, as -inf
 * does, and a pick equal to the token's maximum has softmax factor 1 (the
 * limit when that maximum is +inf or every pick is -inf), so idx always
 * holds k distinct experts in [0, E). */
ds4g_status ds4g_route_topk(const float* logits, int T, int E, int k, int32_t* idx, float* w,
                            void* stream);

/* ---------------------------------------------------------------------------
 * Expert-contiguous permutation ("[DeepSeek V4] Triton FP4 ..." "Step 0":
 * rows grouped per expert).  From idx [T][k]:
 *   offsets [E+1]   exclusive prefix sum of the per-expert slot counts
 *   row_to_slot [S] slot s = t*k + j of permuted row r; within an expert the
 *                   slots are in ascending order (stable)
 *   slot_to_row [S] the inverse
 *   a_perm          row r = row t = row_to_slot[r] / k of x_q (data and
 *                   scales copied; for NVFP4 a_perm->g receives x_q->g)
 * S = T*k; a_perm->rows must be S, same K and fmt as x_q.  Every idx entry
 * must lie in [0, E) (ds4g_route_topk's always do); the device does not
 * check them, and an entry outside that range indexes out of bounds.
 * Workspace: ds4g_permute_workspace_bytes(T, k, E). */
size_t ds4g_permute_workspace_bytes(int T, int k, int E);
ds4g_status ds4g_moe_permute(const int32_t* idx, int T, int k, int E, const ds4g_fp4* x_q,
                             int32_t* offsets, int32_t* row_to_slot, int32_t* slot_to_row,
                             ds4g_fp4* a_perm, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Dispatch: ds4g_route_topk, ds4g_quantize_mx and ds4g_moe_permute as one call
 * (the routing, quantisation and permutation steps of the pages cited at each
 * of those three).  Same arguments and the same results, bit for bit, as
 *   ds4g_route_topk(logits, T, E, k, idx, w);
 *   ds4g_quantize_mx(x, dtype, T, x_q->K, fmt, g_in, x_q, ...);
 *   ds4g_moe_permute(idx, T, k, E, x_q, offsets, row_to_slot, slot_to_row, a_perm, ...);
 * x: [T][x_q->K] bf16 or fp32 (16-byte aligned).  x_q: [T] rows, a_perm:
 * [T*k] rows, both of format fmt (NVFP4: both need g; with g_in NULL the
 * tensor scale is derived from amax |x| as ds4g_quantize_mx does).
 * Up to 512 slots (T*k) one kernel does all three steps (decode batches);
 * larger batches run the separate calls' kernels.  Limits as the separate
 * calls: E <= 1024, 1 <= k <= min(E, 32), K % 64 == 0.  fmt MXFP4 or NVFP4
 * (FP8 activations take the three separate calls).
 * Workspace: ds4g_dispatch_workspace_bytes(T, k, E, fmt, g_in != NULL), 16-byte
 * aligned, owned by the caller. */
size_t ds4g_dispatch_workspace_bytes(int T, int k, int E, int fmt, int has_g_in);
ds4g_status ds4g_moe_dispatch(const float* logits, const void* x, int dtype, int T, int E, int k, int fmt,
                              const float* g_in, int32_t* idx, float* w, ds4g_fp4* x_q, int32_t* offsets,
                              int32_t* row_to_slot, int32_t* slot_to_row, ds4g_fp4* a_perm,
                              void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Grouped block-scaled FP4 GEMM ("DGX Spark native FP4 ..." sec. 1-2; the
 * grouped contiguous GEMM of "[DeepSeek V4] Triton FP4 ..." "Step 0").
 * For every expert e and every row r of its segment [offsets[e],
 * offsets[e+1]) of a (a->rows = S rows, K columns):
 *   y[r][n] = sum_k deq(a[r][k]) * deq(w[e*N + n][k])   (fp32 accumulate;
 *             NVFP4: times a->g[0] * w->g[e])
 * w has E*N rows of K columns, same fmt as a; for NVFP4 w->g holds one fp32
 * tensor scale per expert ([E] floats, each expert's weight matrix being its
 * own tensor).  FP8 activations (a->fmt DS4G_MXFP8, the FP8 x FP4 GEMM of
 * "[DeepSeek V4] Triton FP4 ..." "Step 0") take MXFP4 weights (routed
 * experts) or MXFP8 weights (a shared expert kept in 8 bits, "DGX Spark
 * native FP4 ..." sec. 2); with them SWIGLU_REQUANT writes h as MXFP8 (the
 * "SwiGLU + FP8 quant" step of "Moore Threads ...").
 * epilogue DS4G_EPI_NONE: out = y, fp32 [S][N].
 * epilogue DS4G_EPI_SWIGLU_REQUANT (FC1 with N = 2I): columns [0, I) are the
 *   gate and [I, 2I) the up projection; h = silu(gate) * up (fp32,
 *   silu(x) = x / (1 + e^-x)) is quantised to out_q ([S][I], same rule as
 *   ds4g_quantize_mx; for NVFP4 *out_q->g is the caller's static tensor
 *   scale of h, read, not written); h_debug (nullable) receives h fp32 [S][I].
 * max_rows_per_expert: an upper bound on any segment length (T for top-k
 *   routing); it selects the kernel:
 *   <= 16 rows, K a multiple of 512 (MXFP4) / 256 (NVFP4), N % 128 == 0
 *     (NONE) or I % 64 == 0 (SWIGLU_REQUANT): tensor-core kernel with the
 *     weights as the MMA's M side (decode); with SWIGLU_REQUANT and at most
 *     about two weight tiles per SM (min(E, rows) x I / 64 <= 296) each
 *     tile's K range is split over a CTA pair whose follower sends its
 *     partial sums to the leader.  This kernel is launched with programmatic
 *     stream serialization: it may start while the previous kernel on the
 *     stream ends, and reads no input before that kernel has finished;
 *   > 16 rows and the same K rule, N % 224 == 0 (NONE): tensor-core kernel
 *     with 128-row x 224-column tiles and two accumulators (the epilogue of
 *     one tile overlaps the next tile's MMAs); else N % 256 == 0 (NONE):
 *     128-row x 256-column tiles; SWIGLU_REQUANT with I % 32 == 0: 128-row
 *     tiles of 96 gate + 96 up columns (the last one ragged), two
 *     accumulators;
 *   otherwise: a dp4a weight-streaming kernel (any segment length).
 *   FP8 activations always take the 128-row tensor-core kernel
 *   (kind::mxf8f6f4): K % 512 == 0 and the N rule above, else DS4G_ERR_SHAPE.
 *   With NONE and few tiles for the SMs (a dense GEMM of a few rows, e.g.
 *   M = 1 or 64 at N = 4096) both tensor-core kernels split each tile's K
 *   range into equal parts that add their partial sums into out with fp32
 *   atomics (out is zeroed first on the stream): the result may then differ
 *   in its last bits from run to run.  Chosen from the shapes and
 *   max_rows_per_expert alone.
 * Shapes: K % 64 == 0; NONE needs N % 64 == 0 unless a tensor-core kernel
 *   takes the call; SWIGLU_REQUANT needs I % 32 == 0.  offsets[E] must
 *   equal S. */
ds4g_status ds4g_grouped_gemm_fp4(const ds4g_fp4* a, const int32_t* offsets, int E,
                                  int max_rows_per_expert, const ds4g_fp4* w, int N, int epilogue,
                                  float* out, ds4g_fp4* out_q, float* h_debug, void* stream);

/* ---------------------------------------------------------------------------
 * FC2 with the combine fused ("Moore Threads ..." MoE combine, folded into
 * the GEMM's epilogue): the same grouped GEMM as ds4g_grouped_gemm_fp4 (a has
 * S = T*k rows), but instead of storing y[r][:] each row adds
 * route_w[s] * y[r][:] into out[s / k][:], s = row_to_slot[r].  out fp32
 * [T][N] is zeroed by the call first.  The adds are fp32 atomics, so the
 * order in which a token's k rows are summed is not fixed (results can
 * differ in the last bits from run to run; ds4g_moe_combine is the
 * deterministic alternative).  Kernel choice and shapes as for
 * ds4g_grouped_gemm_fp4 with DS4G_EPI_NONE.  When the output is larger than
 * about half of L2 (T * N * 4 bytes over ~60 MB, prefill sizes) the
 * tensor-core kernel walks its tiles in bands of output columns, all experts
 * of a band before the next, so that a token's k additions to those columns
 * meet in L2. */
ds4g_status ds4g_grouped_gemm_fp4_combine(const ds4g_fp4* a, const int32_t* offsets, int E,
                                          int max_rows_per_expert, const ds4g_fp4* w, int N,
                                          const int32_t* row_to_slot, const float* route_w, int T, int k,
                                          float* out, void* stream);

/* ---------------------------------------------------------------------------
 * ds4g_grouped_gemm_fp4_combine chained to the kernel just before it on the
 * stream (normally the FC1 call that writes a):
 *   - out is NOT zeroed: the weighted rows are added to what it holds (zero
 *     it before the FC1 call, e.g. with ds4g_zero_fill, or leave in it what
 *     the routed experts' sum should be added to);
 *   - with decode-sized segments the launch may start while that previous
 *     kernel still runs, so that the FC2 weights stream in while its last
 *     tiles finish.  The kernel waits for the previous kernel (programmatic
 *     dependent launch, griddepcontrol.wait) before it reads a, row_to_slot,
 *     route_w or out; it reads offsets (and w) before that wait.  So a may be
 *     written by the previous kernel, and every other input must be written
 *     by work that comes before that previous kernel on the stream.  The
 *     layer's own sequence -- ds4g_moe_dispatch (offsets, row_to_slot,
 *     route_w), then FC1 (a = h), then this call -- satisfies it: each
 *     decode-kernel launch of this library releases the next kernel on the
 *     stream only after it has itself waited for its predecessor, so when
 *     this kernel starts, everything before FC1 has completed.
 * Other shapes launch the same kernels as ds4g_grouped_gemm_fp4_combine, in
 * stream order.  Arguments, results within the same bound and errors as
 * ds4g_grouped_gemm_fp4_combine. */
ds4g_status ds4g_grouped_gemm_fp4_combine_chained(const ds4g_fp4* a, const int32_t* offsets, int E,
                                                  int max_rows_per_expert, const ds4g_fp4* w, int N,
                                                  const int32_t* row_to_slot, const float* route_w, int T, int k,
                                                  float* out, void* stream);

/* ---------------------------------------------------------------------------
 * The decode FFN in one launch ("[DeepSeek V4] Triton FP4 ...", "Why Triton
 * is the only way on SM120": launch overhead at decode sizes; the fused
 * SwiGLU + quantisation of "Moore Threads ..."): the work of
 *   ds4g_grouped_gemm_fp4(a, offsets, E, max_rows_per_expert, w1, 2I,
 *                         DS4G_EPI_SWIGLU_REQUANT, NULL, h_q, NULL) followed by
 *   ds4g_grouped_gemm_fp4_combine_chained(h_q, offsets, E, max_rows_per_expert,
 *                                         w2, d, row_to_slot, route_w, T, k, out)
 * as one persistent kernel: each expert's FC2 tiles start as soon as all of
 * that expert's FC1 tiles have stored their h rows (a per-expert completion
 * counter; every wait on one is bounded), so FC2's weight streaming overlaps
 * the end of FC1 with no launch between them.  a: [T*k] rows of d, fmt MXFP4
 * or NVFP4; w1: E*2I rows of d and w2: E*d rows of I, same fmt; h_q: [T*k]
 * rows of I (written; NVFP4: its g is the caller's static tensor scale of h,
 * read); out: fp32 [T][d], added into (zero it before the call, as for the
 * chained combine).  counters: int32 [E + 1] device memory owned by the
 * caller, all zero on entry; the call leaves them zero (its last CTA resets
 * them), also after a device-side wait gave up.  Calls that share a counter
 * array must not overlap on the GPU.  Decode shapes only:
 * max_rows_per_expert <= 16 and the decode kernel's tiling for both GEMMs
 * (MXFP4: d and I multiples of 512, NVFP4: of 256; I % 64 == 0, d % 128 ==
 * 0), E <= 512; otherwise DS4G_ERR_SHAPE.  Launched with programmatic stream
 * serialization like the decode kernel; its CTAs wait on one another, and
 * the grid is sized to be resident on the device at once (one CTA per SM). */
ds4g_status ds4g_moe_ffn_fp4(const ds4g_fp4* a, const int32_t* offsets, int E, int max_rows_per_expert,
                             const ds4g_fp4* w1, const ds4g_fp4* w2, int d, int I, ds4g_fp4* h_q,
                             const int32_t* row_to_slot, const float* route_w, int T, int k, float* out,
                             int32_t* counters, void* stream);

/* ---------------------------------------------------------------------------
 * Segment ids, for expert parallelism across GPUs ("Moore Threads ..." MoE
 * dispatch / combine; "DGX Spark native FP4 ..." sec. 6, several GPUs): a
 * receiving rank holds rows grouped by source rank and, within a source, by
 * its own expert; offsets [nseg + 1] (int32, device, non-decreasing) are
 * those groups' boundaries.  Writes out[r] = s % modulo for every row r of
 * [0, rows), s the group holding row offsets[0] + r (with modulo = experts
 * per rank: the row's local expert).  rows must be offsets[nseg] -
 * offsets[0]; rows beyond the last boundary get the last group. */
ds4g_status ds4g_segment_ids(const int32_t* offsets, int nseg, int modulo, int64_t rows, int32_t* out,
                             void* stream);

/* Zero-fills bytes of device memory at p on the stream (cudaMemsetAsync). */
ds4g_status ds4g_zero_fill(void* p, size_t bytes, void* stream);

/* ---------------------------------------------------------------------------
 * The SwiGLU + requantisation epilogue as its own step ("Moore Threads ..."
 * fused SwiGLU + quant pattern): y1 fp32 [rows][2I] -> h_q (fmt, [rows][I]);
 * h_debug (nullable) receives h fp32.  For NVFP4 *h_q->g is the static
 * tensor scale (input).  I % 32 == 0; fmt MXFP4 or NVFP4 (with FP8
 * activations h is requantised only in FC1's fused epilogue). */
ds4g_status ds4g_swiglu_requant(const float* y1, int64_t rows, int I, int fmt, ds4g_fp4* h_q,
                                float* h_debug, void* stream);

/* ---------------------------------------------------------------------------
 * Combine ("Moore Threads ..." MoE combine): out[t][c] =
 *   sum_{j=0..k-1} w[t][j] * y2[slot_to_row[t*k + j]][c]   (fp32, j order)
 * y2 fp32 [T*k][d], w fp32 [T][k], out fp32 [T][d]; d % 4 == 0. */
ds4g_status ds4g_moe_combine(const float* y2, const int32_t* slot_to_row, const float* w, int T,
                             int k, int d, float* out, void* stream);

/* ---------------------------------------------------------------------------
 * ds4g_moe_permute_static: ds4g_moe_permute without a caller workspace, for
 * callers that cannot allocate device memory at all (a runtime that owns all
 * device memory through its own pool, a plug-in restricted to the buffers it
 * is handed).  The pages have no counterpart; this is a library convenience.
 * Arguments, results and errors are those of ds4g_moe_permute.  The scratch is
 * a file-scope device array of ds4g_permute_static_max_bytes() bytes (256 KiB)
 * that every GPU loading the library keeps until the process exits; a problem
 * whose ds4g_permute_workspace_bytes(T, k, E) exceeds it returns
 * DS4G_ERR_WORKSPACE.  The first call on a device looks the array's device
 * address up for that device (make that first call before any stream
 * capture); a lookup that fails returns DS4G_ERR_CUDA and is tried again on
 * the next call.  All calls share the one array: calls that overlap on the
 * GPU (concurrent streams, or several host threads) race on it and must be
 * serialised by the caller. */
size_t ds4g_permute_static_max_bytes(void);
ds4g_status ds4g_moe_permute_static(const int32_t* idx, int T, int k, int E, const ds4g_fp4* x_q,
                                    int32_t* offsets, int32_t* row_to_slot, int32_t* slot_to_row,
                                    ds4g_fp4* a_perm, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DS4G_H */
