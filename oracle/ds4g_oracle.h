/*
 * ds4g_oracle.h -- the CPU oracle for the block-scaled FP4 routed-expert MoE
 * FFN.  TEST INFRASTRUCTURE ONLY: only the tests, the package's smoke check
 * and the bench's CPU-baseline leg may load it.  It shares no code, header,
 * table or constant with the CUDA library; it is a plain, slow, fp64 restatement
 * of what the path computes, written so that each step can be checked against
 * the pages by eye.
 *
 * Sources ("the pages"):
 *   [P1] "DGX Spark native FP4 matrix instructions: how DwarfStar uses
 *        Blackwell" -- sec. 1 (what the FP4 instruction is: E2M1 = 1 sign,
 *        2 exponent, 1 mantissa bit, UE8M0 block scale; NVFP4 = kind::mxf4nvf4
 *        with UE4M3 scales, scale_vec::4X), sec. 2 (MoE routing; routed-expert
 *        weights and activations stay FP4; batched expert GEMM), sec. 3 (the
 *        FP4 path needs K to be a multiple of 64 or it reports an error).
 *   [P2] "[DeepSeek V4] Triton FP4 optimisation in practice" -- "What is the
 *        FP4 MoE GEMM" (256 experts, 6 active per token, 2 FC per expert),
 *        "Step 0" (m_grouped_fp8_fp4_gemm_nt_contiguous: rows grouped by
 *        expert), "Step 2" (packed FP4: even column = low nibble, odd column =
 *        high nibble).
 *   [P3] "Moore Threads full-link adaptation of DeepSeek-V4" -- fused
 *        SwiGLU + quantisation pattern; MoE routing / dispatch / combine.
 *   [P5] "ik_llama.cpp PR #454: FP8 GGUF creation" -- sec. 5 (the 16 FP4
 *        values map losslessly onto a 16-entry lookup table).
 *   [OCP] OCP Microscaling Formats (MX) Specification v1.0 -- the shared-scale
 *        rule X = 2^(floor(log2(amax)) - emax_elem), emax_elem = 2 for E2M1;
 *        the pages name UE8M0 but not the rule, the workload names the rule.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - E2M1 rounding is round-to-nearest, ties to the even code, |y| > 6
 *     saturates to 6; the code's sign bit is the input's sign bit (so -0 and
 *     small negatives give 0x8).
 *   - An all-zero MX block gets scale byte 0 (shared exponent clamped to -127).
 *   - NVFP4 scale math is fp32: g = amax/(6*448) (g = 1 if amax = 0),
 *     s = E4M3_RNE(amax_b / fp32(6*g)) saturating at 448,
 *     q = E2M1_RNE(v / fp32(dec(s)*g)); dec(s) = 0 gives all-zero codes.
 *   - Routing selects on the raw fp32 logits (ties -> lower expert index),
 *     outputs in descending order, weights = softmax restricted to the k
 *     selected (they sum to 1).
 *   - Permutation is stable: within an expert, ascending slot id s = t*k + j.
 *   - FC1 output columns [0, I) are the gate, [I, 2I) the up projection;
 *     h = silu(gate) * up, silu(x) = x / (1 + e^-x), computed in fp64 from the
 *     fp32-rounded FC1 outputs and rounded to fp32.
 *   - Combine sums w[t][j] * Y2[row(t, j)] over j = 0..k-1.
 */
#ifndef DS4G_ORACLE_H
#define DS4G_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* formats: 0 = MXFP4 (E2M1 + UE8M0 per 32), 1 = NVFP4 (E2M1 + UE4M3 per 16
 * + tensor scale), 2 = MXFP8 (E4M3 + UE8M0 per 32, one byte per element;
 * the FP8 activations of the FP8 x FP4 variant) */

/* element / scale codecs */
double orc_e2m1_decode(int code);
int orc_e2m1_encode(double y);          /* RNE on the E2M1 grid, sign kept, saturating */
double orc_ue8m0_decode(int b);
double orc_ue4m3_decode(int b);         /* unsigned E4M3: bias 7, subnormal m*2^-9 */
int orc_ue4m3_encode(double r);         /* RNE over the 127 finite codes, saturating at 448 */
int orc_lut_decode_check(void);         /* 16-entry-table decode == field decode, 0 = ok */
double orc_e4m3_decode(int code);       /* E4M3: bias 7, subnormal m*2^-9, 0x7F / 0xFF NaN, max 448 */
int orc_e4m3_encode(double y);          /* RNE over the finite codes, sign kept, saturating at 448 */

/* quantisation of fp32 values (bf16 inputs are widened exactly first) */
void orc_quantize_mx(const float* x, int64_t rows, int64_t K, uint8_t* data, uint8_t* scales);
void orc_quantize_nv(const float* x, int64_t rows, int64_t K, const float* g_in,
                     uint8_t* data, uint8_t* scales, float* g_out);
void orc_quantize_mx8(const float* x, int64_t rows, int64_t K, uint8_t* data, uint8_t* scales);
void orc_dequantize(const uint8_t* data, const uint8_t* scales, int fmt, double g,
                    int64_t rows, int64_t K, double* out);

/* routing */
void orc_route_topk(const float* logits, int T, int E, int k, int32_t* idx, double* w);

/* permutation */
void orc_moe_permute(const int32_t* idx, int T, int k, int E, int32_t* offsets,
                     int32_t* row_to_slot, int32_t* slot_to_row);
void orc_gather_rows(const uint8_t* src_data, const uint8_t* src_scales, int64_t K, int fmt,
                     const int32_t* row_to_slot, int64_t S, int k,
                     uint8_t* dst_data, uint8_t* dst_scales);

/* grouped GEMM: out[r][n] = sum_k deq(A[r][k]) * deq(W[e*N+n][k]) (* g_a*g_w for NV).
 * Rows are restricted to [row_begin, row_end) and columns to [n_begin, n_end)
 * so that large problems can be checked on samples; abssum (nullable) gets
 * sum_k |a_k * w_k| per element. out / abssum are [S][N]-indexed. */
void orc_grouped_gemm(const uint8_t* a_data, const uint8_t* a_scales, double g_a,
                      const int32_t* offsets, int E,
                      const uint8_t* w_data, const uint8_t* w_scales, double g_w,
                      int N, int64_t K, int fmt,
                      int64_t row_begin, int64_t row_end, int n_begin, int n_end,
                      double* out, double* abssum);

/* one expert, explicit rows: out[i][n] for the listed rows of A against
 * expert e's weights (w_e points at that expert's first weight row). */
void orc_expert_gemm_rows(const uint8_t* a_data, const uint8_t* a_scales, double g_a,
                          const int64_t* rows, int64_t nrows,
                          const uint8_t* w_e_data, const uint8_t* w_e_scales, double g_w,
                          int n_begin, int n_end, int64_t K, int fmt,
                          double* out, double* abssum);

/* the same with the activations and the weights each in its own format
 * (FP8 activations x FP4 weights: a_fmt 2, w_fmt 0) */
void orc_expert_gemm_rows_mixed(const uint8_t* a_data, const uint8_t* a_scales, double g_a, int a_fmt,
                                const int64_t* rows, int64_t nrows,
                                const uint8_t* w_e_data, const uint8_t* w_e_scales, double g_w, int w_fmt,
                                int n_begin, int n_end, int64_t K, double* out, double* abssum);

/* SwiGLU on fp32 FC1 outputs: h[r][i] = fp32(silu(y1[r][i]) * y1[r][I + i]) */
void orc_swiglu(const float* y1, int64_t rows, int I, float* h);

/* combine: out[t][c] = sum_j w[t][j] * y2[slot_to_row[t*k+j]][c] */
void orc_moe_combine(const double* y2, const int32_t* slot_to_row, const double* w,
                     int T, int k, int d, double* out);

#ifdef __cplusplus
}
#endif

#endif /* DS4G_ORACLE_H */
