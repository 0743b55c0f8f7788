/*
 * ds4g_oracle.c -- CPU oracle (test infrastructure; see ds4g_oracle.h for the
 * sources and the readings).  Plain C11, fp64 unless a step is defined in
 * fp32 by the reading it follows.  Nothing here is shared with the CUDA path.
 */
#include "ds4g_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_MX = 0, ORC_NV = 1, ORC_MX8 = 2 };

/* bytes of one row of K elements, and its block length, per format */
static int64_t row_bytes(int fmt, int64_t K) { return fmt == ORC_MX8 ? K : K / 2; }
static int block_of(int fmt) { return fmt == ORC_NV ? 16 : 32; }

/* ---------------------------------------------------------------------------
 * E2M1 element, [P1] sec. 1: 1 sign bit, 2 exponent bits, 1 mantissa bit,
 * code = s*8 + e*2 + m.  Exponent bias 1: e = 0 is the subnormal m * 0.5,
 * e > 0 is 2^(e-1) * (1 + m/2).  This gives +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}.
 * ------------------------------------------------------------------------- */
double orc_e2m1_decode(int code)
{
    int s = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* Nearest E2M1 value to y; on an exact tie the even code wins (round to
 * nearest even); beyond 6 the nearest value is 6 (saturation).  The sign bit
 * of the code is the sign bit of y. */
int orc_e2m1_encode(double y)
{
    /* the 8 non-negative grid values, from the field decode above */
    static const double grid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    int sign = signbit(y) ? 8 : 0;
    double a = fabs(y);
    if (a >= 6.0) return sign | 7;    /* 6 is the nearest value to anything beyond it */
    int best = 0;
    double best_d = INFINITY;
    for (int c = 0; c < 8; ++c) {
        double d = fabs(a - grid[c]);
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return sign | best;
}

/* UE8M0 scale, [P1] sec. 1: an unsigned power-of-two exponent, 2^(b-127);
 * b = 255 is NaN and is never produced. */
double orc_ue8m0_decode(int b)
{
    if (b == 255) return NAN;
    return ldexp(1.0, b - 127);
}

/* UE4M3 scale, [P1] sec. 1 (NVFP4): E4M3 with the sign bit zero; bias 7,
 * e = 0 subnormal m * 2^-9, largest finite 0x7E = 448, 0x7F is NaN. */
double orc_ue4m3_decode(int b)
{
    b &= 0x7F;
    if (b == 0x7F) return NAN;
    int e = b >> 3, m = b & 7;
    if (e == 0) return ldexp((double)m, -9);
    return ldexp(1.0 + m / 8.0, e - 7);
}

/* Nearest finite UE4M3 value to r >= 0, ties to the even code, saturating. */
int orc_ue4m3_encode(double r)
{
    if (r >= 448.0) return 0x7E;      /* saturation, as for the elements */
    int best = 0;
    double best_d = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double d = fabs(r - orc_ue4m3_decode(c));
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return best;
}

/* [P5] sec. 5: the 16 FP4 codes can be decoded through a 16-entry lookup
 * table with no loss.  Build the table once and compare every code with the
 * field decode (including the sign of zero). */
int orc_lut_decode_check(void)
{
    double lut[16];
    for (int c = 0; c < 16; ++c) lut[c] = orc_e2m1_decode(c);
    for (int c = 0; c < 16; ++c) {
        double a = lut[c], b = orc_e2m1_decode(c);
        if (a != b || signbit(a) != signbit(b)) return 1;
        if (orc_e2m1_encode(a) != c) return 2;
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * E4M3 element (the FP8 activations of [P2] "Step 0",
 * m_grouped_fp8_fp4_gemm_nt_contiguous: FP8 activations x FP4 weights; the
 * E4M3 format of [P5] sec. 1: 4 exponent bits, 3 mantissa bits): code =
 * s*128 + e*8 + m, bias 7; e = 0 is the subnormal m * 2^-9, otherwise
 * 2^(e-7) * (1 + m/8); e = 15, m = 7 is NaN (no infinities), so the largest
 * finite magnitude is 0x7E = 448.
 * ------------------------------------------------------------------------- */
double orc_e4m3_decode(int code)
{
    int s = (code >> 7) & 1;
    int e = (code >> 3) & 15;
    int m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Nearest finite E4M3 value to y, ties to the even code, beyond 448 the
 * nearest finite value (saturation); the code's sign bit is y's sign bit. */
int orc_e4m3_encode(double y)
{
    int sign = signbit(y) ? 0x80 : 0;
    double a = fabs(y);
    if (a >= 448.0) return sign | 0x7E;   /* 448 is the nearest finite value to anything beyond it */
    int best = 0;
    double best_d = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double d = fabs(a - orc_e4m3_decode(c));
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return sign | best;
}

/* packed byte layout, [P2] "Step 2": element k sits in byte k/2, even k in
 * the low nibble, odd k in the high nibble */
static void put_nibble(uint8_t* row, int64_t k, int code)
{
    if (k & 1) row[k >> 1] = (uint8_t)((row[k >> 1] & 0x0F) | (code << 4));
    else row[k >> 1] = (uint8_t)((row[k >> 1] & 0xF0) | (code & 0x0F));
}

static int get_nibble(const uint8_t* row, int64_t k)
{
    return (k & 1) ? (row[k >> 1] >> 4) : (row[k >> 1] & 0x0F);
}

/* ---------------------------------------------------------------------------
 * MXFP4 quantisation, [OCP] sec. 6.3 with the E2M1 element of [P1] sec. 1:
 * per block of 32 along K, shared exponent X = floor(log2(amax)) - 2
 * (2 = largest E2M1 exponent), clamped to [-127, 127], scale byte X + 127,
 * element code = E2M1_RNE(v * 2^-X).
 * ------------------------------------------------------------------------- */
void orc_quantize_mx(const float* x, int64_t rows, int64_t K, uint8_t* data, uint8_t* scales)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const float* xr = x + r * K;
        uint8_t* dr = data + r * (K / 2);
        memset(dr, 0, (size_t)(K / 2));
        for (int64_t b = 0; b < K / 32; ++b) {
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) {
                double v = fabs((double)xr[b * 32 + i]);
                if (v > amax) amax = v;
            }
            int X;
            if (amax == 0.0) {
                X = -127;
            } else {
                int e2;
                frexp(amax, &e2);          /* amax = f * 2^e2, f in [0.5, 1) */
                X = (e2 - 1) - 2;
                if (X < -127) X = -127;
                if (X > 127) X = 127;
            }
            scales[r * (K / 32) + b] = (uint8_t)(X + 127);
            for (int i = 0; i < 32; ++i) {
                double y = ldexp((double)xr[b * 32 + i], -X);
                put_nibble(dr, b * 32 + i, orc_e2m1_encode(y));
            }
        }
    }
}

/* ---------------------------------------------------------------------------
 * NVFP4 quantisation, [P1] sec. 1 (UE4M3 scale per 16 elements) plus an fp32
 * tensor scale g.  The scale arithmetic is fp32 in exactly this order:
 *   g   = amax_tensor / 2688          (2688 = 6 * 448; g = 1 if amax = 0)
 *   s   = E4M3_RNE(amax_block / fp32(6 * g))   saturating at 448
 *   q_i = E2M1_RNE(v_i / fp32(dec(s) * g))     (all codes zero if dec(s) = 0)
 * ------------------------------------------------------------------------- */
void orc_quantize_nv(const float* x, int64_t rows, int64_t K, const float* g_in,
                     uint8_t* data, uint8_t* scales, float* g_out)
{
    float g;
    if (g_in) {
        g = *g_in;
    } else {
        float amax = 0.0f;
        for (int64_t i = 0; i < rows * K; ++i) {
            float v = fabsf(x[i]);
            if (v > amax) amax = v;
        }
        g = (amax == 0.0f) ? 1.0f : amax / 2688.0f;
    }
    if (g_out) *g_out = g;
    const float six_g = 6.0f * g;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const float* xr = x + r * K;
        uint8_t* dr = data + r * (K / 2);
        memset(dr, 0, (size_t)(K / 2));
        for (int64_t b = 0; b < K / 16; ++b) {
            float amax = 0.0f;
            for (int i = 0; i < 16; ++i) {
                float v = fabsf(xr[b * 16 + i]);
                if (v > amax) amax = v;
            }
            float ratio = amax / six_g;
            int s = orc_ue4m3_encode((double)ratio);
            scales[r * (K / 16) + b] = (uint8_t)s;
            float ds = (float)orc_ue4m3_decode(s);
            float denom = ds * g;
            for (int i = 0; i < 16; ++i) {
                float v = xr[b * 16 + i];
                int code;
                if (ds == 0.0f) {
                    code = signbit(v) ? 8 : 0;
                } else {
                    float y = v / denom;
                    code = orc_e2m1_encode((double)y);
                }
                put_nibble(dr, b * 16 + i, code);
            }
        }
    }
}

/* ---------------------------------------------------------------------------
 * MXFP8 quantisation, [OCP] sec. 6.3 with the E4M3 element: per block of 32
 * along K, shared exponent X = floor(log2(amax)) - 8 (8 = largest E4M3
 * exponent, 448 = 1.75 * 2^8), clamped to [-127, 127], scale byte X + 127,
 * element code = E4M3_RNE(v * 2^-X) saturating at 448; one byte per element.
 * ------------------------------------------------------------------------- */
void orc_quantize_mx8(const float* x, int64_t rows, int64_t K, uint8_t* data, uint8_t* scales)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const float* xr = x + r * K;
        for (int64_t b = 0; b < K / 32; ++b) {
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) {
                double v = fabs((double)xr[b * 32 + i]);
                if (v > amax) amax = v;
            }
            int X;
            if (amax == 0.0) {
                X = -127;
            } else {
                int e2;
                frexp(amax, &e2);          /* amax = f * 2^e2, f in [0.5, 1) */
                X = (e2 - 1) - 8;
                if (X < -127) X = -127;
                if (X > 127) X = 127;
            }
            scales[r * (K / 32) + b] = (uint8_t)(X + 127);
            for (int i = 0; i < 32; ++i)
                data[r * K + b * 32 + i] = (uint8_t)orc_e4m3_encode(ldexp((double)xr[b * 32 + i], -X));
        }
    }
}

void orc_dequantize(const uint8_t* data, const uint8_t* scales, int fmt, double g,
                    int64_t rows, int64_t K, double* out)
{
    int blk = block_of(fmt);
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            int sb = scales[r * (K / blk) + k / blk];
            double sc = (fmt == ORC_NV) ? orc_ue4m3_decode(sb) * g : orc_ue8m0_decode(sb);
            double v = (fmt == ORC_MX8) ? orc_e4m3_decode(data[r * K + k])
                                        : orc_e2m1_decode(get_nibble(data + r * (K / 2), k));
            out[r * K + k] = v * sc;
        }
    }
}

/* ---------------------------------------------------------------------------
 * Top-k routing, [P1] sec. 2 (each token goes to a few of the resident
 * experts) and [P2] "What is the FP4 MoE GEMM" (256 experts, 6 active).
 * Selection: k rounds of "largest remaining logit, lower index on ties".
 * Weights: softmax over the selected logits, w_j = e^(l_j - l_max) / sum.
 * ------------------------------------------------------------------------- */
/* Logits outside the finite numbers (the pages assume finite ones): a NaN
 * ranks below every number, as -inf does, so each pick is a distinct expert
 * in [0, E); a pick equal to the maximum has softmax factor exp(0) = 1, which
 * is also the limit when the maximum is +inf or every pick is -inf. */
static double route_key(float v) { return isnan(v) ? -INFINITY : (double)v; }
static double route_factor(double v, double vmax) { return v == vmax ? 1.0 : exp(v - vmax); }

void orc_route_topk(const float* logits, int T, int E, int k, int32_t* idx, double* w)
{
    char* taken = (char*)malloc((size_t)E);
    for (int t = 0; t < T; ++t) {
        const float* l = logits + (int64_t)t * E;
        memset(taken, 0, (size_t)E);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || route_key(l[e]) > route_key(l[best])) best = e;   /* strict: ties keep lower e */
            }
            taken[best] = 1;
            idx[t * k + j] = best;
        }
        double lmax = route_key(l[idx[t * k]]);
        double den = 0.0;
        for (int j = 0; j < k; ++j) den += route_factor(route_key(l[idx[t * k + j]]), lmax);
        for (int j = 0; j < k; ++j) w[t * k + j] = route_factor(route_key(l[idx[t * k + j]]), lmax) / den;
    }
    free(taken);
}

/* ---------------------------------------------------------------------------
 * Permutation into the expert-contiguous ("contiguous" grouped layout of
 * [P2] "Step 0"): counts per expert, exclusive prefix sum -> offsets[E+1],
 * then slots in ascending slot id s = t*k + j fill their expert's segment.
 * row_to_slot[r] = s of permuted row r; slot_to_row is its inverse.
 * ------------------------------------------------------------------------- */
void orc_moe_permute(const int32_t* idx, int T, int k, int E, int32_t* offsets,
                     int32_t* row_to_slot, int32_t* slot_to_row)
{
    int64_t S = (int64_t)T * k;
    int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    for (int e = 0; e <= E; ++e) offsets[e] = 0;
    for (int64_t s = 0; s < S; ++s) offsets[idx[s] + 1] += 1;
    for (int e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
    for (int64_t s = 0; s < S; ++s) {
        int e = idx[s];
        int32_t r = offsets[e] + fill[e]++;
        row_to_slot[r] = (int32_t)s;
        slot_to_row[s] = r;
    }
    free(fill);
}

void orc_gather_rows(const uint8_t* src_data, const uint8_t* src_scales, int64_t K, int fmt,
                     const int32_t* row_to_slot, int64_t S, int k,
                     uint8_t* dst_data, uint8_t* dst_scales)
{
    int blk = block_of(fmt);
    int64_t rb = row_bytes(fmt, K);
    for (int64_t r = 0; r < S; ++r) {
        int64_t t = row_to_slot[r] / k;
        memcpy(dst_data + r * rb, src_data + t * rb, (size_t)rb);
        memcpy(dst_scales + r * (K / blk), src_scales + t * (K / blk), (size_t)(K / blk));
    }
}

/* ---------------------------------------------------------------------------
 * Grouped GEMM, [P1] sec. 2 (batched expert GEMM with FP4 weights and FP4
 * activations) and [P2] "Step 0" (rows contiguous per expert):
 *   out[r][n] = sum_k deq(A[r][k]) * deq(W[e*N + n][k])      (* g_a * g_w, NV)
 * Each product of two E2M1 values and their scales is exact in fp64; the sum
 * is accumulated in fp64 in k order.
 * ------------------------------------------------------------------------- */
static void decode_row(const uint8_t* data, const uint8_t* scales, int64_t row, int64_t K,
                       int fmt, double* out)
{
    orc_dequantize(data + row * row_bytes(fmt, K), scales + row * (K / block_of(fmt)), fmt, 1.0, 1, K, out);
}

void orc_expert_gemm_rows(const uint8_t* a_data, const uint8_t* a_scales, double g_a,
                          const int64_t* rows, int64_t nrows,
                          const uint8_t* w_e_data, const uint8_t* w_e_scales, double g_w,
                          int n_begin, int n_end, int64_t K, int fmt,
                          double* out, double* abssum)
{
    orc_expert_gemm_rows_mixed(a_data, a_scales, g_a, fmt, rows, nrows, w_e_data, w_e_scales, g_w, fmt,
                               n_begin, n_end, K, out, abssum);
}

/* The same with activations and weights in their own formats: the FP8
 * activation x FP4 weight GEMM of [P2] "Step 0" (a_fmt MX8, w_fmt MX).  A
 * product of an E4M3 and an E2M1 value with their power-of-two scales has at
 * most 6 significant bits, so it is exact in fp64 as well. */
void orc_expert_gemm_rows_mixed(const uint8_t* a_data, const uint8_t* a_scales, double g_a, int a_fmt,
                                const int64_t* rows, int64_t nrows,
                                const uint8_t* w_e_data, const uint8_t* w_e_scales, double g_w, int w_fmt,
                                int n_begin, int n_end, int64_t K, double* out, double* abssum)
{
    int ncols = n_end - n_begin;
    int fmt = w_fmt;
    double* arows = (double*)malloc(sizeof(double) * (size_t)(nrows * K));
    for (int64_t i = 0; i < nrows; ++i) decode_row(a_data, a_scales, rows[i], K, a_fmt, arows + i * K);
    double gg = (a_fmt == ORC_NV ? g_a : 1.0) * (w_fmt == ORC_NV ? g_w : 1.0);
#pragma omp parallel
    {
        double* wrow = (double*)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(dynamic, 4)
        for (int n = n_begin; n < n_end; ++n) {
            decode_row(w_e_data, w_e_scales, n, K, w_fmt, wrow);
            for (int64_t i = 0; i < nrows; ++i) {
                const double* ar = arows + i * K;
                double acc = 0.0, aacc = 0.0;
                for (int64_t kk = 0; kk < K; ++kk) {
                    double p = ar[kk] * wrow[kk];
                    acc += p;
                    aacc += fabs(p);
                }
                out[i * ncols + (n - n_begin)] = acc * gg;
                if (abssum) abssum[i * ncols + (n - n_begin)] = aacc * gg;
            }
        }
        free(wrow);
    }
    free(arows);
}

void orc_grouped_gemm(const uint8_t* a_data, const uint8_t* a_scales, double g_a,
                      const int32_t* offsets, int E,
                      const uint8_t* w_data, const uint8_t* w_scales, double g_w,
                      int N, int64_t K, int fmt,
                      int64_t row_begin, int64_t row_end, int n_begin, int n_end,
                      double* out, double* abssum)
{
    int blk = block_of(fmt);
    int ncols = n_end - n_begin;
    for (int e = 0; e < E; ++e) {
        int64_t lo = offsets[e] > row_begin ? offsets[e] : row_begin;
        int64_t hi = offsets[e + 1] < row_end ? offsets[e + 1] : row_end;
        if (hi <= lo) continue;
        int64_t nr = hi - lo;
        int64_t* rows = (int64_t*)malloc(sizeof(int64_t) * (size_t)nr);
        for (int64_t i = 0; i < nr; ++i) rows[i] = lo + i;
        double* o = (double*)malloc(sizeof(double) * (size_t)(nr * ncols));
        double* s = abssum ? (double*)malloc(sizeof(double) * (size_t)(nr * ncols)) : NULL;
        orc_expert_gemm_rows(a_data, a_scales, g_a, rows, nr,
                             w_data + (int64_t)e * N * row_bytes(fmt, K), w_scales + (int64_t)e * N * (K / blk),
                             g_w, n_begin, n_end, K, fmt, o, s);
        for (int64_t i = 0; i < nr; ++i) {
            for (int c = 0; c < ncols; ++c) {
                out[(lo + i) * (int64_t)N + n_begin + c] = o[i * ncols + c];
                if (abssum) abssum[(lo + i) * (int64_t)N + n_begin + c] = s[i * ncols + c];
            }
        }
        free(rows);
        free(o);
        free(s);
    }
}

/* ---------------------------------------------------------------------------
 * SwiGLU on the FC1 output, the fused "SwiGLU + quant" pattern of [P3]:
 * h = silu(gate) * up, silu(x) = x / (1 + e^-x); gate = column i, up =
 * column I + i.  fp64 from the fp32 FC1 values, rounded once to fp32.
 * ------------------------------------------------------------------------- */
void orc_swiglu(const float* y1, int64_t rows, int I, float* h)
{
    for (int64_t r = 0; r < rows; ++r) {
        for (int i = 0; i < I; ++i) {
            double g = y1[r * 2 * I + i];
            double u = y1[r * 2 * I + I + i];
            h[r * I + i] = (float)(g / (1.0 + exp(-g)) * u);
        }
    }
}

/* ---------------------------------------------------------------------------
 * Combine, the MoE combine step of [P3]: each token's output is the routing
 * weighted sum of its k expert outputs, j = 0..k-1 in order.
 * ------------------------------------------------------------------------- */
void orc_moe_combine(const double* y2, const int32_t* slot_to_row, const double* w,
                     int T, int k, int d, double* out)
{
    for (int t = 0; t < T; ++t) {
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j)
                acc += w[t * k + j] * y2[(int64_t)slot_to_row[t * k + j] * d + c];
            out[(int64_t)t * d + c] = acc;
        }
    }
}
