// common.cuh -- shared device helpers of libds4g (sm_100a): FP4 / scale
// codecs written from the format definitions, the device error word, and
// small launch utilities.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ds4g.h"

namespace ds4g {

constexpr int kNumSMs = 148;

// Error word raised by device-side bounded waits; read and cleared by
// ds4g_check_device().  Defined here: the library is one translation unit.
__device__ unsigned int g_device_error = 0;

enum DeviceError : unsigned int {
    kErrNone = 0,
    kErrWaitTimeout = 1u,      // an mbarrier wait exceeded its iteration cap
    kErrBadOffsets = 2u,       // offsets[E] larger than the row count
};

__device__ __forceinline__ void raise_error(unsigned int e) { atomicOr(&g_device_error, e); }

// ---------------------------------------------------------------------------
// E2M1 ("DGX Spark native FP4 matrix instructions ..." sec. 1): 1 sign bit,
// 2 exponent bits, 1 mantissa bit; magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}.
// Round to nearest, ties to the even code, saturating at 6.  `a` is |y|.
__device__ __forceinline__ uint32_t e2m1_mag_code(float a)
{
    uint32_t c;
    if (a <= 0.25f) c = 0;
    else if (a < 0.75f) c = 1;
    else if (a <= 1.25f) c = 2;
    else if (a < 1.75f) c = 3;
    else if (a <= 2.5f) c = 4;
    else if (a < 3.5f) c = 5;
    else if (a <= 5.0f) c = 6;
    else c = 7;
    return c;
}

// code with the sign bit taken from y's sign bit (so -0 gives 0x8)
__device__ __forceinline__ uint32_t e2m1_code(float y)
{
    return e2m1_mag_code(fabsf(y)) | ((__float_as_uint(y) >> 28) & 8u);
}

// Two values at once with the hardware conversion (round to nearest even,
// saturating to +-6, sign kept): low nibble = lo, high nibble = hi.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi)
{
    uint32_t d;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(d)
        : "f"(hi), "f"(lo));
    return d;
}

// Two values as E4M3 bytes with the hardware conversion (round to nearest
// even, saturating to +-448, sign kept): low byte = lo, high byte = hi.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi)
{
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
    return d;
}

// MX shared exponent X = floor(log2(amax)) - EMAX, clamped to [-127, 127]
// (OCP MX rule; EMAX is the element's largest exponent: 2 for E2M1, 8 for
// E4M3), from the bits.
template <int EMAX = 2>
__device__ __forceinline__ int mx_shared_exp(float amax)
{
    uint32_t b = __float_as_uint(amax);
    if (b == 0) return -127;
    int ef = (int)((b >> 23) & 0xFF);
    int fl;
    if (ef == 0) {  // subnormal: value = m * 2^-149
        uint32_t m = b & 0x7FFFFF;
        fl = (31 - __clz(m)) - 149;
    } else {
        fl = ef - 127;
    }
    int X = fl - EMAX;
    return X < -127 ? -127 : (X > 127 ? 127 : X);
}

// 2^e as fp32 for e in [-149, 127] (exact; subnormal below -126)
__device__ __forceinline__ float exp2i(int e)
{
    if (e >= -126) return __uint_as_float((uint32_t)(e + 127) << 23);
    return __uint_as_float(1u << (e + 149));
}

// UE4M3 (unsigned E4M3, bias 7, subnormals m * 2^-9, max 448): decode
__device__ __forceinline__ float ue4m3_value(uint32_t b)
{
    uint32_t e = (b >> 3) & 0xF, m = b & 7;
    if (e == 0) return (float)m * 0.001953125f;      // m * 2^-9
    return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// UE4M3 round to nearest even of r >= 0, saturating at 448 (code 0x7E)
__device__ __forceinline__ uint32_t ue4m3_encode(float r)
{
    uint32_t b = __float_as_uint(r);
    int ef = (int)((b >> 23) & 0xFF);
    int E = ef - 127;
    if (E < -6) {
        // subnormal range: r * 2^9 in [0, 8), exact product, RNE to an integer
        return (uint32_t)__float2int_rn(__fmul_rn(r, 512.0f));
    }
    if (E > 8) return 0x7E;
    uint32_t m23 = b & 0x7FFFFF;
    uint32_t q = m23 >> 20;
    uint32_t rem = m23 & 0xFFFFF;
    if (rem > 0x80000u || (rem == 0x80000u && (q & 1u))) q += 1;
    uint32_t code = ((uint32_t)(E + 7) << 3) + q;
    return code > 0x7Eu ? 0x7Eu : code;
}

// 2 * E2M1 magnitude of codes 0..7 as bytes: {0,1,2,3,4,6,8,12}
constexpr uint32_t kLutLo = 0x03020100u;
constexpr uint32_t kLutHi = 0x0C080604u;

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// SwiGLU element ("Moore Threads full-link adaptation of DeepSeek-V4", the
// fused SwiGLU + quantisation step): silu(g) * u = g u / (1 + e^-g) in fp32
// with the hardware's fast exponential and division (__expf: at most
// 2 + floor(1.173 |x|) ulp; __fdividef: at most 2 ulp for divisors in
// [2^-126, 2^126]; CUDA C Programming Guide, intrinsic functions), so h is
// within (5 + 1.173 |g|) 2^-23 |h| of silu(g) u for the fp32 g, u it gets.
// The IEEE-rounded form costs a fifth of the prefill FC1 kernel's time
// (measured), because this epilogue runs between two tiles' mainloops.
// Every kernel that computes h (fused epilogues and the standalone step) uses
// this one function, so they give the same bits for the same g and u.
__device__ __forceinline__ float swiglu_f32(float g, float u)
{
    return __fdividef(__fmul_rn(g, u), __fadd_rn(1.0f, __expf(-g)));
}

// internal GEMM operand mode: MXFP8 activations with MXFP8 weights (the
// shared expert's FP8 weights); DS4G_MXFP8 as a GEMM mode means MXFP8
// activations with MXFP4 weights
constexpr int kFmtFp8Fp8 = 3;
// FP8 (E4M3) activations, either weight format
__host__ __device__ constexpr bool fp8_act(int fmt) { return fmt == DS4G_MXFP8 || fmt == kFmtFp8Fp8; }

// internal epilogue mode: FC2 with the weighted combine fused (adds into the
// token outputs instead of storing per-row results)
constexpr int kEpiCombine = 2;
constexpr int kEpiFfn = 3;        // decode kernel: FC1 + SwiGLU + requantisation, then FC2 + combine, one launch

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

__device__ __forceinline__ void red_add_v2(float* addr, float a, float b)
{
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(addr), "f"(a), "f"(b) : "memory");
}

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace ds4g
