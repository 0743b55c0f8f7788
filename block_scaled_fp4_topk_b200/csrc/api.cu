// api.cu -- the C ABI of libds4g (declared in include/ds4g.h): host-side
// argument and shape validation, then the kernel launches.  Nothing is
// launched when validation fails ("DGX Spark native FP4 matrix instructions
// ..." sec. 3: the FP4 path checks that K is a multiple of 64 and reports an
// error instead of silently taking another path).
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.cuh"

using namespace ds4g;

static inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }
static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static inline ds4g_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DS4G_OK : DS4G_ERR_CUDA; }
static inline int block_of(int fmt) { return fmt == DS4G_NVFP4 ? 16 : 32; }

static ds4g_status check_fp4(const ds4g_fp4* t, int64_t rows, int64_t K, int fmt, bool need_g)
{
    if (!t) return DS4G_ERR_INVALID_ARG;
    if (t->fmt != fmt || t->rows != rows || t->K != K) return DS4G_ERR_SHAPE;
    if (rows > 0 && (!t->data || !t->scales)) return DS4G_ERR_INVALID_ARG;   // empty tensors may be NULL
    if (!aligned16(t->data) || !aligned16(t->scales)) return DS4G_ERR_INVALID_ARG;
    if (need_g && fmt == DS4G_NVFP4 && !t->g) return DS4G_ERR_INVALID_ARG;
    return DS4G_OK;
}

extern "C" {

const char* ds4g_status_str(ds4g_status s)
{
    switch (s) {
    case DS4G_OK: return "ok";
    case DS4G_ERR_INVALID_ARG: return "invalid argument";
    case DS4G_ERR_SHAPE: return "unsupported shape (K must be a multiple of 64; see ds4g.h)";
    case DS4G_ERR_UNSUPPORTED: return "device is not sm_100 (B200 class)";
    case DS4G_ERR_CUDA: return "CUDA error";
    case DS4G_ERR_DEVICE: return "a device-side bounded wait gave up";
    case DS4G_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

ds4g_status ds4g_device_supported(void)
{
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DS4G_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return DS4G_ERR_CUDA;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return DS4G_ERR_CUDA;
    return (major == 10 && minor == 0) ? DS4G_OK : DS4G_ERR_UNSUPPORTED;
}

ds4g_status ds4g_check_device(void* stream)
{
    if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return DS4G_ERR_CUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return DS4G_ERR_CUDA;
    if (v != 0 && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return DS4G_ERR_CUDA;
    return v ? DS4G_ERR_DEVICE : DS4G_OK;
}

size_t ds4g_quantize_workspace_bytes(int fmt, int has_g_in)
{
    return (fmt == DS4G_NVFP4 && !has_g_in) ? 16 : 0;
}

ds4g_status ds4g_quantize_mx(const void* x, int dtype, int64_t rows, int64_t K, int fmt, const float* g_in,
                             ds4g_fp4* out, void* workspace, size_t ws_bytes, void* stream)
{
    if (fmt != DS4G_MXFP4 && fmt != DS4G_NVFP4 && fmt != DS4G_MXFP8) return DS4G_ERR_INVALID_ARG;
    if (dtype != DS4G_BF16 && dtype != DS4G_F32) return DS4G_ERR_INVALID_ARG;
    if (rows < 0 || K <= 0) return DS4G_ERR_SHAPE;
    if (K % 64 != 0) return DS4G_ERR_SHAPE;
    if (rows > 0 && (!x || !aligned16(x))) return DS4G_ERR_INVALID_ARG;
    ds4g_status st = check_fp4(out, rows, K, fmt, true);
    if (st != DS4G_OK) return st;
    if (fmt == DS4G_NVFP4 && !g_in) {
        if (!workspace || ws_bytes < ds4g_quantize_workspace_bytes(fmt, 0) || !aligned16(workspace))
            return DS4G_ERR_WORKSPACE;
    }
    return cuda_status(launch_quantize(x, dtype, rows, K, fmt, g_in, out->data, out->scales,
                                       fmt == DS4G_NVFP4 ? out->g : nullptr, workspace, S(stream)));
}

ds4g_status ds4g_route_topk(const float* logits, int T, int E, int k, int32_t* idx, float* w, void* stream)
{
    if (T < 0 || E < 1 || E > 1024 || k < 1 || k > E || k > 32) return DS4G_ERR_INVALID_ARG;
    if (T > 0 && (!logits || !idx || !w)) return DS4G_ERR_INVALID_ARG;
    return cuda_status(launch_route_topk(logits, T, E, k, idx, w, S(stream)));
}

size_t ds4g_permute_workspace_bytes(int T, int k, int E)
{
    if (T < 0 || k < 1 || E < 1) return 0;
    return permute_workspace_bytes(T, k, E);
}

ds4g_status ds4g_moe_permute(const int32_t* idx, int T, int k, int E, const ds4g_fp4* x_q, int32_t* offsets,
                             int32_t* row_to_slot, int32_t* slot_to_row, ds4g_fp4* a_perm, void* workspace,
                             size_t ws_bytes, void* stream)
{
    if (T < 0 || k < 1 || E < 1 || E > 4096 || k > E) return DS4G_ERR_INVALID_ARG;
    if (!offsets || !x_q || !a_perm) return DS4G_ERR_INVALID_ARG;
    const int64_t S_ = (int64_t)T * k;
    if (S_ > 0x7FFFFFFF) return DS4G_ERR_SHAPE;
    if (S_ > 0 && (!idx || !row_to_slot || !slot_to_row)) return DS4G_ERR_INVALID_ARG;
    const int64_t K = x_q->K;
    if (K <= 0 || K % 64 != 0) return DS4G_ERR_SHAPE;
    ds4g_status st = check_fp4(x_q, T, K, x_q->fmt, true);
    if (st != DS4G_OK) return st;
    st = check_fp4(a_perm, S_, K, x_q->fmt, true);
    if (st != DS4G_OK) return st;
    if (S_ > 0 && (!workspace || ws_bytes < ds4g_permute_workspace_bytes(T, k, E) || !aligned16(workspace)))
        return DS4G_ERR_WORKSPACE;
    return cuda_status(launch_permute(idx, T, k, E, x_q->data, x_q->scales, x_q->g, K, x_q->fmt, offsets,
                                      row_to_slot, slot_to_row, a_perm->data, a_perm->scales, a_perm->g, workspace,
                                      S(stream)));
}

size_t ds4g_dispatch_workspace_bytes(int T, int k, int E, int fmt, int has_g_in)
{
    if (T < 0 || k < 1 || E < 1) return 0;
    return dispatch_workspace_bytes(T, k, E, fmt, has_g_in);
}

ds4g_status ds4g_moe_dispatch(const float* logits, const void* x, int dtype, int T, int E, int k, int fmt,
                              const float* g_in, int32_t* idx, float* w, ds4g_fp4* x_q, int32_t* offsets,
                              int32_t* row_to_slot, int32_t* slot_to_row, ds4g_fp4* a_perm, void* workspace,
                              size_t ws_bytes, void* stream)
{
    if (fmt != DS4G_MXFP4 && fmt != DS4G_NVFP4) return DS4G_ERR_INVALID_ARG;
    if (dtype != DS4G_BF16 && dtype != DS4G_F32) return DS4G_ERR_INVALID_ARG;
    if (T < 0 || E < 1 || E > 1024 || k < 1 || k > E || k > 32) return DS4G_ERR_INVALID_ARG;
    if (!x_q || !a_perm || !offsets) return DS4G_ERR_INVALID_ARG;
    const int64_t S_ = (int64_t)T * k;
    if (S_ > 0x7FFFFFFF) return DS4G_ERR_SHAPE;
    const int64_t K = x_q->K;
    if (K <= 0 || K % 64 != 0) return DS4G_ERR_SHAPE;
    if (T > 0 && (!logits || !x || !aligned16(x) || !idx || !w || !row_to_slot || !slot_to_row))
        return DS4G_ERR_INVALID_ARG;
    ds4g_status st = check_fp4(x_q, T, K, fmt, true);
    if (st != DS4G_OK) return st;
    st = check_fp4(a_perm, S_, K, fmt, true);
    if (st != DS4G_OK) return st;
    const size_t need = ds4g_dispatch_workspace_bytes(T, k, E, fmt, g_in != nullptr);
    if (S_ > 0 && (!workspace || ws_bytes < need || !aligned16(workspace))) return DS4G_ERR_WORKSPACE;
    if (S_ == 0) {
        // nothing routed: what the separate calls do on an empty batch
        // (offsets all zero; the permuted tensor takes x_q's tensor scale)
        if (cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), S(stream)) != cudaSuccess) return DS4G_ERR_CUDA;
        if (fmt == DS4G_NVFP4 &&
            cudaMemcpyAsync(a_perm->g, x_q->g, sizeof(float), cudaMemcpyDeviceToDevice, S(stream)) != cudaSuccess)
            return DS4G_ERR_CUDA;
        return DS4G_OK;
    }
    return cuda_status(launch_dispatch(logits, x, dtype, T, E, k, K, fmt, g_in, idx, w, x_q->data, x_q->scales,
                                       x_q->g, offsets, row_to_slot, slot_to_row, a_perm->data, a_perm->scales,
                                       a_perm->g, workspace, S(stream)));
}

// chained: FC2 + combine adding into out (not zeroed) and launched to
// overlap the previous kernel on the stream (decode kernel only)
static ds4g_status grouped_gemm(const ds4g_fp4* a, const int32_t* offsets, int E, int max_rows_per_expert,
                                const ds4g_fp4* w, int N, int epilogue, float* out, ds4g_fp4* out_q, float* h_debug,
                                const int32_t* row_to_slot, const float* route_w, int k, int T, void* stream,
                                bool chained = false)
{
    if (!a || !w || !offsets || E < 1 || N < 1 || max_rows_per_expert < 0) return DS4G_ERR_INVALID_ARG;
    const int fmt = a->fmt;
    if (fmt != DS4G_MXFP4 && fmt != DS4G_NVFP4 && fmt != DS4G_MXFP8) return DS4G_ERR_INVALID_ARG;
    const int64_t K = a->K;
    if (K <= 0 || K % 64 != 0) return DS4G_ERR_SHAPE;
    ds4g_status st = check_fp4(a, a->rows, K, fmt, true);
    if (st != DS4G_OK) return st;
    // FP8 (MXFP8) activations multiply MXFP4 weights (routed experts) or
    // MXFP8 weights (the shared expert); FP4 activations, weights of their own
    // format
    if (fmt == DS4G_MXFP8 && w->fmt != DS4G_MXFP4 && w->fmt != DS4G_MXFP8) return DS4G_ERR_SHAPE;
    st = check_fp4(w, (int64_t)E * N, K, fmt == DS4G_MXFP8 ? w->fmt : fmt, true);
    if (st != DS4G_OK) return st;
    const int mode = (fmt == DS4G_MXFP8 && w->fmt == DS4G_MXFP8) ? kFmtFp8Fp8 : fmt;   // the kernel's operand mode
    // kernel choice: decode-sized segments (<= 16 rows) take the swapped
    // tensor-core kernel (weights as the MMA's M side) when the tiling fits;
    // longer segments the 128 x 224 / 128 x 256 tensor-core kernel; shapes neither fits
    // take the dp4a GEMV kernel (any segment length).  FP8 activations run on
    // the 128-row tensor-core kernel at every segment length.
    const bool swiglu = epilogue == DS4G_EPI_SWIGLU_REQUANT;
    const bool tc_shape = gemm_tc_supports(fmt, K) &&
                          (!swiglu ? (N % 256 == 0 || N % 224 == 0) : (N % 2 == 0 && (N / 2) % 32 == 0));
    if (fmt == DS4G_MXFP8 && !tc_shape) return DS4G_ERR_SHAPE;
    const bool dtc = fmt != DS4G_MXFP8 && max_rows_per_expert <= 16 && gemv_tc_supports(fmt, K, N, epilogue, E);
    const bool gemv = fmt != DS4G_MXFP8 && !dtc && (max_rows_per_expert <= 8 || !tc_shape);
    const int64_t Sr = a->rows;
    if (!swiglu) {
        if (Sr > 0 && (!out || !aligned16(out))) return DS4G_ERR_INVALID_ARG;
        if (gemv && N % 64 != 0) return DS4G_ERR_SHAPE;      // the dp4a kernel's column tiles
    } else {
        if (N % 2 != 0) return DS4G_ERR_SHAPE;
        const int I = N / 2;
        if (I % 32 != 0) return DS4G_ERR_SHAPE;
        st = check_fp4(out_q, Sr, I, fmt, true);
        if (st != DS4G_OK) return st;
        if (h_debug && !aligned16(h_debug)) return DS4G_ERR_INVALID_ARG;
    }
    if ((int64_t)E * N > 0x7FFFFFFF) return DS4G_ERR_SHAPE;
    GemmArgs g;
    g.a_data = a->data;
    g.a_scales = a->scales;
    g.a_g = a->g;
    g.S = Sr;
    g.offsets = offsets;
    g.E = E;
    g.w_data = w->data;
    g.w_scales = w->scales;
    g.w_g = w->g;
    g.N = N;
    g.K = K;
    g.fmt = mode;
    g.epilogue = epilogue;
    g.out = out;
    g.oq_data = out_q ? out_q->data : nullptr;
    g.oq_scales = out_q ? out_q->scales : nullptr;
    g.oq_g = out_q ? out_q->g : nullptr;
    g.h_debug = h_debug;
    g.max_rows = max_rows_per_expert;
    g.r2s = row_to_slot;
    g.route_w = route_w;
    g.topk = k;
    g.chained = chained ? 1 : 0;
    g.band_tiles = 0;
    g.ksplit = 1;
    if (epilogue == kEpiCombine && T > 0 && !chained) {
        cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * (size_t)T * N, S(stream));
        if (e != cudaSuccess) return DS4G_ERR_CUDA;
    }
    return cuda_status(dtc ? launch_gemv_tc(g, S(stream)) : gemv ? launch_gemv(g, S(stream)) : launch_gemm_tc(g, S(stream)));
}

ds4g_status ds4g_grouped_gemm_fp4(const ds4g_fp4* a, const int32_t* offsets, int E, int max_rows_per_expert,
                                  const ds4g_fp4* w, int N, int epilogue, float* out, ds4g_fp4* out_q,
                                  float* h_debug, void* stream)
{
    if (epilogue != DS4G_EPI_NONE && epilogue != DS4G_EPI_SWIGLU_REQUANT) return DS4G_ERR_INVALID_ARG;
    return grouped_gemm(a, offsets, E, max_rows_per_expert, w, N, epilogue, out, out_q, h_debug, nullptr, nullptr, 0,
                        0, stream);
}

ds4g_status ds4g_grouped_gemm_fp4_combine(const ds4g_fp4* a, const int32_t* offsets, int E, int max_rows_per_expert,
                                          const ds4g_fp4* w, int N, const int32_t* row_to_slot, const float* route_w,
                                          int T, int k, float* out, void* stream)
{
    if (T < 0 || k < 1) return DS4G_ERR_INVALID_ARG;
    if (a && a->rows != (int64_t)T * k) return DS4G_ERR_SHAPE;
    if (T > 0 && (!row_to_slot || !route_w || !out)) return DS4G_ERR_INVALID_ARG;
    return grouped_gemm(a, offsets, E, max_rows_per_expert, w, N, kEpiCombine, out, nullptr, nullptr, row_to_slot,
                        route_w, k, T, stream);
}

ds4g_status ds4g_grouped_gemm_fp4_combine_chained(const ds4g_fp4* a, const int32_t* offsets, int E,
                                                  int max_rows_per_expert, const ds4g_fp4* w, int N,
                                                  const int32_t* row_to_slot, const float* route_w, int T, int k,
                                                  float* out, void* stream)
{
    if (T < 0 || k < 1) return DS4G_ERR_INVALID_ARG;
    if (a && a->rows != (int64_t)T * k) return DS4G_ERR_SHAPE;
    if (T > 0 && (!row_to_slot || !route_w || !out)) return DS4G_ERR_INVALID_ARG;
    return grouped_gemm(a, offsets, E, max_rows_per_expert, w, N, kEpiCombine, out, nullptr, nullptr, row_to_slot,
                        route_w, k, T, stream, true);
}

ds4g_status ds4g_moe_ffn_fp4(const ds4g_fp4* a, const int32_t* offsets, int E, int max_rows_per_expert,
                             const ds4g_fp4* w1, const ds4g_fp4* w2, int d, int I, ds4g_fp4* h_q,
                             const int32_t* row_to_slot, const float* route_w, int T, int k, float* out,
                             int32_t* counters, void* stream)
{
    if (!a || !offsets || !w1 || !w2 || !h_q || E < 1 || d < 1 || I < 1 || T < 0 || k < 1 ||
        max_rows_per_expert < 0)
        return DS4G_ERR_INVALID_ARG;
    const int fmt = a->fmt;
    if (fmt != DS4G_MXFP4 && fmt != DS4G_NVFP4) return DS4G_ERR_INVALID_ARG;
    if (a->rows != (int64_t)T * k) return DS4G_ERR_SHAPE;
    if (max_rows_per_expert > 16 || !ffn_dtc_supports(fmt, d, I, E)) return DS4G_ERR_SHAPE;
    ds4g_status st = check_fp4(a, a->rows, d, fmt, true);
    if (st != DS4G_OK) return st;
    st = check_fp4(w1, (int64_t)E * 2 * I, d, fmt, true);
    if (st != DS4G_OK) return st;
    st = check_fp4(w2, (int64_t)E * d, I, fmt, true);
    if (st != DS4G_OK) return st;
    st = check_fp4(h_q, a->rows, I, fmt, true);
    if (st != DS4G_OK) return st;
    if ((int64_t)E * 2 * I > 0x7FFFFFFF || (int64_t)E * d > 0x7FFFFFFF) return DS4G_ERR_SHAPE;
    if (T > 0 && (!row_to_slot || !route_w || !out || !counters || !aligned16(out))) return DS4G_ERR_INVALID_ARG;
    GemmArgs g1 = {};
    g1.a_data = a->data;
    g1.a_scales = a->scales;
    g1.a_g = a->g;
    g1.S = a->rows;
    g1.offsets = offsets;
    g1.E = E;
    g1.w_data = w1->data;
    g1.w_scales = w1->scales;
    g1.w_g = w1->g;
    g1.N = 2 * I;
    g1.K = d;
    g1.fmt = fmt;
    g1.epilogue = DS4G_EPI_SWIGLU_REQUANT;
    g1.oq_data = h_q->data;
    g1.oq_scales = h_q->scales;
    g1.oq_g = h_q->g;
    g1.max_rows = max_rows_per_expert;
    g1.ksplit = 1;
    GemmArgs g2 = {};
    g2.a_data = h_q->data;
    g2.a_scales = h_q->scales;
    g2.a_g = h_q->g;
    g2.S = a->rows;
    g2.offsets = offsets;
    g2.E = E;
    g2.w_data = w2->data;
    g2.w_scales = w2->scales;
    g2.w_g = w2->g;
    g2.N = d;
    g2.K = I;
    g2.fmt = fmt;
    g2.epilogue = kEpiCombine;
    g2.out = out;
    g2.max_rows = max_rows_per_expert;
    g2.r2s = row_to_slot;
    g2.route_w = route_w;
    g2.topk = k;
    g2.ksplit = 1;
    return cuda_status(launch_ffn_dtc(g1, g2, counters, S(stream)));
}

ds4g_status ds4g_segment_ids(const int32_t* offsets, int nseg, int modulo, int64_t rows, int32_t* out,
                             void* stream)
{
    if (nseg < 1 || modulo < 1 || rows < 0) return DS4G_ERR_INVALID_ARG;
    if (rows > 0 && (!offsets || !out)) return DS4G_ERR_INVALID_ARG;
    return cuda_status(launch_segment_ids(offsets, nseg, modulo, rows, out, S(stream)));
}

ds4g_status ds4g_zero_fill(void* p, size_t bytes, void* stream)
{
    if (bytes == 0) return DS4G_OK;
    if (!p) return DS4G_ERR_INVALID_ARG;
    return cudaMemsetAsync(p, 0, bytes, S(stream)) == cudaSuccess ? DS4G_OK : DS4G_ERR_CUDA;
}

ds4g_status ds4g_swiglu_requant(const float* y1, int64_t rows, int I, int fmt, ds4g_fp4* h_q, float* h_debug,
                                void* stream)
{
    if (fmt != DS4G_MXFP4 && fmt != DS4G_NVFP4) return DS4G_ERR_INVALID_ARG;
    if (rows < 0 || I <= 0 || I % 32 != 0) return DS4G_ERR_SHAPE;
    if (rows > 0 && !y1) return DS4G_ERR_INVALID_ARG;
    ds4g_status st = check_fp4(h_q, rows, I, fmt, true);
    if (st != DS4G_OK) return st;
    return cuda_status(launch_swiglu_requant(y1, rows, I, fmt, h_q->data, h_q->scales, h_q->g, h_debug, S(stream)));
}

ds4g_status ds4g_moe_combine(const float* y2, const int32_t* slot_to_row, const float* w, int T, int k, int d,
                             float* out, void* stream)
{
    if (T < 0 || k < 1 || d < 1) return DS4G_ERR_INVALID_ARG;
    if (d % 4 != 0) return DS4G_ERR_SHAPE;
    if (T > 0 && (!y2 || !slot_to_row || !w || !out || !aligned16(y2) || !aligned16(out)))
        return DS4G_ERR_INVALID_ARG;
    return cuda_status(launch_combine(y2, slot_to_row, w, T, k, d, out, S(stream)));
}

}  // extern "C"
