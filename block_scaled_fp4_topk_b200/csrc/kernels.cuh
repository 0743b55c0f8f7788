// kernels.cuh -- launch functions of libds4g's kernels (host side); the C ABI
// in api.cu validates arguments and calls these.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ds4g {

cudaError_t launch_quantize(const void* x, int dtype, int64_t rows, int64_t K, int fmt, const float* g_in,
                            uint8_t* data, uint8_t* scales, float* g_out, void* ws, cudaStream_t st);

cudaError_t launch_route_topk(const float* logits, int T, int E, int k, int32_t* idx, float* w,
                              cudaStream_t st);

size_t permute_workspace_bytes(int T, int k, int E);
size_t dispatch_workspace_bytes(int T, int k, int E, int fmt, int has_g_in);
cudaError_t launch_dispatch(const float* logits, const void* x, int dtype, int Tn, int E, int k, int64_t d, int fmt,
                            const float* g_in, int32_t* idx, float* w, uint8_t* xd, uint8_t* xs, float* xg,
                            int32_t* offsets, int32_t* r2s, int32_t* s2r, uint8_t* ad, uint8_t* as, float* ag,
                            void* ws, cudaStream_t st);
cudaError_t launch_permute(const int32_t* idx, int T, int k, int E, const uint8_t* xd, const uint8_t* xs,
                           const float* xg, int64_t K, int fmt, int32_t* offsets, int32_t* row_to_slot,
                           int32_t* slot_to_row, uint8_t* ad, uint8_t* as, float* ag, void* ws,
                           cudaStream_t st);

cudaError_t launch_segment_ids(const int32_t* offsets, int nseg, int modulo, int64_t rows, int32_t* out,
                               cudaStream_t st);

struct GemmArgs {
    const uint8_t* a_data;
    const uint8_t* a_scales;
    const float* a_g;
    int64_t S;            // rows of a
    const int32_t* offsets;
    int E;
    const uint8_t* w_data;
    const uint8_t* w_scales;
    const float* w_g;
    int N;
    int64_t K;
    int fmt;
    int epilogue;
    float* out;
    uint8_t* oq_data;
    uint8_t* oq_scales;
    const float* oq_g;
    float* h_debug;
    int max_rows;
    const int32_t* r2s;      // combine epilogue: row -> slot, routing weights, k
    const float* route_w;
    int topk;
    int chained;             // decode kernel: launched to overlap the previous kernel on the stream
    int band_tiles;          // prefill kernel, combine epilogue: column tiles per band of the tile order (0: all)
    int ksplit;              // plain epilogue with few tiles: equal K parts added into the zeroed output (0, 1: none)
};

cudaError_t launch_gemv(const GemmArgs& a, cudaStream_t st);
bool gemm_tc_supports(int fmt, int64_t K);
cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t st);
bool gemv_tc_supports(int fmt, int64_t K, int N, int epilogue, int E);
cudaError_t launch_gemv_tc(const GemmArgs& a, cudaStream_t st);
bool ffn_dtc_supports(int fmt, int64_t d, int I, int E);
cudaError_t launch_ffn_dtc(const GemmArgs& fc1, const GemmArgs& fc2, int32_t* ctr, cudaStream_t st);

cudaError_t launch_swiglu_requant(const float* y1, int64_t rows, int I, int fmt, uint8_t* hd, uint8_t* hs,
                                  const float* hg, float* h_debug, cudaStream_t st);

cudaError_t launch_combine(const float* y2, const int32_t* slot_to_row, const float* w, int T, int k, int d,
                           float* out, cudaStream_t st);

}  // namespace ds4g
