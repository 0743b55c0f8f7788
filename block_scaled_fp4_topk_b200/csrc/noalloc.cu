// noalloc.cu -- ds4g_moe_permute_static: the expert permutation for callers
// that must not allocate device memory at all, not even a workspace of their
// own (for example a host runtime that hands all device memory to its own
// pool at start-up and forbids later allocations, or a plug-in that may only
// touch the buffers it is given).  Its scratch space is a file-scope device
// array that every GPU loading the library holds until the process exits.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace ds4g {

// scratch of the multi-CTA permutation (per-chunk expert histograms), E * B
// 32-bit counters with B = ceil(T * k / 256) (256 slots per chunk); the
// single-CTA path used for T * k <= 512 needs none
constexpr size_t kStaticPermuteScratchBytes = 256 * 1024;
static __device__ __align__(256) int32_t g_permute_scratch[kStaticPermuteScratchBytes / sizeof(int32_t)];

constexpr int kMaxDevices = 64;
static void* g_scratch_ptr[kMaxDevices];
static std::mutex g_scratch_mutex;

// device address of the scratch array on the current device (the array's
// host-side name is only a stand-in, never a device address).  Looked up on
// the first call on each device and kept only once a lookup has succeeded: a
// lookup that fails (for example one attempted during a stream capture) is
// reported to that caller and tried again on the next call.
static cudaError_t static_scratch(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_permute_scratch);
        if (e != cudaSuccess) {
            cudaGetLastError();   // the failure is returned here, not left for the next CUDA call
            return e;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace ds4g

extern "C" size_t ds4g_permute_static_max_bytes(void) { return ds4g::kStaticPermuteScratchBytes; }

extern "C" ds4g_status ds4g_moe_permute_static(const int32_t* idx, int T, int k, int E, const ds4g_fp4* x_q,
                                               int32_t* offsets, int32_t* row_to_slot, int32_t* slot_to_row,
                                               ds4g_fp4* a_perm, void* stream)
{
    using namespace ds4g;
    if (T < 0 || k < 1 || E < 1 || E > 4096 || k > E) return DS4G_ERR_INVALID_ARG;
    if (ds4g_permute_workspace_bytes(T, k, E) > kStaticPermuteScratchBytes) return DS4G_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (static_scratch(&scratch) != cudaSuccess || !scratch) return DS4G_ERR_CUDA;
    return ds4g_moe_permute(idx, T, k, E, x_q, offsets, row_to_slot, slot_to_row, a_perm, scratch,
                            kStaticPermuteScratchBytes, stream);
}
