// unity.cu -- libds4g is built as one translation unit so the device error
// word defined in api.cu is the one every kernel raises (no relocatable
// device code needed).
#include "api.cu"
#include "quantize.cu"
#include "route.cu"
#include "permute.cu"
#include "dispatch.cu"
#include "gemv.cu"
#include "gemm_tc.cu"
#include "gemv_tc.cu"
#include "swiglu.cu"
#include "combine.cu"
#include "noalloc.cu"
