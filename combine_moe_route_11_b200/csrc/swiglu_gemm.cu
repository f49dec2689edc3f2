// Grouped SwiGLU expert GEMM on the tensor cores (tcgen05), reading the
// rank-major receive buffer in place.  Not built yet: reports unsupported.
#include "moe_internal.cuh"

namespace moe {

cudaError_t launch_swiglu(const moe_plan&, int32_t, const void*, const int32_t*, const int32_t*,
                          const void*, const void*, void*, void*, void*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace moe
