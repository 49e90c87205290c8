// Prefill GEMM (tcgen05) - under construction.
#include "nvq_internal.h"

namespace nvq {

size_t gemm_workspace_size(int64_t M, int64_t, int64_t K) {
  return static_cast<size_t>(M) * static_cast<size_t>(K) * 4u + 256u;
}

cudaError_t launch_gemm(const uint8_t*, const uint8_t*, float, int64_t, int64_t,
                        const int8_t*, const uint16_t*, int64_t, float*, void*,
                        cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace nvq
