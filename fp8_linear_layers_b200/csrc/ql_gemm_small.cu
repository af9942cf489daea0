// ql_gemm_small.cu -- small-M tcgen05 GEMM (being written).
#include "ql_common.cuh"
#include "ql_internal.h"

namespace ql {
size_t gemm_small_workspace_bytes(ql_scheme, int64_t, int64_t, int64_t, int) { return 0; }
cudaError_t launch_gemm_small(ql_scheme, const uint16_t*, const void*, const float*, int64_t,
                              int64_t, int64_t, uint16_t*, void*, size_t, const ql_debug*, int,
                              DevStatus*, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace ql
