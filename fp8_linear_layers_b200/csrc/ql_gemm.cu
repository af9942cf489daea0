// ql_gemm.cu -- large-M tcgen05 GEMM (being written).
#include "ql_common.cuh"
#include "ql_internal.h"

namespace ql {
size_t gemm_workspace_bytes(ql_scheme, int64_t, int64_t, int64_t, int) { return 0; }
cudaError_t launch_gemm(ql_scheme, const void*, const float*, const void*, const float*, int64_t,
                        int64_t, int64_t, uint16_t*, void*, size_t, const ql_debug*, int,
                        DevStatus*, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace ql
