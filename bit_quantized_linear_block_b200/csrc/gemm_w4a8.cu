// INT8-route GEMM (placeholder until the on-chip bf16 expansion kernel lands).
#include "ql_common.cuh"
#include "launchers.h"

namespace ql {
ql_status launch_gemm_w4a8(const void*, const float*, int64_t, const ql_weights*, void*, cudaStream_t,
                           int*) {
  return QL_ERR_UNSUPPORTED_SHAPE;
}
}  // namespace ql
