// Q-ARVD integer GEMM (placeholder until the kind::i8 kernel lands).
#include "ql_common.cuh"
#include "launchers.h"

namespace ql {
ql_status launch_gemm_qarvd(const void*, const float*, int64_t, const ql_weights*, void*, cudaStream_t,
                            int*) {
  return QL_ERR_UNSUPPORTED_SHAPE;
}
}  // namespace ql
