// Tensor-core Hessian accumulation (placeholder until the tcgen05 kernel lands).
#include "common.cuh"

namespace gptq {

bool hessian_tc_supported(gptq_dtype, int64_t, int64_t, int64_t, const void*) { return false; }
size_t hessian_tc_workspace_bytes(int64_t, int64_t) { return 0; }
gptq_status hessian_tc(const void*, gptq_dtype, int64_t, int64_t, int64_t, float, float*, void*,
                       cudaStream_t) {
  return GPTQ_ERR_UNSUPPORTED;
}

}  // namespace gptq
