// Placeholder for the tcgen05 Hessian contraction (replaced by the tensor-core kernel).
#include "common.cuh"
#include "kernels.h"

namespace gptq {
gptq_status hessian_syrk_tc(cudaStream_t, float*, const void*, int, int64_t, int, int64_t, float,
                            int32_t*) {
  return GPTQ_ERR_UNSUPPORTED;
}
}  // namespace gptq
