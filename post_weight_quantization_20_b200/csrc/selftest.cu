// Self-test of the bounded device waits: an mbarrier that nothing arrives on.
// The wait is the one the tensor-core pipelines use, with a shortened limit; when
// it runs out the kernel reports GPTQ_ERR_TIMEOUT and returns (nothing is in
// flight, so the context stays usable).
#include "kernels.h"
#include "tc_common.cuh"

namespace gptq {
namespace {

constexpr uint32_t SELFTEST_WAIT_LIMIT = 1u << 16;

__global__ void k_selftest_mbarrier(int32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);   // one arrival expected; none will come
    abort_flag = 0;
    tc::fence_barrier_init();
  }
  __syncthreads();
  const bool ok = tc::mbar_wait(&bar, 0, &abort_flag, SELFTEST_WAIT_LIMIT);
  if (!ok && threadIdx.x == 0) raise_status(status, GPTQ_ERR_TIMEOUT);
}

}  // namespace

gptq_status selftest_mbarrier(cudaStream_t st, int32_t* status) {
  GPTQ_LAUNCH(k_selftest_mbarrier, 1, 32, 0, st, status);
  return GPTQ_OK;
}

}  // namespace gptq
