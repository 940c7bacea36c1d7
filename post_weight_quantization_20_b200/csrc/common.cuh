// Shared helpers of libgptq: status handling, launch accounting, element loads.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include "gptq.h"

namespace gptq {

void note_launch();  // counts every kernel launch issued by the library
void note_error(cudaError_t e, const char* where);  // remembers the last CUDA failure

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

__device__ __forceinline__ void raise_status(int32_t* st, int bits) {
  if (st) atomicOr(st, bits);
}

__device__ __forceinline__ float load_f32(const void* p, int dt, int64_t idx) {
  if (dt == GPTQ_F32) return static_cast<const float*>(p)[idx];
  if (dt == GPTQ_F16) return __half2float(static_cast<const __half*>(p)[idx]);
  return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[idx]);
}

// An NVTX range around one ABI call, so that a profiler can select a call's
// kernels (e.g. ncu --nvtx --nvtx-include "gptq_prepare/"); without a tool
// attached the push and pop return at once.
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

// Opt a kernel into more than 48 KB of dynamic shared memory (idempotent).
template <typename K>
inline cudaError_t allow_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

}  // namespace gptq

// Launch a kernel, count it, and turn a launch error into GPTQ_ERR_CUDA.
#define GPTQ_LAUNCH(kernel, grid, block, smem, stream, ...)                 \
  do {                                                                      \
    kernel<<<(grid), (block), (smem), (stream)>>>(__VA_ARGS__);             \
    ::gptq::note_launch();                                                  \
    const cudaError_t e_ = cudaGetLastError();                              \
    if (e_ != cudaSuccess) {                                                \
      ::gptq::note_error(e_, #kernel);                                      \
      return GPTQ_ERR_CUDA;                                                 \
    }                                                                       \
  } while (0)

#define GPTQ_CUDA(call)                                                     \
  do {                                                                      \
    const cudaError_t e_ = (call);                                          \
    if (e_ != cudaSuccess) {                                                \
      ::gptq::note_error(e_, #call);                                        \
      return GPTQ_ERR_CUDA;                                                 \
    }                                                                       \
  } while (0)

#define GPTQ_TRY(expr)                          \
  do {                                          \
    gptq_status s_ = (expr);                    \
    if (s_ != GPTQ_OK) return s_;               \
  } while (0)
