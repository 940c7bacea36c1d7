// The operand U of the lazy trailing update W[:, e:] -= Err U[blk, e:]
// (GPTQ量化算法深度解析 §2.4), prepared once per layer for the 3xTF32 products of
// gemm_tc.cu: split as U = hi + lo (hi = U with its low 13 mantissa bits cleared,
// exact in tf32; lo = U - hi) and transposed (Ut[n][k] = U[k][n]) so that the
// product reads it K-major.  The sweep writes the errors already split.
#include <algorithm>

#include "kernels.h"
#include "tc_common.cuh"

namespace gptq {
namespace {

// Transposing split of the C x C matrix U: hi[n][k] = U[k][n] with its low 13
// mantissa bits cleared (exact in tf32), lo[n][k] = U[k][n] - hi[n][k].
// 32 x 32 tiles through shared memory keep both sides coalesced.
__global__ void k_split_tf32_t(const float* U, int C, float* hi, float* lo) {
  __shared__ float tile[32][33];
  const int k0 = blockIdx.y * 32, n0 = blockIdx.x * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;   // 32 x 8
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    const int k = k0 + ty + i, n = n0 + tx;
    tile[ty + i][tx] = (k < C && n < C) ? U[int64_t(k) * C + n] : 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    const int n = n0 + ty + i, k = k0 + tx;
    if (n < C && k < C) {
      const float v = tile[tx][ty + i];
      const float h = __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
      hi[int64_t(n) * C + k] = h;
      lo[int64_t(n) * C + k] = v - h;
    }
  }
}

}  // namespace

bool trailing_tc_supported(int C) {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  return major == 10 && minor == 0 && (C % 4) == 0 && encode_tiled_fn() != nullptr;
}

gptq_status split_tf32_t(cudaStream_t st, const float* U, int C, float* hi, float* lo) {
  if (C <= 0) return GPTQ_OK;
  dim3 grid((C + 31) / 32, (C + 31) / 32), block(32, 8);
  GPTQ_LAUNCH(k_split_tf32_t, grid, block, 0, st, U, C, hi, lo);
  return GPTQ_OK;
}

}  // namespace gptq
