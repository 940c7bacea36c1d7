// Hessian accumulation, GPTQ量化算法深度解析 §3.1 step 1:
//   H <- H * n/(n+m) + (2/(n+m)) * X^T X     (upper triangle only)
// The running-mean scale is applied by a pre-pass over the upper triangle; the
// contraction then adds (2/(n+m)) * X^T X with fp32 atomics so that token
// splits of one tile can land in any order.  This file holds the SIMT fp32
// contraction (any element type and stride); 16-bit X with TMA-compatible
// strides goes to the tcgen05 kernel in hessian_tc.cu.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace gptq {

__global__ void k_hess_prescale(float* H, int C, float alpha, int overwrite) {
  const int64_t total = int64_t(C) * C;
  for (int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; idx < total;
       idx += int64_t(gridDim.x) * blockDim.x) {
    const int i = int(idx / C), j = int(idx % C);
    if (i <= j) H[idx] = overwrite ? 0.f : H[idx] * alpha;
  }
}

// Decode the p-th upper-triangular tile pair (bi <= bj), p = bj(bj+1)/2 + bi.
__device__ __forceinline__ void upper_pair(int p, int* bi, int* bj) {
  int j = int((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);
  while ((j + 1) * (j + 2) / 2 <= p) ++j;
  while (j * (j + 1) / 2 > p) --j;
  *bj = j;
  *bi = p - j * (j + 1) / 2;
}

constexpr int HS_T = 32;  // tokens per smem stage

template <int DT>
__global__ void __launch_bounds__(256)
k_hess_syrk_simt(float* H, const void* X, int64_t m, int C, int64_t ldx, float beta,
                 int64_t tok_per_split) {
  int bi, bj;
  upper_pair(blockIdx.x, &bi, &bj);
  const int i0 = bi * 64, j0 = bj * 64;
  const int64_t tb = int64_t(blockIdx.y) * tok_per_split;
  const int64_t te = min(m, tb + tok_per_split);
  __shared__ float As[HS_T][64 + 1];
  __shared__ float Bs[HS_T][64 + 1];
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  float acc[4][4] = {};
  for (int64_t t0 = tb; t0 < te; t0 += HS_T) {
#pragma unroll
    for (int x = 0; x < (HS_T * 64) / 256; ++x) {
      const int e = tid + 256 * x;
      const int tt = e / 64, cc = e % 64;
      const int64_t t = t0 + tt;
      const bool tv = t < te;
      As[tt][cc] = (tv && i0 + cc < C) ? load_f32(X, DT, t * ldx + i0 + cc) : 0.f;
      Bs[tt][cc] = (tv && j0 + cc < C) ? load_f32(X, DT, t * ldx + j0 + cc) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int tt = 0; tt < HS_T; ++tt) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[tt][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[tt][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gi = i0 + ty + 16 * i;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gj = j0 + tx + 16 * j;
      if (gi <= gj && gj < C) atomicAdd(H + int64_t(gi) * C + gj, beta * acc[i][j]);
    }
  }
}

gptq_status hessian_prescale(cudaStream_t st, float* H, int C, double alpha, bool overwrite) {
  const int64_t total = int64_t(C) * C;
  int blocks = int(std::min<int64_t>((total + 255) / 256, 148 * 16));
  GPTQ_LAUNCH(k_hess_prescale, blocks, 256, 0, st, H, C, float(alpha), overwrite ? 1 : 0);
  return GPTQ_OK;
}

gptq_status hessian_syrk_simt(cudaStream_t st, float* H, const void* X, int dt, int64_t m, int C,
                              int64_t ldx, float beta) {
  const int nt = (C + 63) / 64;
  const int pairs = nt * (nt + 1) / 2;
  const int64_t want = 148 * 8;
  int64_t splits = std::max<int64_t>(1, want / pairs);
  splits = std::min<int64_t>(splits, (m + HS_T - 1) / HS_T);
  splits = std::min<int64_t>(splits, 65535);
  int64_t per = (m + splits - 1) / splits;
  per = (per + HS_T - 1) / HS_T * HS_T;
  splits = (m + per - 1) / per;
  dim3 grid(pairs, unsigned(splits));
  if (dt == GPTQ_F32) {
    GPTQ_LAUNCH(k_hess_syrk_simt<GPTQ_F32>, grid, 256, 0, st, H, X, m, C, ldx, beta, per);
  } else if (dt == GPTQ_F16) {
    GPTQ_LAUNCH(k_hess_syrk_simt<GPTQ_F16>, grid, 256, 0, st, H, X, m, C, ldx, beta, per);
  } else {
    GPTQ_LAUNCH(k_hess_syrk_simt<GPTQ_BF16>, grid, 256, 0, st, H, X, m, C, ldx, beta, per);
  }
  return GPTQ_OK;
}

}  // namespace gptq
