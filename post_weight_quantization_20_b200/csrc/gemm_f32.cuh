// Generic fp32 SIMT GEMM used by the blocked Cholesky / triangular inverse:
//   D[m][n] = beta * D[m][n] + alpha * sum_k A(m,k) * B(k,n)
// with A(m,k) = A[m*sam + k*sak], B(k,n) = B[k*sbk + n*sbn] (strides express
// transposes).  64x64 output tile per CTA, 256 threads, 4x4 outputs per thread.
// tri = 1 skips output tiles strictly above the diagonal (tile_m < tile_n).
// A CTA reads all of its K range before it writes, so D may alias an operand
// when N fits in one tile column (or M in one tile row) and the aliased operand
// covers exactly the CTA's own output tile.
#pragma once
#include "common.cuh"

namespace gptq {

constexpr int GM_BM = 64, GM_BN = 64, GM_BK = 16, GM_THREADS = 256;

static __global__ void __launch_bounds__(GM_THREADS)
k_gemm_f32(int M, int N, int K, float alpha, const float* A, int64_t sam,
           int64_t sak, const float* B, int64_t sbk, int64_t sbn, float beta,
           float* D, int64_t ldd, int tri) {
  const int tm = blockIdx.y, tn = blockIdx.x;
  if (tri && tm < tn) return;
  __shared__ float As[GM_BK][GM_BM + 4];
  __shared__ float Bs[GM_BK][GM_BN + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int m0 = tm * GM_BM, n0 = tn * GM_BN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += GM_BK) {
#pragma unroll
    for (int x = 0; x < (GM_BM * GM_BK) / GM_THREADS; ++x) {
      const int e = tid + x * GM_THREADS;
      int mm, kk;
      if (sak == 1) { mm = e / GM_BK; kk = e % GM_BK; } else { mm = e % GM_BM; kk = e / GM_BM; }
      const int gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < M && gk < K) ? A[gm * sam + gk * sak] : 0.f;
    }
#pragma unroll
    for (int x = 0; x < (GM_BN * GM_BK) / GM_THREADS; ++x) {
      const int e = tid + x * GM_THREADS;
      int nn, kk;
      if (sbn == 1) { nn = e % GM_BN; kk = e / GM_BN; } else { nn = e / GM_BK; kk = e % GM_BK; }
      const int gn = n0 + nn, gk = k0 + kk;
      Bs[kk][nn] = (gn < N && gk < K) ? B[gk * sbk + gn * sbn] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < GM_BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty + 16 * i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx + 16 * j;
      if (gn >= N) continue;
      float* d = D + gm * ldd + gn;
      *d = (beta == 0.f) ? alpha * acc[i][j] : fmaf(beta, *d, alpha * acc[i][j]);
    }
  }
}

static inline gptq_status gemm_f32(cudaStream_t st, int M, int N, int K, float alpha, const float* A,
                            int64_t sam, int64_t sak, const float* B, int64_t sbk, int64_t sbn,
                            float beta, float* D, int64_t ldd, int tri) {
  if (M <= 0 || N <= 0) return GPTQ_OK;
  dim3 grid((N + GM_BN - 1) / GM_BN, (M + GM_BM - 1) / GM_BM);
  GPTQ_LAUNCH(k_gemm_f32, grid, GM_THREADS, 0, st, M, N, K, alpha, A, sam, sak, B, sbk, sbn,
              beta, D, ldd, tri);
  return GPTQ_OK;
}

}  // namespace gptq
