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

constexpr int GM_BM = 64, GM_BN = 64, GM_BK = 64, GM_THREADS = 256;
constexpr int GM_LD = 68;                               // padded smem row (floats)
constexpr int GM_SMEM_FLOATS = 2 * GM_BK * GM_LD;       // A and B chunks

// One GEMM problem: D = beta*D + alpha*A*B over an M x N output.
struct GemmProb {
  int M, N, K;
  float alpha, beta;
  const float* A;
  int64_t sam, sak;
  const float* B;
  int64_t sbk, sbn;
  float* D;
  int64_t ldd;
  int tri;       // skip output tiles strictly above the diagonal
  int tiles_n;   // tiles along N
  int ntiles;    // tiles_m * tiles_n (0 when M or N is 0)
};

static inline __host__ __device__ GemmProb make_prob(int M, int N, int K, float alpha, const float* A, int64_t sam,
                                 int64_t sak, const float* B, int64_t sbk, int64_t sbn, float beta,
                                 float* D, int64_t ldd, int tri) {
  GemmProb p{M, N, K, alpha, beta, A, sam, sak, B, sbk, sbn, D, ldd, tri, 0, 0};
  if (M > 0 && N > 0) {
    p.tiles_n = (N + GM_BN - 1) / GM_BN;
    p.ntiles = ((M + GM_BM - 1) / GM_BM) * p.tiles_n;
  }
  return p;
}

// The CTA's 64x64 output tile (tm, tn) of problem p; all of K is read before D is
// written.  K is consumed in 64-wide chunks: each chunk of A and B is loaded in
// one round (16 independent loads per thread), then 64 rank-1 steps read the
// shared tiles as float4 (thread (ty, tx) owns rows 4ty..4ty+3, cols 4tx..4tx+3).
// sm: GM_SMEM_FLOATS floats of shared memory.
static __device__ __forceinline__ void gemm_tile(const GemmProb& p, int tm, int tn, float* sm) {
  float* As = sm;                  // [k][m], stride GM_LD
  float* Bs = sm + GM_BK * GM_LD;  // [k][n], stride GM_LD
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int m0 = tm * GM_BM, n0 = tn * GM_BN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < p.K; k0 += GM_BK) {
#pragma unroll
    for (int x = 0; x < (GM_BM * GM_BK) / GM_THREADS; ++x) {
      const int e = tid + x * GM_THREADS;
      int mm, kk;
      if (p.sak == 1) { mm = e >> 6; kk = e & 63; } else { mm = e & 63; kk = e >> 6; }
      const int gm = m0 + mm, gk = k0 + kk;
      As[kk * GM_LD + mm] = (gm < p.M && gk < p.K) ? p.A[gm * p.sam + gk * p.sak] : 0.f;
    }
#pragma unroll
    for (int x = 0; x < (GM_BN * GM_BK) / GM_THREADS; ++x) {
      const int e = tid + x * GM_THREADS;
      int nn, kk;
      if (p.sbn == 1) { nn = e & 63; kk = e >> 6; } else { nn = e >> 6; kk = e & 63; }
      const int gn = n0 + nn, gk = k0 + kk;
      Bs[kk * GM_LD + nn] = (gn < p.N && gk < p.K) ? p.B[gk * p.sbk + gn * p.sbn] : 0.f;
    }
    __syncthreads();
#pragma unroll 16
    for (int kk = 0; kk < GM_BK; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(As + kk * GM_LD + 4 * ty);
      const float4 b = *reinterpret_cast<const float4*>(Bs + kk * GM_LD + 4 * tx);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + 4 * ty + i;
    if (gm >= p.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + 4 * tx + j;
      if (gn >= p.N) continue;
      float* d = p.D + gm * p.ldd + gn;
      *d = (p.beta == 0.f) ? p.alpha * acc[i][j] : fmaf(p.beta, *d, p.alpha * acc[i][j]);
    }
  }
}

static __global__ void __launch_bounds__(GM_THREADS) k_gemm_f32(GemmProb p) {
  const int tm = blockIdx.y, tn = blockIdx.x;
  if (p.tri && tm < tn) return;
  __shared__ __align__(16) float sm[GM_SMEM_FLOATS];
  gemm_tile(p, tm, tn, sm);
}

static inline gptq_status gemm_f32(cudaStream_t st, int M, int N, int K, float alpha, const float* A,
                            int64_t sam, int64_t sak, const float* B, int64_t sbk, int64_t sbn,
                            float beta, float* D, int64_t ldd, int tri) {
  if (M <= 0 || N <= 0) return GPTQ_OK;
  dim3 grid((N + GM_BN - 1) / GM_BN, (M + GM_BM - 1) / GM_BM);
  GPTQ_LAUNCH(k_gemm_f32, grid, GM_THREADS, 0, st,
              make_prob(M, N, K, alpha, A, sam, sak, B, sbk, sbn, beta, D, ldd, tri));
  return GPTQ_OK;
}

}  // namespace gptq
