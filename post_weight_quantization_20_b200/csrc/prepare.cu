// Damping, column order and the inverse Cholesky factor:
//   GPTQ量化算法深度解析 §3.1 step 2, §2.4 (Cholesky), §3.3 (damp_percent, desc_act).
//
// U (upper, U^T U = Hp^-1) is obtained without forming Hp^-1.  With J the
// order-reversing permutation, factor the reversed matrix A = J Hp J = M M^T
// (M lower, blocked right-looking Cholesky), invert M by blocked forward
// substitution, and read U = J M^-1 J back reversed: Hp = V V^T with
// V = J M J upper, and U = V^-1.  Both halves cost C^3/3 flops.
//
// The factorization runs on a Cp x Cp copy (Cp = C rounded up to 64) whose
// padding is the identity, so every 64-block is full.
#include <algorithm>

#include "common.cuh"
#include "gemm_f32.cuh"
#include "kernels.h"

namespace gptq {

constexpr int NB = 64;  // diagonal block of the factorization

struct PrepLayout {
  int Cp, nblk;
  float *A, *Bx, *T, *diag, *lam;
  int32_t* cnt;
};

static PrepLayout prep_layout(void* ws, int64_t C) {
  PrepLayout L{};
  L.nblk = int((C + NB - 1) / NB);
  L.Cp = L.nblk * NB;
  const size_t cp2 = size_t(L.Cp) * L.Cp * sizeof(float);
  char* p = static_cast<char*>(ws);
  L.A = reinterpret_cast<float*>(p);            p += align256(cp2);
  L.Bx = reinterpret_cast<float*>(p);           p += align256(cp2);
  L.T = reinterpret_cast<float*>(p);            p += align256(size_t(L.nblk) * NB * NB * 4);
  L.diag = reinterpret_cast<float*>(p);         p += align256(size_t(C) * 4);
  L.lam = reinterpret_cast<float*>(p);          p += 256;
  L.cnt = reinterpret_cast<int32_t*>(p);        p += align256(size_t(C) * 4);
  return L;
}

size_t prepare_ws_bytes(int64_t C) {
  const int64_t nblk = (C + NB - 1) / NB, Cp = nblk * NB;
  const size_t cp2 = size_t(Cp) * Cp * sizeof(float);
  return 2 * align256(cp2) + align256(size_t(nblk) * NB * NB * 4) + align256(size_t(C) * 4) +
         256 + align256(size_t(C) * 4);
}

// lambda = damp * mean(diag H); flags a non-finite diagonal.
__global__ void __launch_bounds__(1024)
k_diag_lambda(const float* H, int C, float damp, float* diag, float* lam, int32_t* st) {
  __shared__ double part[32];
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  double s = 0.0;
  for (int i = threadIdx.x; i < C; i += blockDim.x) {
    const float d = H[int64_t(i) * C + i];
    diag[i] = d;
    if (!isfinite(d)) bad = 1;
    s += double(d);
  }
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0.0;
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) {
      *lam = float(double(damp) * (v / double(C)));
      if (bad) raise_status(st, GPTQ_ERR_NONFINITE);
    }
  }
}

__global__ void k_iota(int32_t* perm, int C) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < C) perm[i] = i;
}

// perm[rank(i)] = i, rank = #{j : d_j > d_i or (d_j == d_i and j < i)}: a stable
// descending order of the diagonal computed by counting.
__global__ void __launch_bounds__(256) k_rank_perm(const float* d, int C, int32_t* perm) {
  __shared__ float tile[2048];
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const float di = i < C ? d[i] : 0.f;
  int rank = 0;
  for (int j0 = 0; j0 < C; j0 += 2048) {
    __syncthreads();
    for (int k = threadIdx.x; k < 2048; k += blockDim.x) tile[k] = j0 + k < C ? d[j0 + k] : 0.f;
    __syncthreads();
    const int n = min(2048, C - j0);
    for (int k = 0; k < n; ++k) {
      const float dj = tile[k];
      rank += (dj > di) | ((dj == di) & (j0 + k < i));
    }
  }
  if (i < C && rank < C) perm[rank] = i;
}

__global__ void k_perm_count(const int32_t* perm, int C, int32_t* cnt, int32_t* st) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= C) return;
  const int p = perm[i];
  if (p < 0 || p >= C) raise_status(st, GPTQ_ERR_INVALID_ARG);
  else atomicAdd(cnt + p, 1);
}

__global__ void k_perm_check(const int32_t* cnt, int C, int32_t* st) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < C && cnt[i] != 1) raise_status(st, GPTQ_ERR_INVALID_ARG);
}

// A = J (H + lambda I)[perm][:, perm] J padded with the identity; Bx = I.
__global__ void k_gather_rev(const float* H, int C, int Cp, const int32_t* perm, const float* lam,
                             float* A, float* Bx) {
  const int64_t total = int64_t(Cp) * Cp;
  const float l = *lam;
  for (int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; idx < total;
       idx += int64_t(gridDim.x) * blockDim.x) {
    const int a = int(idx / Cp), b = int(idx % Cp);
    float v;
    if (a < C && b < C) {
      int i = perm[C - 1 - a], j = perm[C - 1 - b];
      i = min(max(i, 0), C - 1);
      j = min(max(j, 0), C - 1);
      const int lo = min(i, j), hi = max(i, j);
      v = H[int64_t(lo) * C + hi] + (a == b ? l : 0.f);
    } else {
      v = (a == b) ? 1.f : 0.f;
    }
    A[idx] = v;
    Bx[idx] = (a == b) ? 1.f : 0.f;
  }
}

// Unblocked Cholesky of the 64x64 diagonal block at (k0, k0) in shared memory,
// followed by the inverse of the factor.  Writes the factor back into A (lower,
// zeros above) and the inverse to T.  A non-positive or non-finite pivot raises
// GPTQ_ERR_NOT_PD and is replaced by 1 so no NaN spreads.
__global__ void __launch_bounds__(256)
k_potrf_diag(float* A, int64_t lda, int k0, float* T, int32_t* st) {
  __shared__ float S[NB][NB + 1];
  __shared__ float Ti[NB][NB + 1];
  __shared__ int bad;
  const int tid = threadIdx.x;
  for (int e = tid; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    S[r][c] = A[int64_t(k0 + r) * lda + k0 + c];
  }
  if (tid == 0) bad = 0;
  __syncthreads();
  for (int j = 0; j < NB; ++j) {
    if (tid == 0) {
      float p = S[j][j];
      if (!(p > 0.f) || !isfinite(p)) { bad = 1; p = 1.f; }
      S[j][j] = sqrtf(p);
    }
    __syncthreads();
    const float djj = S[j][j];
    if (tid > j && tid < NB) S[tid][j] = S[tid][j] / djj;
    __syncthreads();
    for (int e = tid; e < NB * NB; e += blockDim.x) {
      const int r = e / NB, c = e % NB;
      if (c > j && r >= c) S[r][c] = fmaf(-S[r][j], S[c][j], S[r][c]);
    }
    __syncthreads();
  }
  // inverse of the lower factor, one column per thread (forward substitution)
  if (tid < NB) {
    const int c = tid;
    for (int i = 0; i < c; ++i) Ti[i][c] = 0.f;
    Ti[c][c] = 1.f / S[c][c];
    for (int i = c + 1; i < NB; ++i) {
      float s = 0.f;
      for (int l = c; l < i; ++l) s = fmaf(S[i][l], Ti[l][c], s);
      Ti[i][c] = -s / S[i][i];
    }
  }
  __syncthreads();
  for (int e = tid; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    A[int64_t(k0 + r) * lda + k0 + c] = (c <= r) ? S[r][c] : 0.f;
    T[e] = Ti[r][c];
  }
  if (tid == 0 && bad) raise_status(st, GPTQ_ERR_NOT_PD);
}

// U[a][b] = Minv[C-1-a][C-1-b] for a <= b, 0 below the diagonal.
__global__ void k_write_u(const float* Bx, int Cp, int C, float* U) {
  const int64_t total = int64_t(C) * C;
  for (int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; idx < total;
       idx += int64_t(gridDim.x) * blockDim.x) {
    const int a = int(idx / C), b = int(idx % C);
    U[idx] = (a <= b) ? Bx[int64_t(C - 1 - a) * Cp + (C - 1 - b)] : 0.f;
  }
}

static int grid_for(int64_t n) { return int(std::min<int64_t>((n + 255) / 256, 148 * 32)); }

gptq_status prepare_run(cudaStream_t st, const float* H, int C, const gptq_config& cfg, float* U,
                        int32_t* perm, void* ws, int32_t* status) {
  PrepLayout L = prep_layout(ws, C);
  GPTQ_LAUNCH(k_diag_lambda, 1, 1024, 0, st, H, C, cfg.damp, L.diag, L.lam, status);
  const int pb = (C + 255) / 256;
  if (cfg.act_order == GPTQ_ORDER_NATURAL) {
    GPTQ_LAUNCH(k_iota, pb, 256, 0, st, perm, C);
  } else if (cfg.act_order == GPTQ_ORDER_DESC_DIAG) {
    GPTQ_LAUNCH(k_iota, pb, 256, 0, st, perm, C);
    GPTQ_LAUNCH(k_rank_perm, pb, 256, 0, st, L.diag, C, perm);
  } else {
    GPTQ_CUDA(cudaMemsetAsync(L.cnt, 0, size_t(C) * 4, st));
    GPTQ_LAUNCH(k_perm_count, pb, 256, 0, st, perm, C, L.cnt, status);
    GPTQ_LAUNCH(k_perm_check, pb, 256, 0, st, L.cnt, C, status);
  }
  const int Cp = L.Cp;
  const int64_t lda = Cp;
  GPTQ_LAUNCH(k_gather_rev, grid_for(int64_t(Cp) * Cp), 256, 0, st, H, C, Cp, perm, L.lam, L.A,
              L.Bx);
  for (int k = 0; k < L.nblk; ++k) {
    const int k0 = k * NB;
    float* Tk = L.T + size_t(k) * NB * NB;
    GPTQ_LAUNCH(k_potrf_diag, 1, 256, 0, st, L.A, lda, k0, Tk, status);
    const int rest = Cp - k0 - NB;
    float* panel = L.A + int64_t(k0 + NB) * lda + k0;
    // panel: L[k0+NB:, k-block] = A[k0+NB:, k-block] * T^T
    GPTQ_TRY(gemm_f32(st, rest, NB, NB, 1.f, panel, lda, 1, Tk, 1, NB, 0.f, panel, lda, 0));
    // trailing: A[k0+NB:, k0+NB:] -= P P^T (lower tiles)
    GPTQ_TRY(gemm_f32(st, rest, rest, NB, -1.f, panel, lda, 1, panel, 1, lda, 1.f,
                      L.A + int64_t(k0 + NB) * lda + k0 + NB, lda, 1));
    // inverse, block row k: X_k = T * B[k-block, 0:k0+NB]
    float* brow = L.Bx + int64_t(k0) * lda;
    GPTQ_TRY(gemm_f32(st, NB, k0 + NB, NB, 1.f, Tk, NB, 1, brow, lda, 1, 0.f, brow, lda, 0));
    // B[k0+NB:, 0:k0+NB] -= L[k0+NB:, k-block] * X_k
    GPTQ_TRY(gemm_f32(st, rest, k0 + NB, NB, -1.f, panel, lda, 1, brow, lda, 1, 1.f,
                      L.Bx + int64_t(k0 + NB) * lda, lda, 0));
  }
  GPTQ_LAUNCH(k_write_u, grid_for(int64_t(C) * C), 256, 0, st, L.Bx, Cp, C, U);
  return GPTQ_OK;
}

}  // namespace gptq
