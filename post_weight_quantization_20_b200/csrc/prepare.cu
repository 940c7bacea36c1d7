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
#include "tc_common.cuh"

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

// ---------------------------------------------------------------------------
// Diagonal blocks: Cholesky factor L of the 64x64 block and T = L^-1, by four
// warps holding the block in registers (the CTA only stages it in and out).
//
// Warps 0-1 factor: thread c holds column c.  At step j the owner of column j has
// published it to shared memory; every thread forms 1/sqrt(pivot) itself, threads
// c > j apply the rank-1 update A[:, c] -= L[:, j] L[c][j] to their column as
// A[:, c] -= A[:, j] (A[c][j] / pivot), and column j, scaled, is written out as
// L[:, j].  The owner of column j+1 publishes it when its update is done.
// Warps 2-3 invert, one step behind: thread r holds row r of the forward
// substitution L B = I, and step i subtracts (L[r][i] / L[i][i]) B[i][:] from rows
// r > i, with row B[i][:] published by its owner; finally T[r][:] = B[r][:] / L[r][r].
// Every register index is static (a thread's column or row is its own), the loop
// body is short, and the steps are separated by one 128-thread barrier.  Entries
// above the diagonal hold scratch values that are never read; the outputs are
// masked to the lower triangle.
// ---------------------------------------------------------------------------
constexpr int LDS = NB + 1;   // padded row of the 64x64 shared tiles
constexpr int DF_BCAST = 2 * NB * LDS;                 // broadcast area after the two tiles
static_assert(GM_SMEM_FLOATS >= DF_BCAST + 5 * NB, "shared buffer holds the broadcasts");

__device__ __forceinline__ void df_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// 1/sqrt(p): hardware estimate refined by one Newton step
__device__ __forceinline__ float rsqrt_nr(float p) {
  const float y0 = rsqrtf(p);
  return y0 * fmaf(-0.5f * p * y0, y0, 1.5f);
}

// S: the block on entry, L on exit.  Ti: T on exit.  bc: 5 * NB floats.
__device__ __forceinline__ void quad_factor(float* S, float* Ti, float* bc, int32_t* st,
                                            const int tid) {
  float* colb = bc;               // [2][NB]: column j of the trailing matrix
  float* rowb = bc + 2 * NB;      // [2][NB]: row i of B
  float* sinv = bc + 4 * NB;      // [NB]: 1 / L[j][j]
  float v[NB];
  if (tid < NB) {
    const int c = tid;
#pragma unroll
    for (int r = 0; r < NB; ++r) v[r] = S[r * LDS + c];
    colb[c] = S[c * LDS];         // column 0 (symmetric: row 0)
  } else {
    const int r = tid - NB;
#pragma unroll
    for (int c = 0; c < NB; ++c) v[c] = (c == r) ? 1.f : 0.f;
    rowb[r] = (r == 0) ? 1.f : 0.f;
  }
  bool bad = false;
  df_bar();
#pragma unroll 1
  for (int j = 0; j <= NB; ++j) {
    if (tid < NB) {
      if (j < NB) {
        const int c = tid;
        const float* col = colb + (j & 1) * NB;
        float p = col[j];
        const bool okp = (p > 0.f) && (p < 3.0e38f);
        bad |= (c == 0) && !okp;
        p = okp ? p : 1.f;
        const float inv = rsqrt_nr(p);
        const float cc = col[c];
        S[c * LDS + j] = (c > j) ? cc * inv : ((c == j) ? p * inv : 0.f);
        if (c == 0) sinv[j] = inv;
        if (c > j) {
          const float sc = cc * inv * inv;
#pragma unroll
          for (int q = 0; q < NB / 4; ++q) {
            const float4 x = *reinterpret_cast<const float4*>(col + 4 * q);
            v[4 * q + 0] = fmaf(-x.x, sc, v[4 * q + 0]);
            v[4 * q + 1] = fmaf(-x.y, sc, v[4 * q + 1]);
            v[4 * q + 2] = fmaf(-x.z, sc, v[4 * q + 2]);
            v[4 * q + 3] = fmaf(-x.w, sc, v[4 * q + 3]);
          }
          if (c == j + 1) {
            float* nx = colb + ((j + 1) & 1) * NB;
#pragma unroll
            for (int q = 0; q < NB / 4; ++q)
              *reinterpret_cast<float4*>(nx + 4 * q) =
                  make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          }
        }
      }
    } else if (j >= 1) {
      // inverse step i = j - 1 (needs L[:, i] and 1/L[i][i], written in step i)
      const int r = tid - NB, i = j - 1;
      if (r > i) {
        const float k = S[r * LDS + i] * sinv[i];
        const float* row = rowb + (i & 1) * NB;
#pragma unroll
        for (int q = 0; q < NB / 4; ++q) {
          const float4 x = *reinterpret_cast<const float4*>(row + 4 * q);
          v[4 * q + 0] = fmaf(-k, x.x, v[4 * q + 0]);
          v[4 * q + 1] = fmaf(-k, x.y, v[4 * q + 1]);
          v[4 * q + 2] = fmaf(-k, x.z, v[4 * q + 2]);
          v[4 * q + 3] = fmaf(-k, x.w, v[4 * q + 3]);
        }
        if (r == i + 1) {
          float* nx = rowb + ((i + 1) & 1) * NB;
#pragma unroll
          for (int q = 0; q < NB / 4; ++q)
            *reinterpret_cast<float4*>(nx + 4 * q) =
                make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      }
    }
    df_bar();
  }
  if (tid >= NB) {
    const int r = tid - NB;
    const float ir = sinv[r];
#pragma unroll
    for (int c = 0; c < NB; ++c) Ti[r * LDS + c] = (c <= r) ? v[c] * ir : 0.f;
  }
  if (bad) raise_status(st, GPTQ_ERR_NOT_PD);
}

// Factor the diagonal block at (k0, k0) of A in place (L, zeros above the
// diagonal) and write T = L^-1 (64x64, row-major).  Called by all GM_THREADS
// threads of the CTA with sm = GM_SMEM_FLOATS floats of shared memory.
__device__ __forceinline__ void diag_factor(float* A, int64_t lda, int k0, float* T, int32_t* st,
                                         float* sm) {
  float* S = sm;
  float* Ti = sm + NB * LDS;
  const int tid = threadIdx.x;
#pragma unroll
  for (int x = 0; x < (NB * NB) / GM_THREADS; ++x) {
    const int e = tid + GM_THREADS * x;
    S[(e >> 6) * LDS + (e & 63)] = A[int64_t(k0 + (e >> 6)) * lda + k0 + (e & 63)];
  }
  __syncthreads();
  if (tid < 2 * NB) quad_factor(S, Ti, sm + DF_BCAST, st, tid);
  __syncthreads();
#pragma unroll
  for (int x = 0; x < (NB * NB) / GM_THREADS; ++x) {
    const int e = tid + GM_THREADS * x;
    const int r = e >> 6, c = e & 63;
    A[int64_t(k0 + r) * lda + k0 + c] = S[r * LDS + c];
    T[e] = Ti[r * LDS + c];
  }
}

// ---------------------------------------------------------------------------
// Persistent factorization + inversion.  One cooperative launch; phases are
// separated by a grid barrier whose spin is bounded (GPTQ_ERR_TIMEOUT, then
// every CTA unwinds).  Step k:
//   phase A: panel L[k0+NB:, k] = A[k0+NB:, k] T_k^T   and   X_k = T_k Bx[k, 0:k0+NB]
//   phase B: A[k0+NB:, k0+NB:] -= P P^T (lower tiles), Bx[k0+NB:, 0:k0+NB] -= P X_k;
//            CTA 0 updates the next diagonal block and factors it (lookahead).
// ---------------------------------------------------------------------------
struct FactorArgs {
  float* A;
  float* Bx;
  float* T;
  int lda;
  int nblk;
  unsigned* bar;       // monotonically increasing arrival counter (zeroed before launch)
  int* abort_flag;     // set when a barrier gave up
  int32_t* status;
};

constexpr uint32_t BARRIER_SPIN_LIMIT = 1u << 24;

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ bool grid_barrier(const FactorArgs& a, unsigned& epoch) {
  __shared__ int ok;
  __syncthreads();
  ++epoch;
  if (threadIdx.x == 0) {
    ok = 1;
    __threadfence();
    atomicAdd(a.bar, 1u);
    const unsigned target = epoch * gridDim.x;
    uint32_t it = 0;
    while (ld_acquire(a.bar) < target) {
      if (++it > BARRIER_SPIN_LIMIT || *(volatile int*)a.abort_flag) {
        if (atomicExch(a.abort_flag, 1) == 0) raise_status(a.status, GPTQ_ERR_TIMEOUT);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
    __threadfence();
  }
  __syncthreads();
  return ok != 0;
}

// lower-triangular tile t of an nr x nr tile grid: t = tm (tm + 1) / 2 + tn, tn <= tm
__device__ __forceinline__ void lower_tile(int t, int& tm, int& tn) {
  int m = int((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
  while ((m + 1) * (m + 2) / 2 <= t) ++m;
  while (m * (m + 1) / 2 > t) --m;
  tm = m;
  tn = t - m * (m + 1) / 2;
}

__global__ void __launch_bounds__(GM_THREADS, 2) k_factor_persistent(FactorArgs a) {
  // one buffer: GEMM chunks, or the tiles of the diagonal factor
  __shared__ __align__(16) float sm[GM_SMEM_FLOATS];
  const int64_t lda = a.lda;
  unsigned epoch = 0;
  if (blockIdx.x == 0) diag_factor(a.A, lda, 0, a.T, a.status, sm);
  if (!grid_barrier(a, epoch)) return;
  for (int k = 0; k < a.nblk; ++k) {
    const int k0 = k * NB;
    const float* Tk = a.T + size_t(k) * NB * NB;
    const int rest = a.lda - k0 - NB;
    const int nr = rest / NB;
    float* panel = a.A + int64_t(k0 + NB) * lda + k0;
    float* brow = a.Bx + int64_t(k0) * lda;
    // phase A
    const GemmProb pan = make_prob(rest, NB, NB, 1.f, panel, lda, 1, Tk, 1, NB, 0.f, panel, lda, 0);
    const GemmProb xk = make_prob(NB, k0 + NB, NB, 1.f, Tk, NB, 1, brow, lda, 1, 0.f, brow, lda, 0);
    for (int t = blockIdx.x; t < pan.ntiles + xk.ntiles; t += gridDim.x) {
      if (t < pan.ntiles) gemm_tile(pan, t, 0, sm);
      else gemm_tile(xk, 0, t - pan.ntiles, sm);
    }
    if (!grid_barrier(a, epoch)) return;
    if (rest == 0) break;
    // phase B
    const GemmProb syrk = make_prob(rest, rest, NB, -1.f, panel, lda, 1, panel, 1, lda, 1.f,
                                    a.A + int64_t(k0 + NB) * lda + k0 + NB, lda, 1);
    const GemmProb bup = make_prob(rest, k0 + NB, NB, -1.f, panel, lda, 1, brow, lda, 1, 1.f,
                                   a.Bx + int64_t(k0 + NB) * lda, lda, 0);
    const int n_syrk = nr * (nr + 1) / 2;
    const int n_total = n_syrk + bup.ntiles;
    if (blockIdx.x == 0) {
      gemm_tile(syrk, 0, 0, sm);
      __syncthreads();
      diag_factor(a.A, lda, k0 + NB, a.T + size_t(k + 1) * NB * NB, a.status, sm);
    }
    const int workers = gridDim.x > 1 ? gridDim.x - 1 : 1;
    const int first = gridDim.x > 1 ? int(blockIdx.x) - 1 : 0;
    if (gridDim.x == 1 || blockIdx.x > 0) {
      for (int t = 1 + first; t < n_total; t += workers) {
        if (t < n_syrk) {
          int tm, tn;
          lower_tile(t, tm, tn);
          gemm_tile(syrk, tm, tn, sm);
        } else {
          const int u = t - n_syrk;
          gemm_tile(bup, u / bup.tiles_n, u % bup.tiles_n, sm);
        }
      }
    }
    if (!grid_barrier(a, epoch)) return;
  }
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
  GPTQ_LAUNCH(k_gather_rev, grid_for(int64_t(Cp) * Cp), 256, 0, st, H, C, Cp, perm, L.lam, L.A,
              L.Bx);
  // Blocked right-looking Cholesky of A interleaved with the blocked forward
  // substitution that turns Bx = I into M^-1, in one persistent cooperative launch.
  unsigned* bar = reinterpret_cast<unsigned*>(reinterpret_cast<char*>(L.lam) + 64);
  int* abort_flag = reinterpret_cast<int*>(reinterpret_cast<char*>(L.lam) + 128);
  GPTQ_CUDA(cudaMemsetAsync(reinterpret_cast<char*>(L.lam) + 64, 0, 128, st));
  FactorArgs fa{L.A, L.Bx, L.T, Cp, L.nblk, bar, abort_flag, status};
  int per_sm = 0;
  GPTQ_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_factor_persistent,
                                                          GM_THREADS, 0));
  const int sms = sm_count();
  if (per_sm <= 0 || sms <= 0) return GPTQ_ERR_CUDA;
  // enough CTAs for the largest phase, at most what can be co-resident
  const int nr0 = Cp / NB - 1;
  const int most = std::max(1, std::max(nr0 * (nr0 + 1) / 2 + nr0, nr0 + Cp / NB));
  const int grid = std::min(std::min(per_sm, 2) * sms, most + 1);
  void* args[] = {&fa};
  GPTQ_CUDA(cudaLaunchCooperativeKernel(reinterpret_cast<void*>(k_factor_persistent), dim3(grid),
                                        dim3(GM_THREADS), args, 0, st));
  note_launch();
  GPTQ_LAUNCH(k_write_u, grid_for(int64_t(C) * C), 256, 0, st, L.Bx, Cp, C, U);
  return GPTQ_OK;
}

}  // namespace gptq
