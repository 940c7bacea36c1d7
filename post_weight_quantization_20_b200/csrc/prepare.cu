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
#include <climits>

#include "common.cuh"
#include "gemm_f32.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace gptq {

constexpr int NB = 64;  // diagonal block of the factorization

constexpr int MAX_FACTOR_GRID = 1024;   // CTAs of the persistent factorization (at most)

// Above OUTER_MIN_COLS columns the factorization is blocked twice: the persistent
// kernel runs OUTER_BLOCKS 64-column steps at a time inside an outer panel, and two
// tensor-core products with K = 64 * OUTER_BLOCKS update the rest.
constexpr int OUTER_BLOCKS = 8;
constexpr int OUTER_K = OUTER_BLOCKS * 64;
constexpr int OUTER_MIN_COLS = 3584;   // measured: at 3072 columns one launch is faster

struct PrepLayout {
  int Cp, nblk;
  float *A, *Bx, *T, *diag, *lam;
  int32_t* cnt;
  int32_t* smid;   // [MAX_FACTOR_GRID]: the SM each CTA of the factorization runs on
  float *Lh, *Ll, *Mh, *Ml;   // outer path: TF32 splits, Cp x OUTER_K each (else null)
};

static bool outer_path(int64_t Cp) { return Cp > OUTER_MIN_COLS; }

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
  L.smid = reinterpret_cast<int32_t*>(p);       p += align256(size_t(MAX_FACTOR_GRID) * 4);
  if (outer_path(L.Cp)) {
    const size_t sz = align256(size_t(L.Cp) * OUTER_K * 4);
    L.Lh = reinterpret_cast<float*>(p);         p += sz;
    L.Ll = reinterpret_cast<float*>(p);         p += sz;
    L.Mh = reinterpret_cast<float*>(p);         p += sz;
    L.Ml = reinterpret_cast<float*>(p);         p += sz;
  }
  return L;
}

size_t prepare_ws_bytes(int64_t C) {
  const int64_t nblk = (C + NB - 1) / NB, Cp = nblk * NB;
  const size_t cp2 = size_t(Cp) * Cp * sizeof(float);
  return 2 * align256(cp2) + align256(size_t(nblk) * NB * NB * 4) + align256(size_t(C) * 4) +
         256 + align256(size_t(C) * 4) + align256(size_t(MAX_FACTOR_GRID) * 4) +
         (outer_path(Cp) ? 4 * align256(size_t(Cp) * OUTER_K * 4) : 0);
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

// The same gather in three coalesced passes, for C up to the columns whose row fits
// in shared memory (the one-pass gather above reads H column-scattered, ~10x its bytes):
//   1. S = H with its lower triangle filled from the upper (32 x 32 tiles, the lower
//      ones transposed through shared memory), into the Bx buffer;
//   2. A[a][:] = S[i][perm[C-1-b]] with i = perm[C-1-a]: one CTA per row a stages
//      row i of S in shared memory and writes row a of A in order (lambda on the
//      diagonal, identity padding);
//   3. Bx = I.
constexpr int GATHER_SMEM_MAX_COLS = 56 * 1024;

__global__ void k_sym_full(const float* H, int C, float* S, int lds) {
  __shared__ float t[32][33];
  const int bi = blockIdx.y, bj = blockIdx.x;       // output tile (rows bi, cols bj)
  const int tx = threadIdx.x, ty = threadIdx.y;      // 32 x 8
  const int si = bi <= bj ? bi : bj, sj = bi <= bj ? bj : bi;   // the upper source tile
#pragma unroll
  for (int k = 0; k < 32; k += 8) {
    const int r = si * 32 + ty + k, c = sj * 32 + tx;
    t[ty + k][tx] = (r < C && c < C) ? H[int64_t(r) * C + c] : 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 32; k += 8) {
    const int rr = ty + k, cc = tx;                  // position inside the output tile
    const int r = bi * 32 + rr, c = bj * 32 + cc;
    if (r >= C || c >= C) continue;
    float v;
    if (bi < bj) v = t[rr][cc];
    else if (bi > bj) v = t[cc][rr];
    else v = rr <= cc ? t[rr][cc] : t[cc][rr];
    S[int64_t(r) * lds + c] = v;
  }
}

__global__ void __launch_bounds__(1024)
k_gather_rows(const float* S, int lds, int C, int Cp, const int32_t* perm, const float* lam,
              float* A) {
  extern __shared__ float srow[];
  const int a = blockIdx.x;
  float* arow = A + int64_t(a) * Cp;
  if (a >= C) {
    for (int b = threadIdx.x; b < Cp; b += blockDim.x) arow[b] = (a == b) ? 1.f : 0.f;
    return;
  }
  int i = perm[C - 1 - a];
  i = min(max(i, 0), C - 1);
  // the whole padded row (lds floats, lds % 4 == 0, 16-byte aligned rows) in 16-byte loads
  const float4* src = reinterpret_cast<const float4*>(S + int64_t(i) * lds);
  float4* s4 = reinterpret_cast<float4*>(srow);
  for (int b = threadIdx.x; b < lds / 4; b += blockDim.x) s4[b] = src[b];
  __syncthreads();
  const float l = *lam;
  for (int b = threadIdx.x; b < Cp; b += blockDim.x) {
    float v;
    if (b < C) {
      int j = perm[C - 1 - b];
      j = min(max(j, 0), C - 1);
      v = srow[j] + (a == b ? l : 0.f);
    } else {
      v = (a == b) ? 1.f : 0.f;
    }
    arow[b] = v;
  }
}

__global__ void k_unit_diag(float* Bx, int Cp) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < Cp) Bx[int64_t(i) * Cp + i] = 1.f;
}

// ---------------------------------------------------------------------------
// Diagonal blocks: Cholesky factor L of the 64x64 block and T = L^-1 by one CTA
// holding the block in registers, four columns per step.
//
// Warps 0-3 factor: thread (c, h) holds rows 32h .. 32h+31 of column c of the
// trailing matrix.  At block step b (columns j0 = 4b .. j0+3) the owners of those
// columns have published them, P (64 x 4, P[r][q] = A[r][j0+q]).  Every thread
// factors the 4x4 pivot block P1 = L11 L11^T itself and forms M = L11^-1 and
// W = P1^-1 = M^T M.  Then, with p_c = P[c][:] the own row of P,
//   L[c][j0..j0+3] = M p_c               (this is L11's row for c in the block)
//   A[:, c]       -= P (W p_c)           (c > j0+3: the rank-4 trailing update)
// and the owners of the next four columns publish them.
// Warps 4-7 invert, one block step behind: thread (r, h) holds columns
// 32h .. 32h+31 of row r of the forward substitution L B = I.  With B_blk the four
// published rows j0..j0+3,
//   B[r] -= (W p_r)^T B_blk                    for r > j0+3,
//   B[r] -= (e_{r-j0} - M[r-j0][:])^T B_blk   for r in the block,
// which leaves T = L^-1 in the rows when the last block is done.  The factor
// threads hand the coefficient vectors over through shared memory.
// Every register index is static, the loop body is short, and block steps are
// separated by one CTA barrier.  Entries above the diagonal hold scratch values
// that are never read; the outputs are masked to the lower triangle.
// ---------------------------------------------------------------------------
constexpr int LDS = NB + 1;   // padded row of the 64x64 shared tiles
constexpr int KB = 4;         // columns per block step
constexpr int NSTEP = NB / KB;
constexpr int HR = NB / 2;    // rows (or columns) per thread
// broadcasts P [2][KB][NB], Bp [2][KB][NB], cw [2][NB][KB]; they live in the T
// tile, which is written only after the last step
constexpr int DF_BCAST_FLOATS = 3 * 2 * KB * NB;
static_assert(DF_BCAST_FLOATS <= NB * LDS, "the T tile holds the broadcasts");
static_assert((NB * LDS) % 4 == 0, "the T tile is 16-byte aligned");
static_assert(GM_THREADS == 4 * NB, "two roles x two halves x NB threads");

// 1/sqrt(p): hardware estimate refined by one Newton step
__device__ __forceinline__ float rsqrt_nr(float p) {
  const float y0 = rsqrtf(p);
  return y0 * fmaf(-0.5f * p * y0, y0, 1.5f);
}

// 1/sqrt of a pivot; a pivot that is not positive and finite is flagged and
// replaced by 1 so that the step stays finite.
__device__ __forceinline__ float pivot_rsqrt(float p, bool& bad) {
  const bool ok = (p > 0.f) && (p < 3.0e38f);
  bad |= !ok;
  return rsqrt_nr(ok ? p : 1.f);
}

__device__ __forceinline__ void put4(float* dst, const float* v) {
#pragma unroll
  for (int g = 0; g < HR / 4; ++g)
    *reinterpret_cast<float4*>(dst + 4 * g) = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
}

// v[i] -= sum_q c[q] X[q][i] for the thread's 32 entries; X: KB rows of stride NB
__device__ __forceinline__ void rank4(float* v, const float* X, const float (&c)[KB]) {
#pragma unroll
  for (int g = 0; g < HR / 4; ++g) {
    const float4 x0 = *reinterpret_cast<const float4*>(X + 0 * NB + 4 * g);
    const float4 x1 = *reinterpret_cast<const float4*>(X + 1 * NB + 4 * g);
    const float4 x2 = *reinterpret_cast<const float4*>(X + 2 * NB + 4 * g);
    const float4 x3 = *reinterpret_cast<const float4*>(X + 3 * NB + 4 * g);
    v[4 * g + 0] = fmaf(-c[0], x0.x, fmaf(-c[1], x1.x, fmaf(-c[2], x2.x, fmaf(-c[3], x3.x, v[4 * g + 0]))));
    v[4 * g + 1] = fmaf(-c[0], x0.y, fmaf(-c[1], x1.y, fmaf(-c[2], x2.y, fmaf(-c[3], x3.y, v[4 * g + 1]))));
    v[4 * g + 2] = fmaf(-c[0], x0.z, fmaf(-c[1], x1.z, fmaf(-c[2], x2.z, fmaf(-c[3], x3.z, v[4 * g + 2]))));
    v[4 * g + 3] = fmaf(-c[0], x0.w, fmaf(-c[1], x1.w, fmaf(-c[2], x2.w, fmaf(-c[3], x3.w, v[4 * g + 3]))));
  }
}

// S: the block on entry, L on exit.  Ti: T on exit, and the broadcasts before.
// Called by all GM_THREADS threads.
__device__ __forceinline__ void block_factor(float* S, float* Ti, int32_t* st, const int tid) {
  float* Pb = Ti;                        // [2][KB][NB]
  float* Bb = Ti + 2 * KB * NB;          // [2][KB][NB]
  float* cwb = Ti + 4 * KB * NB;         // [2][NB][KB]
  const bool fac = tid < 2 * NB;
  const int own = tid & (NB - 1);        // column (factor) or row (inverse) index
  const int h = (tid >> 6) & 1;          // which half of it
  float v[HR];
  bool bad = false;
  if (fac) {
#pragma unroll
    for (int i = 0; i < HR; ++i) v[i] = S[(HR * h + i) * LDS + own];
  } else {
#pragma unroll
    for (int i = 0; i < HR; ++i) v[i] = (HR * h + i == own) ? 1.f : 0.f;
  }
  __syncthreads();                       // S is read before the broadcasts start
  if (own < KB) put4((fac ? Pb : Bb) + own * NB + HR * h, v);
  __syncthreads();
#pragma unroll 1
  for (int b = 0; b <= NSTEP; ++b) {
    if (fac) {
      if (b < NSTEP) {
        const int c = own, j0 = KB * b, cq = c - j0;
        const float* P = Pb + (b & 1) * KB * NB;
        // the pivot block (lower part) and the thread's own row of P
        float a[KB][KB], pc[KB];
#pragma unroll
        for (int q = 0; q < KB; ++q) {
          const float4 x = *reinterpret_cast<const float4*>(P + q * NB + j0);
          a[0][q] = x.x; a[1][q] = x.y; a[2][q] = x.z; a[3][q] = x.w;   // a[row][col]
          pc[q] = P[q * NB + c];
        }
        // L11 (lower) and its diagonal reciprocals
        float l[KB][KB], id[KB];
#pragma unroll
        for (int q = 0; q < KB; ++q) {
          float d = a[q][q];
#pragma unroll
          for (int k = 0; k < q; ++k) d = fmaf(-l[q][k], l[q][k], d);
          id[q] = pivot_rsqrt(d, bad);
          l[q][q] = d * id[q];
#pragma unroll
          for (int r = q + 1; r < KB; ++r) {
            float x = a[r][q];
#pragma unroll
            for (int k = 0; k < q; ++k) x = fmaf(-l[r][k], l[q][k], x);
            l[r][q] = x * id[q];
          }
        }
        // M = L11^-1 (lower)
        float m[KB][KB];
#pragma unroll
        for (int q = 0; q < KB; ++q) {
          m[q][q] = id[q];
#pragma unroll
          for (int r = q + 1; r < KB; ++r) {
            float x = 0.f;
#pragma unroll
            for (int k = q; k < r; ++k) x = fmaf(l[r][k], m[k][q], x);
            m[r][q] = -x * id[r];
          }
        }
        // own row of L: M p_c;  coefficients W p_c = M^T (M p_c)
        float lr[KB], w[KB];
#pragma unroll
        for (int q = 0; q < KB; ++q) {
          float x = 0.f;
#pragma unroll
          for (int k = 0; k <= q; ++k) x = fmaf(m[q][k], pc[k], x);
          lr[q] = x;
        }
#pragma unroll
        for (int q = 0; q < KB; ++q) {
          float x = 0.f;
#pragma unroll
          for (int k = q; k < KB; ++k) x = fmaf(m[k][q], lr[k], x);
          w[q] = x;
        }
        const bool below = cq >= KB, inblk = (cq >= 0) && !below;
        if (h == 0) {
          // coefficients for the inverse threads (row c of B), and L[c][j0..j0+3]
          float cw[KB];
#pragma unroll
          for (int q = 0; q < KB; ++q) {
            float mi = 0.f;
#pragma unroll
            for (int k = q; k < KB; ++k) mi = (cq == k) ? m[k][q] : mi;   // M is lower
            cw[q] = below ? w[q] : (inblk ? ((cq == q ? 1.f : 0.f) - mi) : 0.f);
          }
          *reinterpret_cast<float4*>(cwb + (b & 1) * NB * KB + c * KB) =
              make_float4(cw[0], cw[1], cw[2], cw[3]);
#pragma unroll
          for (int q = 0; q < KB; ++q)
            S[c * LDS + j0 + q] = (below || (inblk && q <= cq)) ? lr[q] : 0.f;
        }
        // rank-4 update of the thread's column; columns at or left of the block
        // take zero coefficients
#pragma unroll
        for (int q = 0; q < KB; ++q) w[q] = below ? w[q] : 0.f;
        rank4(v, P + HR * h, w);
        // the owners of the next block's columns publish them
        if (cq >= KB && cq < 2 * KB) put4(Pb + ((b + 1) & 1) * KB * NB + (cq - KB) * NB + HR * h, v);
      }
    } else if (b >= 1) {
      // inverse step for block b - 1
      const int r = own, bb = b - 1, j0 = KB * bb, rq = r - j0;
      const float4 cv = *reinterpret_cast<const float4*>(cwb + (bb & 1) * NB * KB + r * KB);
      const float cw[KB] = {cv.x, cv.y, cv.z, cv.w};
      rank4(v, Bb + (bb & 1) * KB * NB + HR * h, cw);
      if (rq >= KB && rq < 2 * KB) put4(Bb + (b & 1) * KB * NB + (rq - KB) * NB + HR * h, v);
    }
    __syncthreads();
  }
  if (!fac) {
#pragma unroll
    for (int i = 0; i < HR; ++i) Ti[own * LDS + HR * h + i] = (HR * h + i <= own) ? v[i] : 0.f;
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
  block_factor(S, Ti, st, tid);
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
  int32_t* smid;       // [gridDim.x]
  int kb, ke;          // the 64-column steps this launch runs, [kb, ke)
  int lim;             // outer limit in blocks: SYRK columns and M^-1 rows stay below it
};

// Spins of a grid-barrier wait before it gives up (each a ~64 ns sleep and an
// acquire load from L2: about a second).  A legitimate wait is at most one phase
// of tiles, a few milliseconds even at C = 49152.
constexpr uint32_t BARRIER_SPIN_LIMIT = 1u << 21;

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

// Self-test: CTA 1 leaves without arriving, so CTA 0's barrier wait runs out (it
// then sets the abort flag and GPTQ_ERR_TIMEOUT).  The slot holds the counter at
// +0 and the abort flag at +64; the host zeroes it first.
__global__ void k_selftest_grid_barrier(unsigned* slot, int32_t* status) {
  if (blockIdx.x != 0) return;
  FactorArgs a{};
  a.bar = slot;
  a.abort_flag = reinterpret_cast<int*>(reinterpret_cast<char*>(slot) + 64);
  a.status = status;
  unsigned epoch = 0;
  grid_barrier(a, epoch);
}

// lower-triangular tile t of an nr x nr tile grid: t = tm (tm + 1) / 2 + tn, tn <= tm
__device__ __forceinline__ void lower_tile(int t, int& tm, int& tn) {
  int m = int((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
  while ((m + 1) * (m + 2) / 2 <= t) ++m;
  while (m * (m + 1) / 2 > t) --m;
  tm = m;
  tn = t - m * (m + 1) / 2;
}

// ---------------------------------------------------------------------------
// The products of the factorization: 64x64 output tiles with K = 64, software
// pipelined across a CTA's tiles.  A tile's operands (and its output, when the
// tile accumulates into it) are fetched into registers while the CTA's previous
// tile computes.  A is row-major (m, k); B is row-major (k, n) or stored (n, k);
// an operand stored with k contiguous is read as float4 along k and transposed on
// its way to shared memory (consecutive threads take consecutive rows, so the
// stores hit distinct banks).  All extents are multiples of 64 and every tile
// origin is 16-byte aligned (the factorization runs on a Cp x Cp copy, Cp a
// multiple of 64).  A tile reads all of its operands before it writes, so its
// output may overwrite an operand tile it alone reads (the in-place panel solve).
// ---------------------------------------------------------------------------
struct Tile64 {
  const float* a;
  const float* b;
  float* d;
  int64_t lda_, ldb, ldd;
  float alpha;
  bool bt;    // B stored (n, k)
  bool acc;   // D += alpha A B (else D = alpha A B)
};

struct Fetch64 {
  float4 a[4], b[4], d[4];
};

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }

__device__ __forceinline__ void fetch64(const Tile64& T, Fetch64& f) {
  const int tid = threadIdx.x, rm = tid & 63, rq = tid >> 6;      // row, k-quad
#pragma unroll
  for (int i = 0; i < 4; ++i) f.a[i] = ld4(T.a + rm * T.lda_ + 4 * (rq + 4 * i));
  if (T.bt) {
#pragma unroll
    for (int i = 0; i < 4; ++i) f.b[i] = ld4(T.b + rm * T.ldb + 4 * (rq + 4 * i));
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) f.b[i] = ld4(T.b + ((tid >> 4) + 16 * i) * T.ldb + 4 * (tid & 15));
  }
  if (T.acc) {
    const int tx = tid & 15, ty = tid >> 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) f.d[i] = ld4(T.d + (4 * ty + i) * T.ldd + 4 * tx);
  }
}

// registers -> shared: As[k][m], Bs[k][n]
__device__ __forceinline__ void stash64(bool bt, const Fetch64& f, float* sm) {
  float* As = sm;
  float* Bs = sm + GM_BK * GM_LD;
  const int tid = threadIdx.x, rm = tid & 63, rq = tid >> 6;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int k = 4 * (rq + 4 * i);
    As[(k + 0) * GM_LD + rm] = f.a[i].x;
    As[(k + 1) * GM_LD + rm] = f.a[i].y;
    As[(k + 2) * GM_LD + rm] = f.a[i].z;
    As[(k + 3) * GM_LD + rm] = f.a[i].w;
  }
  if (bt) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int k = 4 * (rq + 4 * i);
      Bs[(k + 0) * GM_LD + rm] = f.b[i].x;
      Bs[(k + 1) * GM_LD + rm] = f.b[i].y;
      Bs[(k + 2) * GM_LD + rm] = f.b[i].z;
      Bs[(k + 3) * GM_LD + rm] = f.b[i].w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<float4*>(Bs + ((tid >> 4) + 16 * i) * GM_LD + 4 * (tid & 15)) = f.b[i];
  }
}

// Runs work items t, t + step, ... < end; map(t) gives the item's tile.  Called
// uniformly by the whole CTA; leaves sm free for reuse on return.
template <class Map>
__device__ __forceinline__ void run_tiles64(int t, int step, int end, const Map& map, float* sm) {
  if (t >= end) return;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  Tile64 T = map(t);
  Fetch64 f;
  fetch64(T, f);
  for (;;) {
    __syncthreads();                       // the previous tile is done with sm
    stash64(T.bt, f, sm);
    float4 dold[4] = {f.d[0], f.d[1], f.d[2], f.d[3]};
    float* const d = T.d;
    const int64_t ldd = T.ldd;
    const float alpha = T.alpha;
    const bool acc = T.acc;
    __syncthreads();
    const int tnext = t + step;
    if (tnext < end) {
      T = map(tnext);
      fetch64(T, f);
    }
    const float* As = sm;
    const float* Bs = sm + GM_BK * GM_LD;
    float c[4][4] = {};
#pragma unroll 16
    for (int kk = 0; kk < GM_BK; ++kk) {
      const float4 x = *reinterpret_cast<const float4*>(As + kk * GM_LD + 4 * ty);
      const float4 y = *reinterpret_cast<const float4*>(Bs + kk * GM_LD + 4 * tx);
      const float xv[4] = {x.x, x.y, x.z, x.w};
      const float yv[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) c[i][j] = fmaf(xv[i], yv[j], c[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float4 o = make_float4(alpha * c[i][0], alpha * c[i][1], alpha * c[i][2], alpha * c[i][3]);
      if (acc) {
        o.x += dold[i].x; o.y += dold[i].y; o.z += dold[i].z; o.w += dold[i].w;
      }
      *reinterpret_cast<float4*>(d + (4 * ty + i) * ldd + 4 * tx) = o;
    }
    if (tnext >= end) break;
    t = tnext;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(GM_THREADS, 2) k_factor_persistent(FactorArgs a) {
  // one buffer: GEMM chunks, or the tiles of the diagonal factor
  __shared__ __align__(16) float sm[GM_SMEM_FLOATS];
  __shared__ int idle_cta;
  const int64_t lda = a.lda;
  unsigned epoch = 0;
  if (threadIdx.x == 0) {
    unsigned id;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(id));
    a.smid[blockIdx.x] = int32_t(id);
  }
  if (blockIdx.x == 0)
    diag_factor(a.A, lda, a.kb * NB, a.T + size_t(a.kb) * NB * NB, a.status, sm);
  if (!grid_barrier(a, epoch)) return;
  // CTA 0 carries the serial chain (the next diagonal block's update and factor).
  // A CTA that shares its SM would take half of its issue slots, so that CTA, if
  // there is one, sits the tile phases out; every CTA finds it by the same scan.
  if (threadIdx.x == 0) idle_cta = INT_MAX;
  __syncthreads();
  {
    const volatile int32_t* sid = a.smid;
    const int32_t s0 = sid[0];
    for (int b = 1 + int(threadIdx.x); b < int(gridDim.x); b += blockDim.x)
      if (sid[b] == s0) atomicMin(&idle_cta, b);
  }
  __syncthreads();
  const int idle = idle_cta == INT_MAX ? -1 : idle_cta;
  const int nw = int(gridDim.x) - (idle >= 0 ? 1 : 0);                 // working CTAs
  const int rank = int(blockIdx.x) - (idle >= 0 && int(blockIdx.x) > idle ? 1 : 0);
  const bool works = int(blockIdx.x) != idle;
  for (int k = a.kb; k < a.ke; ++k) {
    const int k0 = k * NB;
    const float* Tk = a.T + size_t(k) * NB * NB;
    const int rest = a.lda - k0 - NB;
    const int nr = rest / NB;
    float* panel = a.A + int64_t(k0 + NB) * lda + k0;
    float* brow = a.Bx + int64_t(k0) * lda;
    // phase A: the panel solve L[k0+64:, k] = A[k0+64:, k] T_k^T (in place), and
    // X_k = T_k Bx[k, 0:k0+64] (in place)
    const auto phase_a = [&](int t) {
      Tile64 T;
      if (t < nr) {
        T.a = panel + int64_t(t) * NB * lda; T.lda_ = lda;
        T.b = Tk;                            T.ldb = NB;  T.bt = true;
        T.d = panel + int64_t(t) * NB * lda; T.ldd = lda;
      } else {
        const int u = t - nr;
        T.a = Tk;                            T.lda_ = NB;
        T.b = brow + u * NB;                 T.ldb = lda; T.bt = false;
        T.d = brow + u * NB;                 T.ldd = lda;
      }
      T.alpha = 1.f;
      T.acc = false;
      return T;
    };
    if (works) run_tiles64(rank, nw, nr + k + 1, phase_a, sm);
    if (!grid_barrier(a, epoch)) return;
    if (rest == 0 || k + 1 >= a.lim) break;
    // phase B: A[k0+64:, k0+64:lim] -= P P^T (lower tiles of the columns below the
    // outer limit, all rows) and Bx[k0+64:lim, 0:k0+64] -= P X_k
    const int ncol = a.lim - k - 1;                        // SYRK tile columns
    const int n_syrk = ncol * nr - ncol * (ncol - 1) / 2;  // trapezoid: rows tn .. nr-1
    const int nrb = ncol;                                  // M^-1 tile rows
    const int n_total = n_syrk + nrb * (k + 1);
    float* trail = a.A + int64_t(k0 + NB) * lda + k0 + NB;
    float* bxb = a.Bx + int64_t(k0 + NB) * lda;
    const auto phase_b = [&](int t) {
      Tile64 T;
      int tm, tn;
      if (t < n_syrk) {
        // column-major over the trapezoid: column tn holds rows tn .. nr-1
        int u = t;
        tn = 0;
        while (u >= nr - tn) {
          u -= nr - tn;
          ++tn;
        }
        tm = tn + u;
        T.b = panel + int64_t(tn) * NB * lda; T.ldb = lda; T.bt = true;
        T.d = trail + int64_t(tm) * NB * lda + tn * NB;
      } else {
        const int u = t - n_syrk;
        tm = u / (k + 1);
        tn = u - tm * (k + 1);
        T.b = brow + tn * NB;                 T.ldb = lda; T.bt = false;
        T.d = bxb + int64_t(tm) * NB * lda + tn * NB;
      }
      T.a = panel + int64_t(tm) * NB * lda;
      T.lda_ = lda;
      T.ldd = lda;
      T.alpha = -1.f;
      T.acc = true;
      return T;
    };
    if (blockIdx.x == 0 && k + 1 < a.ke) {
      run_tiles64(0, 1, 1, phase_b, sm);     // the next diagonal block first
      diag_factor(a.A, lda, k0 + NB, a.T + size_t(k + 1) * NB * NB, a.status, sm);
    }
    const int workers = nw > 1 ? nw - 1 : 1;
    const int first = nw > 1 ? rank - 1 : 0;
    // without a lookahead (the last step of the launch) the workers start at tile 0
    const int t_lo = (k + 1 < a.ke) ? 1 : 0;
    if (works && (nw == 1 || blockIdx.x > 0))
      run_tiles64(t_lo + first, workers, n_total, phase_b, sm);
    if (!grid_barrier(a, epoch)) return;
  }
}

// the self-test's barrier slot: the library's own, so the call needs no workspace
__device__ __align__(256) unsigned g_selftest_slot[64];

gptq_status selftest_grid_barrier(cudaStream_t st, int32_t* status) {
  unsigned* p = nullptr;
  GPTQ_CUDA(cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_selftest_slot));
  GPTQ_CUDA(cudaMemsetAsync(p, 0, sizeof(g_selftest_slot), st));
  GPTQ_LAUNCH(k_selftest_grid_barrier, 2, 32, 0, st, p, status);
  return GPTQ_OK;
}

// TF32 hi/lo split (hi: the low 13 mantissa bits cleared) of an M x K block with row
// stride lds into M x K outputs with row stride ldo.
__global__ void k_split_rows(const float* src, int64_t lds, int M, int K, float* hi, float* lo,
                             int ldo) {
  const int64_t total = int64_t(M) * K;
  for (int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; idx < total;
       idx += int64_t(gridDim.x) * blockDim.x) {
    const int m = int(idx / K), k = int(idx % K);
    const float v = src[m * lds + k];
    const float h = __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
    hi[int64_t(m) * ldo + k] = h;
    lo[int64_t(m) * ldo + k] = v - h;
  }
}

// The same split, transposed: out[n][k] = src[k * lds + n] for a K x N block.
__global__ void k_split_cols(const float* src, int64_t lds, int K, int N, float* hi, float* lo,
                             int ldo) {
  __shared__ float tile[32][33];
  const int k0 = blockIdx.y * 32, n0 = blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int k = k0 + i, n = n0 + threadIdx.x;
    tile[i][threadIdx.x] = (k < K && n < N) ? src[k * lds + n] : 0.f;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int n = n0 + i, k = k0 + threadIdx.x;
    if (n < N && k < K) {
      const float v = tile[threadIdx.x][i];
      const float h = __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
      hi[int64_t(n) * ldo + k] = h;
      lo[int64_t(n) * ldo + k] = v - h;
    }
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
  if (C <= GATHER_SMEM_MAX_COLS) {
    dim3 tg((C + 31) / 32, (C + 31) / 32), tb(32, 8);
    GPTQ_LAUNCH(k_sym_full, tg, tb, 0, st, H, C, L.Bx, Cp);
    // the attribute is the largest row any call stages, so concurrent calls agree
    GPTQ_CUDA(allow_smem(k_gather_rows, GATHER_SMEM_MAX_COLS * 4));
    // one CTA per row: its source row fills up to 224 KB of shared memory, so 32
    // warps per CTA keep enough loads and stores in flight
    GPTQ_LAUNCH(k_gather_rows, Cp, 1024, Cp * 4, st, L.Bx, Cp, C, Cp, perm, L.lam, L.A);
    GPTQ_CUDA(cudaMemsetAsync(L.Bx, 0, size_t(Cp) * Cp * sizeof(float), st));
    GPTQ_LAUNCH(k_unit_diag, (Cp + 255) / 256, 256, 0, st, L.Bx, Cp);
  } else {
    GPTQ_LAUNCH(k_gather_rev, grid_for(int64_t(Cp) * Cp), 256, 0, st, H, C, Cp, perm, L.lam, L.A,
                L.Bx);
  }
  // Blocked right-looking Cholesky of A interleaved with the blocked forward
  // substitution that turns Bx = I into M^-1, in persistent cooperative launches:
  // one for everything, or, above OUTER_MIN_COLS, one per outer panel of
  // OUTER_BLOCKS steps followed by the outer panel's update of the rest on the
  // tensor cores.
  unsigned* bar = reinterpret_cast<unsigned*>(reinterpret_cast<char*>(L.lam) + 64);
  int* abort_flag = reinterpret_cast<int*>(reinterpret_cast<char*>(L.lam) + 128);
  int per_sm = 0;
  GPTQ_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_factor_persistent,
                                                          GM_THREADS, 0));
  const int sms = sm_count();
  if (per_sm <= 0 || sms <= 0) return GPTQ_ERR_CUDA;
  // enough CTAs for the largest phase, at most what can be co-resident
  const int nr0 = Cp / NB - 1;
  const int most = std::max(1, std::max(nr0 * (nr0 + 1) / 2 + nr0, nr0 + Cp / NB));
  const int grid = std::min(std::min(std::min(per_sm, 2) * sms, most + 1), MAX_FACTOR_GRID);
  const int per = outer_path(Cp) ? OUTER_BLOCKS : L.nblk;
  for (int ob = 0; ob < L.nblk; ob += per) {
    const int oe = std::min(ob + per, L.nblk);
    GPTQ_CUDA(cudaMemsetAsync(reinterpret_cast<char*>(L.lam) + 64, 0, 128, st));
    FactorArgs fa{L.A, L.Bx, L.T, Cp, L.nblk, bar, abort_flag, status, L.smid, ob, oe, oe};
    void* args[] = {&fa};
    GPTQ_CUDA(cudaLaunchCooperativeKernel(reinterpret_cast<void*>(k_factor_persistent),
                                          dim3(grid), dim3(GM_THREADS), args, 0, st));
    note_launch();
    if (oe >= L.nblk) break;
    // the outer panel L_b = A[oend:, o0:oend] updates the rest:
    //   A[oend:, oend:] -= L_b L_b^T    and    Bx[oend:, :oend] -= L_b M^-1[o0:oend, :oend]
    const int o0 = ob * NB, oend = oe * NB, K = oend - o0, Mb = Cp - oend;
    GPTQ_LAUNCH(k_split_rows, grid_for(int64_t(Mb) * K), 256, 0, st,
                L.A + int64_t(oend) * Cp + o0, int64_t(Cp), Mb, K, L.Lh, L.Ll, OUTER_K);
    GPTQ_TRY(gemm3_tf32(st, L.A + int64_t(oend) * Cp + oend, Cp, Mb, 0, Mb, K, L.Lh, L.Ll,
                        OUTER_K, 0, L.Lh, L.Ll, OUTER_K, Mb, 0, true, status));
    dim3 sg((oend + 31) / 32, (K + 31) / 32), sb(32, 8);
    GPTQ_LAUNCH(k_split_cols, sg, sb, 0, st, L.Bx + int64_t(o0) * Cp, int64_t(Cp), K, oend, L.Mh,
                L.Ml, OUTER_K);
    GPTQ_TRY(gemm3_tf32(st, L.Bx + int64_t(oend) * Cp, Cp, Mb, 0, oend, K, L.Lh, L.Ll, OUTER_K, 0,
                        L.Mh, L.Ml, OUTER_K, oend, 0, false, status));
  }
  GPTQ_LAUNCH(k_write_u, grid_for(int64_t(C) * C), 256, 0, st, L.Bx, Cp, C, U);
  return GPTQ_OK;
}

}  // namespace gptq
