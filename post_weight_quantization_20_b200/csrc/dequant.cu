// Products straight from the stored form (gptq-for-llama article, ainews.cool,
// "工程细节": matrix products from packed low-bit codes), for decode-sized token
// counts: Y[m][r] = sum_c X[m][c] s[r][g(c)] (code[r][c] - z[r][g(c)]).
//
// The codes are first repacked into SWEEP order (column j of a row holds original
// column perm[j]): every group of g columns is then one contiguous run, and the
// act-order gather (GPTQ量化算法深度解析 §3.3: desc_act needs a gather at inference)
// moves to the small activation block, which each CTA stages once per chunk.  A
// row is read in 32-column units; unit u is exactly words [u*b, u*b + b) of the
// repacked row for every b, so a lane reads b whole words and a warp 128*b
// contiguous bytes.  Per unit (g >= 32, so a unit lies in one group):
//   acc[m] += s * (sum_i code_i x[m][i] - z * sum_i x[m][i])
// with sum_i x[m][i] formed once per unit when X is staged.  fp32 throughout.
// HBM-bound: the codes (R*C*b/8 bytes) and grids (R*G*8) are read once.
#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace {


constexpr int KC = 2048;          // columns of X staged per chunk
constexpr int UNITS = KC / 32;    // 64 units per chunk
constexpr int XLD = 36;           // floats per staged unit (32 + 4 pad: conflict-free float4)
constexpr int WARPS = 8;
constexpr int RW = 4;             // rows per warp
constexpr int ROWS = WARPS * RW;  // rows per CTA: the staged X block serves 32 rows
constexpr int UPL = UNITS / 32;   // units of a chunk per lane


// code i (0..31) of a unit held in words w[0..B-1]
template <int B>
__device__ __forceinline__ uint32_t field(const uint32_t (&w)[B], int i) {
  const int bit = i * B, k = bit >> 5, o = bit & 31;
  uint32_t v = w[k] >> o;
  if (o + B > 32) v |= w[k + 1] << (32 - o);   // only for B = 3 (compile-time after unrolling)
  return v & ((1u << B) - 1u);
}

template <int B>
__device__ __forceinline__ void load_unit(const uint32_t* p, uint32_t (&w)[B]) {
  if constexpr (B == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (B == 2) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x; w[1] = v.y;
  } else if constexpr (B == 8) {
    const uint4 a = *reinterpret_cast<const uint4*>(p);
    const uint4 b = *reinterpret_cast<const uint4*>(p + 4);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else {
#pragma unroll
    for (int k = 0; k < B; ++k) w[k] = __ldg(p + k);
  }
}

// Y (M x R fp32, row-major) = X (M x C, row stride ldx) * Q^T.  Qp: R rows of
// C*B/32 words in sweep order; scales/zeros R x G (G = C/g, or 1 per row);
// perm (nullable = identity): sweep column j reads X column perm[j].
template <int B, int MT>
__global__ void __launch_bounds__(WARPS * 32)
k_dq_gemv(const void* __restrict__ X, int xdt, int64_t ldx, int M, const uint32_t* __restrict__ Qp,
          const float* __restrict__ scales, const float* __restrict__ zeros, int G, int gshift,
          const int32_t* __restrict__ perm, int R, int C, float* __restrict__ Y) {
  extern __shared__ __align__(16) float xs[];     // [MT][UNITS][XLD]
  float* xsum = xs + MT * UNITS * XLD;            // [MT][UNITS]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = blockIdx.x * ROWS + warp * RW;
  const int64_t words = int64_t(C) / 32 * B;     // words per row
  float acc[RW][MT];
#pragma unroll
  for (int a = 0; a < RW; ++a)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[a][m] = 0.f;

  for (int c0 = 0; c0 < C; c0 += KC) {
    const int nu = min(KC, C - c0) >> 5;
    // all of the lane's code words of this chunk (RW rows x UPL units) are loaded
    // first, so that they are in flight while X is staged
    uint32_t w[RW][UPL][B];
#pragma unroll
    for (int a = 0; a < RW; ++a) {
      const int r = r0 + a;
      const uint32_t* row = Qp + int64_t(r) * words + int64_t(c0 >> 5) * B;
#pragma unroll
      for (int j = 0; j < UPL; ++j) {
        const int u = lane + 32 * j;
        if (r < R && u < nu) {
          load_unit<B>(row + int64_t(u) * B, w[a][j]);
        } else {
#pragma unroll
          for (int k = 0; k < B; ++k) w[a][j][k] = 0u;
        }
      }
    }
    __syncthreads();                               // the previous chunk is consumed
    for (int e = threadIdx.x; e < MT * nu * 32; e += blockDim.x) {
      const int m = e / (nu * 32), j = e - m * nu * 32;
      const int col = c0 + j;
      const int src = perm ? perm[col] : col;
      xs[(m * UNITS + (j >> 5)) * XLD + (j & 31)] = m < M ? load_f32(X, xdt, int64_t(m) * ldx + src) : 0.f;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < MT * nu; e += blockDim.x) {
      const int m = e / nu, u = e - m * nu;
      const float* p = xs + (m * UNITS + u) * XLD;
      float t = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) t += p[i];
      xsum[m * UNITS + u] = t;
    }
    __syncthreads();

#pragma unroll
    for (int a = 0; a < RW; ++a) {
      const int r = r0 + a;
      if (r >= R) break;
#pragma unroll
      for (int j = 0; j < UPL; ++j) {
        const int u = lane + 32 * j;
        if (u >= nu) break;
        const int g = gshift < 0 ? 0 : ((c0 + 32 * u) >> gshift);
        const float s = __ldg(scales + int64_t(r) * G + g);
        const float z = __ldg(zeros + int64_t(r) * G + g);
        float p[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) p[m] = 0.f;
#pragma unroll
        for (int i4 = 0; i4 < 32; i4 += 4) {
          float cf[4];
#pragma unroll
          // code -> float without I2F: 2^23 + c as bits, minus 2^23 (exact for c < 2^23)
          for (int q = 0; q < 4; ++q)
            cf[q] = __int_as_float(0x4B000000u | field<B>(w[a][j], i4 + q)) - 8388608.f;
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const float4 xv = *reinterpret_cast<const float4*>(xs + (m * UNITS + u) * XLD + i4);
            p[m] = fmaf(cf[0], xv.x, p[m]);
            p[m] = fmaf(cf[1], xv.y, p[m]);
            p[m] = fmaf(cf[2], xv.z, p[m]);
            p[m] = fmaf(cf[3], xv.w, p[m]);
          }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[a][m] = fmaf(s, p[m] - z * xsum[m * UNITS + u], acc[a][m]);
      }
    }
  }
#pragma unroll
  for (int a = 0; a < RW; ++a)
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float v = acc[a][m];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0 && r0 + a < R && m < M) Y[int64_t(m) * R + r0 + a] = v;
    }
}

// Repack original-order packed rows into sweep order: unit u of row r gathers
// original columns perm[32u .. 32u+31].  One thread per (row, unit).
template <int B>
__global__ void k_repack_sweep(const uint32_t* __restrict__ P, const int32_t* __restrict__ perm,
                               int R, int C, uint32_t* __restrict__ Qp) {
  const int64_t nunit = int64_t(C) / 32;
  const int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= int64_t(R) * nunit) return;
  const int r = int(t / nunit), u = int(t - int64_t(r) * nunit);
  const int64_t nw = (int64_t(C) * B + 31) / 32;
  const uint32_t* src = P + int64_t(r) * nw;
  uint32_t w[B];
#pragma unroll
  for (int k = 0; k < B; ++k) w[k] = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int c = perm ? perm[32 * u + i] : 32 * u + i;
    const int64_t bit = int64_t(c) * B;
    const int64_t k = bit >> 5;
    const int o = int(bit & 31);
    uint32_t v = src[k] >> o;
    if (o + B > 32) v |= src[k + 1] << (32 - o);
    v &= (1u << B) - 1u;
    const int ob = i * B, ok = ob >> 5, oo = ob & 31;
    w[ok] |= v << oo;
    if (oo + B > 32) w[ok + 1] |= v >> (32 - oo);
  }
  uint32_t* dst = Qp + int64_t(r) * nunit * B + int64_t(u) * B;
#pragma unroll
  for (int k = 0; k < B; ++k) dst[k] = w[k];
}


// The same product for 4-bit codes and fp16 X with half2 arithmetic inside each
// 8-code word: nibbles i and i + 4 of a word become one half2 (1024 + c, exact)
// with a single mask-and-or, 1024 is subtracted exactly, and four HFMA2 with the
// matching x pairs accumulate the word in half precision; words are widened to
// fp32 and the group's grid applied per 32-column unit in fp32, as above.  X is
// staged as half2 pairs in the nibble order (x0,x4),(x1,x5),(x2,x6),(x3,x7).
// About 2.5 instructions per code instead of ~4.7; each word's sum carries fp16
// rounding (relative 2^-11 per step).
template <int MT>
__global__ void __launch_bounds__(WARPS * 32)
k_dq_gemv_h2(const __half* __restrict__ X, int64_t ldx, int M, const uint32_t* __restrict__ Qp,
             const float* __restrict__ scales, const float* __restrict__ zeros, int G, int gshift,
             const int32_t* __restrict__ perm, int R, int C, float* __restrict__ Y) {
  extern __shared__ __align__(16) float xsm[];
  __half2* xh = reinterpret_cast<__half2*>(xsm);          // [MT][UNITS][16] pairs
  float* xsum = xsm + MT * UNITS * 16;                      // [MT][UNITS]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = blockIdx.x * ROWS + warp * RW;
  const int64_t words = int64_t(C) / 8;                     // 4-bit codes
  float acc[RW][MT];
#pragma unroll
  for (int a = 0; a < RW; ++a)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[a][m] = 0.f;
  const __half2 k1024 = __floats2half2_rn(1024.f, 1024.f);

  for (int c0 = 0; c0 < C; c0 += KC) {
    const int nu = min(KC, C - c0) >> 5;
    __syncthreads();
    // pair slot e of unit u: word wi = e / 4 within the unit, pair k = e % 4:
    // columns 8 wi + k and 8 wi + k + 4
    for (int e = threadIdx.x; e < MT * nu * 16; e += blockDim.x) {
      const int m = e / (nu * 16), rest = e - m * nu * 16, u = rest >> 4, slot = rest & 15;
      const int j = 32 * u + 8 * (slot >> 2) + (slot & 3);
      const int ca = c0 + j, cb = ca + 4;
      const int sa = perm ? perm[ca] : ca, sb = perm ? perm[cb] : cb;
      __half2 v = __floats2half2_rn(0.f, 0.f);
      if (m < M) v = __halves2half2(X[int64_t(m) * ldx + sa], X[int64_t(m) * ldx + sb]);
      xh[(m * UNITS + u) * 16 + slot] = v;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < MT * nu; e += blockDim.x) {
      const int m = e / nu, u = e - m * nu;
      float t = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 f = __half22float2(xh[(m * UNITS + u) * 16 + i]);
        t += f.x + f.y;
      }
      xsum[m * UNITS + u] = t;
    }
    __syncthreads();

#pragma unroll
    for (int a = 0; a < RW; ++a) {
      const int r = r0 + a;
      if (r >= R) break;
      const uint32_t* row = Qp + int64_t(r) * words + int64_t(c0 >> 5) * 4;
      for (int u = lane; u < nu; u += 32) {
        const uint4 wv = *reinterpret_cast<const uint4*>(row + int64_t(u) * 4);
        const uint32_t w4[4] = {wv.x, wv.y, wv.z, wv.w};
        const int g = gshift < 0 ? 0 : ((c0 + 32 * u) >> gshift);
        const float s = __ldg(scales + int64_t(r) * G + g);
        const float z = __ldg(zeros + int64_t(r) * G + g);
        float p[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) p[m] = 0.f;
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
          __half2 cpair[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t bits = ((w4[wi] >> (4 * k)) & 0x000F000Fu) | 0x64006400u;
            cpair[k] = __hsub2(*reinterpret_cast<const __half2*>(&bits), k1024);
          }
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const uint4 xv = *reinterpret_cast<const uint4*>(xh + (m * UNITS + u) * 16 + 4 * wi);
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
            __half2 h = __floats2half2_rn(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              h = __hfma2(cpair[k], *reinterpret_cast<const __half2*>(&xw[k]), h);
            const float2 f = __half22float2(h);
            p[m] += f.x + f.y;
          }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[a][m] = fmaf(s, p[m] - z * xsum[m * UNITS + u], acc[a][m]);
      }
    }
  }
#pragma unroll
  for (int a = 0; a < RW; ++a)
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float v = acc[a][m];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0 && r0 + a < R && m < M) Y[int64_t(m) * R + r0 + a] = v;
    }
}

}  // namespace

static int grid_1d(int64_t n, int threads) { return int((n + threads - 1) / threads); }

template <int B>
static gptq_status repack_b(cudaStream_t st, const uint32_t* P, const int32_t* perm, int R, int C,
                            uint32_t* Qp) {
  const int64_t n = int64_t(R) * (C / 32);
  if (n == 0) return GPTQ_OK;
  GPTQ_LAUNCH(k_repack_sweep<B>, grid_1d(n, 256), 256, 0, st, P, perm, R, C, Qp);
  return GPTQ_OK;
}

gptq_status repack_sweep_run(cudaStream_t st, const uint32_t* packed, int R, int C, int bits,
                             const int32_t* perm, uint32_t* out) {
  switch (bits) {
    case 2: return repack_b<2>(st, packed, perm, R, C, out);
    case 3: return repack_b<3>(st, packed, perm, R, C, out);
    case 4: return repack_b<4>(st, packed, perm, R, C, out);
    case 8: return repack_b<8>(st, packed, perm, R, C, out);
    default: return GPTQ_ERR_INVALID_ARG;
  }
}

template <int B, int MT>
static gptq_status gemv_bm(cudaStream_t st, const void* X, int xdt, int64_t ldx, int M,
                           const uint32_t* Qp, const float* scales, const float* zeros, int G,
                           int gshift, const int32_t* perm, int R, int C, float* Y) {
  const int smem = (MT * UNITS * XLD + MT * UNITS) * 4;
  GPTQ_CUDA(allow_smem(k_dq_gemv<B, MT>, smem));
  GPTQ_LAUNCH((k_dq_gemv<B, MT>), (R + ROWS - 1) / ROWS, WARPS * 32, smem, st, X, xdt, ldx, M, Qp,
              scales, zeros, G, gshift, perm, R, C, Y);
  return GPTQ_OK;
}

template <int B>
static gptq_status gemv_b(cudaStream_t st, const void* X, int xdt, int64_t ldx, int M,
                          const uint32_t* Qp, const float* scales, const float* zeros, int G,
                          int gshift, const int32_t* perm, int R, int C, float* Y) {
  if (M > 8) {
    // blocks of 8 tokens, one launch each (the weights are read once per block)
    const size_t esz = xdt == GPTQ_F32 ? 4 : 2;
    for (int m0 = 0; m0 < M; m0 += 8) {
      const void* Xb = static_cast<const char*>(X) + size_t(m0) * size_t(ldx) * esz;
      GPTQ_TRY(gemv_b<B>(st, Xb, xdt, ldx, min(8, M - m0), Qp, scales, zeros, G, gshift, perm,
                         R, C, Y + int64_t(m0) * R));
    }
    return GPTQ_OK;
  }
  if (M <= 1) return gemv_bm<B, 1>(st, X, xdt, ldx, M, Qp, scales, zeros, G, gshift, perm, R, C, Y);
  if (M <= 2) return gemv_bm<B, 2>(st, X, xdt, ldx, M, Qp, scales, zeros, G, gshift, perm, R, C, Y);
  if (M <= 4) return gemv_bm<B, 4>(st, X, xdt, ldx, M, Qp, scales, zeros, G, gshift, perm, R, C, Y);
  return gemv_bm<B, 8>(st, X, xdt, ldx, M, Qp, scales, zeros, G, gshift, perm, R, C, Y);
}

template <int MT>
static gptq_status gemv_h2_m(cudaStream_t st, const __half* X, int64_t ldx, int M, const uint32_t* Qp,
                             const float* scales, const float* zeros, int G, int gshift,
                             const int32_t* perm, int R, int C, float* Y) {
  const int smem = MT * UNITS * 16 * 4 + MT * UNITS * 4;
  GPTQ_CUDA(allow_smem(k_dq_gemv_h2<MT>, smem));
  GPTQ_LAUNCH(k_dq_gemv_h2<MT>, (R + ROWS - 1) / ROWS, WARPS * 32, smem, st, X, ldx, M, Qp, scales,
              zeros, G, gshift, perm, R, C, Y);
  return GPTQ_OK;
}

gptq_status dequant_matmul_run(cudaStream_t st, const void* X, int xdt, int M, int C, int64_t ldx,
                               const uint32_t* Qp, const float* scales, const float* zeros,
                               int bits, int g, const int32_t* perm, float* Y, int R,
                               int half_sums) {
  if (R == 0) return GPTQ_OK;
  const int G = g > 0 ? (C + g - 1) / g : 1;
  const int gshift = g > 0 ? (g == 32 ? 5 : g == 64 ? 6 : 7) : -1;
  if (half_sums && bits == 4 && xdt == GPTQ_F16 && M <= 2) {
    const __half* Xh = static_cast<const __half*>(X);
    if (M <= 1) return gemv_h2_m<1>(st, Xh, ldx, M, Qp, scales, zeros, G, gshift, perm, R, C, Y);
    return gemv_h2_m<2>(st, Xh, ldx, M, Qp, scales, zeros, G, gshift, perm, R, C, Y);
  }
  switch (bits) {
    case 2: return gemv_b<2>(st, X, xdt, ldx, M, Qp, scales, zeros, G, gshift, perm, R, C, Y);
    case 3: return gemv_b<3>(st, X, xdt, ldx, M, Qp, scales, zeros, G, gshift, perm, R, C, Y);
    case 4: return gemv_b<4>(st, X, xdt, ldx, M, Qp, scales, zeros, G, gshift, perm, R, C, Y);
    case 8: return gemv_b<8>(st, X, xdt, ldx, M, Qp, scales, zeros, G, gshift, perm, R, C, Y);
    default: return GPTQ_ERR_INVALID_ARG;
  }
}

}  // namespace gptq
