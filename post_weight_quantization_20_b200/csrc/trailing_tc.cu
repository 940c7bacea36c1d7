// Lazy trailing update on the tensor cores, GPTQ量化算法深度解析 §2.4:
//   W[:, e:cend] -= Err * U[i0:i0+K, e:cend]
// Err (rows x K, a column window of a rows x ldE buffer) holds the scaled errors
// of the panel just swept (K = 128) or of a block of eight panels (K = 1024, the
// second level of the lazy update); a call may cover any column range after them.  The product
// is fp32-faithful by a 3xTF32 split: x = hi + lo with hi = x with its low 13
// mantissa bits cleared (exact in tf32) and lo = x - hi, and
//   Err * U ~= Err_hi U_hi + Err_hi U_lo + Err_lo U_hi
// (the dropped lo*lo term is ~2^-22 relative).  The sweep writes Err_hi / Err_lo;
// U is split and transposed once per layer into Ut_hi / Ut_lo (C x C, Ut[n][k] =
// U[k][n]) so that both operands are K-major.
//
// One CTA per 128 x 256 output tile; K in 32-deep stages, two stages
// in flight (96 KB each: Err hi+lo and Ut hi+lo K-major boxes of 32 K-values x
// 128 rows, 128-byte swizzled by TMA).  Warp 0 issues TMA, warp 1 issues tcgen05.mma
// kind::tf32 (M=128, N=256, K=8) into one 256-column TMEM accumulator, then all
// four warps move the accumulator through shared memory and subtract it from the
// fp32 working copy in coalesced row segments.
#include <algorithm>

#include "kernels.h"
#include "tc_common.cuh"

namespace gptq {
namespace {

constexpr int TM = 128, TN = 256, TK = 32;   // K = 32 per stage, K / 32 stages
constexpr int A_BOX = TM * TK * 4;                         // 16 KB: 128 rows x 128 B
constexpr int B_BOX = 128 * TK * 4;                        // 16 KB: 128 N-rows x 128 B
constexpr int STAGE = 2 * A_BOX + 2 * (TN / 128) * B_BOX;  // 96 KB
constexpr int BUFS = 2;
constexpr int THREADS = 128;
constexpr int SMEM = BUFS * STAGE + 1024 + 128;
constexpr int EP_LD = TN + 4;                              // staged accumulator row (floats)
static_assert(TM * EP_LD * 4 <= BUFS * STAGE, "the stage buffers hold the accumulator tile");

__global__ void __launch_bounds__(THREADS, 1)
k_trailing_tc(const __grid_constant__ CUtensorMap ehi, const __grid_constant__ CUtensorMap elo,
              const __grid_constant__ CUtensorMap uhi, const __grid_constant__ CUtensorMap ulo,
              float* Wk, int R, int C, int i0, int e, int cend, int kE0, int nk,
              uint32_t idesc, int vec, int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + BUFS * STAGE);
  uint64_t* empty = full + BUFS;
  uint64_t* done = empty + BUFS;
  uint64_t* drain = done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * TM, n0 = e + blockIdx.x * TN;

  if (threadIdx.x == 0) {
    for (int b = 0; b < BUFS; ++b) {
      tc::mbar_init(full + b, 1);
      tc::mbar_init(empty + b, 1);
    }
    tc::mbar_init(done, 1);
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, TN);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  int64_t issued = 0;             // stages filled by the producer thread

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < nk; ++s) {
      const int b = s % BUFS;
      if (s >= BUFS && !tc::mbar_wait(empty + b, ((s / BUFS) - 1) & 1, abort_flag)) break;
      uint8_t* st = smem + b * STAGE;
      tc::mbar_expect_tx(full + b, STAGE);
      const int k0 = s * TK;
      tc::tma_load_2d(st, &ehi, kE0 + k0, m0, full + b);
      tc::tma_load_2d(st + A_BOX, &elo, kE0 + k0, m0, full + b);
      uint8_t* bh = st + 2 * A_BOX;
      uint8_t* bl = bh + (TN / 128) * B_BOX;
      for (int q = 0; q < TN / 128; ++q) {
        tc::tma_load_2d(bh + q * B_BOX, &uhi, i0 + k0, n0 + 128 * q, full + b);
        tc::tma_load_2d(bl + q * B_BOX, &ulo, i0 + k0, n0 + 128 * q, full + b);
      }
      ++issued;
    }
  } else if (warp == 1 && lane == 0) {
    bool ok = true;
    for (int s = 0; s < nk && ok; ++s) {
      const int b = s % BUFS;
      if (!tc::mbar_wait(full + b, (s / BUFS) & 1, abort_flag)) { ok = false; break; }
      tc::fence_after_sync();
      const uint8_t* st = smem + b * STAGE;
      const uint8_t* ah = st;
      const uint8_t* al = st + A_BOX;
      const uint8_t* bh = st + 2 * A_BOX;
      const uint8_t* bl = bh + (TN / 128) * B_BOX;
#pragma unroll
      for (int kk = 0; kk < TK / 8; ++kk) {
        // both operands K-major: 8 K-values = 32 bytes into each 128-byte row,
        // 8-row groups 1024 bytes apart (the two 128-row B boxes are contiguous)
        const uint64_t dah = tc::smem_desc_sw128(ah + kk * 32, 16, 1024);
        const uint64_t dal = tc::smem_desc_sw128(al + kk * 32, 16, 1024);
        const uint64_t dbh = tc::smem_desc_sw128(bh + kk * 32, 16, 1024);
        const uint64_t dbl = tc::smem_desc_sw128(bl + kk * 32, 16, 1024);
        const uint32_t first = (s == 0 && kk == 0) ? 0u : 1u;
        tc::mma_tf32(tmem, dah, dbh, idesc, first);
        tc::mma_tf32(tmem, dah, dbl, idesc, 1u);
        tc::mma_tf32(tmem, dal, dbh, idesc, 1u);
      }
      tc::mma_commit(empty + b);
    }
    if (ok) tc::mma_commit(done);
  }
  // epilogue: the accumulator goes through shared memory (the stage buffers are
  // free once every MMA has completed) so that W is updated with coalesced row
  // segments and many loads in flight.  Warp w owns TMEM lanes (rows) 32w..32w+31.
  __syncwarp();
  const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(done, 0, abort_flag));
  float* stg = reinterpret_cast<float*>(smem);             // [TM][EP_LD]
  if (ok) {
    tc::fence_after_sync();
    float* srow = stg + (warp * 32 + lane) * EP_LD;
    for (int c = 0; c < TN / 16; ++c) {
      uint32_t v[16];
      tc::tmem_ld_32x16(tmem + (uint32_t(warp * 32) << 16) + uint32_t(c * 16), v);
      tc::tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<float4*>(srow + c * 16 + 4 * q) =
            make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                        __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
    }
  }
  __syncthreads();
  if (ok) {
    // warp w: rows 32w .. 32w+31, eight at a time; lane l: column quads l and
    // l + 32 of each row.  A batch's loads are all issued before its stores (the
    // compiler cannot reorder a load of one row past the store of another).
    constexpr int RB = 8;
    const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i0 = 0; i0 < 32; i0 += RB) {
      float4 w[RB][2];
#pragma unroll
      for (int j = 0; j < RB; ++j) {
        const int row = m0 + warp * 32 + i0 + j;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int col = n0 + 4 * (lane + 32 * h);
          w[j][h] = (vec && row < R && col + 4 <= cend)
                        ? *reinterpret_cast<const float4*>(Wk + int64_t(row) * C + col)
                        : zero4;
        }
      }
#pragma unroll
      for (int j = 0; j < RB; ++j) {
        const int rr = warp * 32 + i0 + j, row = m0 + rr;
        if (row >= R) continue;
        float* wrow = Wk + int64_t(row) * C;
        const float* srow = stg + rr * EP_LD;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int cq = lane + 32 * h, col = n0 + 4 * cq;
          const float4 a = *reinterpret_cast<const float4*>(srow + 4 * cq);
          if (vec && col + 4 <= cend) {
            float4 x = w[j][h];
            x.x -= a.x; x.y -= a.y; x.z -= a.z; x.w -= a.w;
            *reinterpret_cast<float4*>(wrow + col) = x;
          } else {
            const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (col + q < cend) wrow[col + q] -= av[q];
          }
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (*abort_flag) {
    // A wait gave up (the flag is final here and the branch uniform): the
    // producer's copies and the issued MMAs land before TMEM is freed.
    if (warp == 0 && lane == 0) tc::drain_tma_ring(full, BUFS, issued);
    if (warp == 1 && lane == 0) {
      tc::mma_commit(drain);
      tc::mbar_drain(drain, 0);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (threadIdx.x == 0) raise_status(status, GPTQ_ERR_TIMEOUT);
  }
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, TN);
  }
}

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

bool encode_2d(CUtensorMap* m, const float* base, uint64_t inner, uint64_t outer, uint64_t ld,
               uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {ld * 4};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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

gptq_status trailing_update_tc(cudaStream_t st, float* Wk, int R, int C, int i0, int K, int e,
                               int cend, const float* Ehi, const float* Elo, int ldE, int kE0,
                               const float* Uthi, const float* Utlo, int32_t* status) {
  if (e >= cend || R <= 0) return GPTQ_OK;
  if (cend > C || K <= 0 || K % TK || kE0 % TK || kE0 + K > ldE || e < i0 + K)
    return GPTQ_ERR_INVALID_ARG;
  CUtensorMap mehi, melo, muhi, mulo;
  if (!encode_2d(&mehi, Ehi, uint64_t(ldE), uint64_t(R), uint64_t(ldE), TK, TM) ||
      !encode_2d(&melo, Elo, uint64_t(ldE), uint64_t(R), uint64_t(ldE), TK, TM) ||
      !encode_2d(&muhi, Uthi, uint64_t(C), uint64_t(C), uint64_t(C), TK, 128) ||
      !encode_2d(&mulo, Utlo, uint64_t(C), uint64_t(C), uint64_t(C), TK, 128))
    return GPTQ_ERR_UNSUPPORTED;
  // idesc: D f32, A/B tf32, both K-major, N = 256, M = 128
  const uint32_t idesc = (1u << 4) | (2u << 7) | (2u << 10) | (uint32_t(TN >> 3) << 17) |
                         (uint32_t(TM >> 4) << 24);
  const int vec = ((C & 3) == 0 && (reinterpret_cast<uintptr_t>(Wk) & 15) == 0) ? 1 : 0;
  GPTQ_CUDA(allow_smem(k_trailing_tc, SMEM));
  dim3 grid((cend - e + TN - 1) / TN, (R + TM - 1) / TM);
  GPTQ_LAUNCH(k_trailing_tc, grid, THREADS, SMEM, st, mehi, melo, muhi, mulo, Wk, R, C, i0, e,
              cend, kE0, K / TK, idesc, vec, status);
  return GPTQ_OK;
}

}  // namespace gptq
