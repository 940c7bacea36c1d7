// fp32-faithful products on the 5th-generation tensor cores:
//   D[m][n] -= sum_k A[m][k] B[n][k]        (3xTF32, both operands K-major)
// the shape of the lazy trailing update W[:, e:] -= Err U[blk, e:] of GPTQ量化算法深度解析
// §2.4 (A = the scaled errors, B = U transposed) and of the outer updates of the
// blocked Cholesky factorization and its inverse (§3.1 step 2).
//
// Each operand is given split as x = hi + lo, hi = x with its low 13 mantissa bits
// cleared (exact in tf32), and the product is Ahi Bhi + Ahi Blo + Alo Bhi (the
// dropped lo*lo term is ~2^-22 relative).
//
// Precision.  The tensor core's fp32 accumulation does not round to nearest, so a
// long chain of MMAs into one TMEM accumulator drifts by about an ulp of the
// running sum per MMA (over a K = 512 update that made the factor's error five
// times that of round-to-nearest fp32).  The MMAs therefore accumulate one stage,
// 32 K-values (12 MMAs), into one of two TMEM buffers, and the epilogue adds each
// such segment into registers with round-to-nearest fp32 adds while the MMAs fill
// the other buffer.  At the end of a tile the registers are subtracted from D.
//
// Persistent grid of one CTA per SM over 128 x 256 output tiles in grouped order
// (GROUP_M row tiles per group, so that the tiles in flight together share
// operand rows in L2).  Per CTA:
//   warp 0      TMA producer (2-stage ring; a stage is 32 K-values of A hi/lo and
//               B hi/lo in 128-byte swizzled rows, 96 KB).  Rows of 128 bytes halve
//               the TMA row requests per byte against 64-byte rows (16 K-values
//               per stage, four 48 KB stages), which measured 8-10% slower.
//   warp 1      TMEM allocator and MMA issuer (tcgen05.mma kind::tf32, M=128 N=256 K=8)
//   warps 2-9   epilogue: two warps per TMEM lane quadrant, 128 columns each
// Every mbarrier wait is bounded; a wait that gives up sets GPTQ_ERR_TIMEOUT and
// the CTA drains its own copies and MMAs before it frees TMEM and exits.
#include <algorithm>

#include "kernels.h"
#include "tc_common.cuh"

namespace gptq {

namespace {

constexpr int TM = 128, TN = 256, TK = 32;
constexpr int A_BOX = TM * TK * 4;                 // 16 KB: 128 rows x 128 B
constexpr int B_BOX = 128 * TK * 4;                // 16 KB: 128 N-rows x 128 B
constexpr int STAGE = 2 * A_BOX + 2 * (TN / 128) * B_BOX;   // 96 KB
constexpr int STAGES = 2;
constexpr int THREADS = 320;
constexpr int SMEM = STAGES * STAGE + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t TMEM_COLS = 2 * TN;
constexpr int GROUP_M = 16;

struct Prob {
  float* D;
  int64_t ldd;
  int M;             // rows of D
  int n_lo, n_hi;    // columns of D written: [n_lo, n_hi)
  int a_k0, b_k0;    // K offset of A's and of B's tensor maps
  int nk;            // K / TK
  int ntm, ntn;      // tile grid
  int lower;         // skip tiles with no entry on or below the diagonal (n - n_lo <= m)
  int vec;           // D rows 16-byte aligned
  uint32_t wait_limit;   // polls of an mbarrier wait before it gives up
};

// t-th tile in grouped order: GROUP_M row tiles, all column tiles, then the next group.
__device__ __forceinline__ void tile_of(const Prob& p, int t, int& tm, int& tn) {
  const int per_group = GROUP_M * p.ntn;
  const int g = t / per_group, r = t - g * per_group;
  const int gm = min(GROUP_M, p.ntm - g * GROUP_M);
  tm = g * GROUP_M + r % gm;
  tn = r / gm;
}

__device__ __forceinline__ bool tile_live(const Prob& p, int tm, int tn) {
  return !p.lower || tn * TN <= tm * TM + (TM - 1);
}

// 320 threads: three warps share a register file quarter of 16k registers, which
// caps a thread at 168 registers
__global__ void __launch_bounds__(THREADS, 1)
k_gemm3_tf32(const __grid_constant__ CUtensorMap ahi, const __grid_constant__ CUtensorMap alo,
             const __grid_constant__ CUtensorMap bhi, const __grid_constant__ CUtensorMap blo,
             Prob p, uint32_t idesc, int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = p.ntm * p.ntn;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      tc::mbar_init(full + i, 1);
      tc::mbar_init(empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(acc_full + i, 1);
      tc::mbar_init(acc_empty + i, 8);
    }
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  int64_t issued = 0;             // stages filled by the producer thread

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
        int tm, tn;
        tile_of(p, w, tm, tn);
        if (!tile_live(p, tm, tn)) continue;
        const int m0 = tm * TM, n0 = p.n_lo + tn * TN;
        for (int s = 0; s < p.nk; ++s) {
          if (!tc::mbar_wait(empty + stage, phase ^ 1u, abort_flag, p.wait_limit)) { ok = false; break; }
          uint8_t* st = smem + stage * STAGE;
          tc::mbar_expect_tx(full + stage, STAGE);
          const int k0 = s * TK;
          tc::tma_load_2d(st, &ahi, p.a_k0 + k0, m0, full + stage);
          tc::tma_load_2d(st + A_BOX, &alo, p.a_k0 + k0, m0, full + stage);
          uint8_t* bh = st + 2 * A_BOX;
          uint8_t* bl = bh + (TN / 128) * B_BOX;
#pragma unroll
          for (int q = 0; q < TN / 128; ++q) {
            tc::tma_load_2d(bh + q * B_BOX, &bhi, p.b_k0 + k0, n0 + 128 * q, full + stage);
            tc::tma_load_2d(bl + q * B_BOX, &blo, p.b_k0 + k0, n0 + 128 * q, full + stage);
          }
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
        int tm, tn;
        tile_of(p, w, tm, tn);
        if (!tile_live(p, tm, tn)) continue;
        for (int s = 0; s < p.nk && ok; ++s) {
          // one stage is one TMEM segment
          if (!tc::mbar_wait(acc_empty + acc, acc_phase ^ 1u, abort_flag, p.wait_limit)) { ok = false; break; }
          if (!tc::mbar_wait(full + stage, phase, abort_flag, p.wait_limit)) { ok = false; break; }
          tc::fence_after_sync();
          const uint32_t d = tmem_base + uint32_t(acc * TN);
          // Both operands K-major in 128-byte rows: 8 K-values = 32 bytes, 8-row groups
          // 1024 bytes apart (the two 128-row B boxes are contiguous).  The small cross
          // products go first, into the fresh accumulator, and the hi*hi products
          // after them, so that the accumulator's truncation is charged mostly at the
          // magnitude of the small sums.
          const uint8_t* ah = smem + stage * STAGE;
          const uint8_t* al = ah + A_BOX;
          const uint8_t* bh = ah + 2 * A_BOX;
          const uint8_t* bl = bh + (TN / 128) * B_BOX;
#pragma unroll
          for (int kk = 0; kk < TK / 8; ++kk) {
            const uint64_t dah = tc::smem_desc_sw128(ah + kk * 32, 16, 1024);
            const uint64_t dal = tc::smem_desc_sw128(al + kk * 32, 16, 1024);
            const uint64_t dbh = tc::smem_desc_sw128(bh + kk * 32, 16, 1024);
            const uint64_t dbl = tc::smem_desc_sw128(bl + kk * 32, 16, 1024);
            tc::mma_tf32(d, dah, dbl, idesc, kk == 0 ? 0u : 1u);
            tc::mma_tf32(d, dal, dbh, idesc, 1u);
          }
#pragma unroll
          for (int kk = 0; kk < TK / 8; ++kk) {
            const uint64_t dah = tc::smem_desc_sw128(ah + kk * 32, 16, 1024);
            const uint64_t dbh = tc::smem_desc_sw128(bh + kk * 32, 16, 1024);
            tc::mma_tf32(d, dah, dbh, idesc, 1u);
          }
          tc::mma_commit(empty + stage);
          tc::mma_commit(acc_full + acc);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
      }
    }
  } else {
    // epilogue warps 2..9: TMEM lanes 32*(warp % 4) .. +31, columns 128*half .. +127
    const int lane_base = (warp & 3) * 32;
    const int half = (warp - 2) >> 2;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      int tm, tn;
      tile_of(p, w, tm, tn);
      if (!tile_live(p, tm, tn)) continue;
      float r[128];
#pragma unroll
      for (int q = 0; q < 128; ++q) r[q] = 0.f;
      for (int s = 0; s < p.nk; ++s) {
        if (!tc::mbar_wait(acc_full + acc, acc_phase, abort_flag, p.wait_limit)) { ok = false; break; }
        tc::fence_after_sync();
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t v[16];
          tc::tmem_ld_32x16(tmem_base + (uint32_t(lane_base) << 16) +
                                uint32_t(acc * TN + half * 128 + c * 16), v);
          tc::tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 16; ++q) r[c * 16 + q] += __uint_as_float(v[q]);
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(acc_empty + acc);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) break;
      const int row = tm * TM + lane_base + lane;
      if (row < p.M) {
        const int cb = p.n_lo + tn * TN + half * 128;
        float* drow = p.D + int64_t(row) * p.ldd;
#pragma unroll
        for (int q = 0; q < 128; q += 4) {
          const int col = cb + q;
          if (p.vec && col + 3 < p.n_hi) {
            float4 x = *reinterpret_cast<const float4*>(drow + col);
            x.x -= r[q]; x.y -= r[q + 1]; x.z -= r[q + 2]; x.w -= r[q + 3];
            *reinterpret_cast<float4*>(drow + col) = x;
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              if (col + i < p.n_hi) drow[col + i] -= r[q + i];
          }
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (*abort_flag) {
    // A wait gave up (every role has left its loop, so the flag is final and the
    // branch is uniform): the producer's copies and the issued MMAs land before
    // TMEM is freed and the CTA exits.
    if (warp == 0 && lane == 0) tc::drain_tma_ring(full, STAGES, issued);
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
    tc::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

bool encode_k_major(CUtensorMap* m, const float* base, uint64_t ld, uint64_t rows,
                    uint32_t box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {ld, rows};
  const cuuint64_t strides[1] = {ld * 4};
  const cuuint32_t box[2] = {uint32_t(TK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

gptq_status gemm3_tf32(cudaStream_t st, float* D, int64_t ldd, int M, int n_lo, int n_hi, int K,
                       const float* Ahi, const float* Alo, int lda, int a_k0, const float* Bhi,
                       const float* Blo, int ldb, int b_rows, int b_k0, bool lower,
                       int32_t* status) {
  if (M <= 0 || n_hi <= n_lo || K <= 0) return GPTQ_OK;
  // K windows start on 16-byte boundaries (TMA x coordinate) and are whole stages
  if (K % TK || a_k0 % 4 || b_k0 % 4 || a_k0 + K > lda || b_k0 + K > ldb || n_lo < 0 ||
      n_hi > b_rows || n_hi > ldd || (lower && n_lo != 0))
    return GPTQ_ERR_INVALID_ARG;
  if ((lda % 4) || (ldb % 4)) return GPTQ_ERR_UNSUPPORTED;
  CUtensorMap mah, mal, mbh, mbl;
  if (!encode_k_major(&mah, Ahi, uint64_t(lda), uint64_t(M), TM) ||
      !encode_k_major(&mal, Alo, uint64_t(lda), uint64_t(M), TM) ||
      !encode_k_major(&mbh, Bhi, uint64_t(ldb), uint64_t(b_rows), 128) ||
      !encode_k_major(&mbl, Blo, uint64_t(ldb), uint64_t(b_rows), 128))
    return GPTQ_ERR_UNSUPPORTED;
  Prob p;
  p.D = D;
  p.ldd = ldd;
  p.M = M;
  p.n_lo = n_lo;
  p.n_hi = n_hi;
  p.a_k0 = a_k0;
  p.b_k0 = b_k0;
  p.nk = K / TK;
  p.ntm = (M + TM - 1) / TM;
  p.ntn = (n_hi - n_lo + TN - 1) / TN;
  p.lower = lower ? 1 : 0;
  p.vec = ((ldd & 3) == 0 && (reinterpret_cast<uintptr_t>(D) & 15) == 0) ? 1 : 0;
  p.wait_limit = pipeline_wait_limit();
  int64_t live = int64_t(p.ntm) * p.ntn;
  if (lower) {
    live = 0;
    for (int tm = 0; tm < p.ntm; ++tm)
      live += std::min<int64_t>(p.ntn, (int64_t(tm) * TM + TM - 1) / TN + 1);
  }
  const int P = sm_count();
  if (P <= 0) return GPTQ_ERR_CUDA;
  const int grid = int(std::min<int64_t>(P, live));
  // idesc: D f32, A/B tf32, both K-major, N = 256, M = 128
  const uint32_t idesc = (1u << 4) | (2u << 7) | (2u << 10) | (uint32_t(TN >> 3) << 17) |
                         (uint32_t(TM >> 4) << 24);
  GPTQ_CUDA(allow_smem(k_gemm3_tf32, SMEM));
  GPTQ_LAUNCH(k_gemm3_tf32, grid, THREADS, SMEM, st, mah, mal, mbh, mbl, p, idesc, status);
  return GPTQ_OK;
}

}  // namespace gptq
