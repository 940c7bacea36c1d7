// Hessian contraction on the 5th-generation tensor cores:
//   H[i][j] += beta * sum_t X[t][i] X[t][j]      (upper-triangle tiles, fp16/bf16 in, fp32 acc)
// for GPTQ量化算法深度解析 §3.1 step 1.
//
// Two forms: on CTA pairs (the second kernel below, 256 x 256 tiles, the default)
// and on one SM per tile (the first, for a device on which clusters of two cannot
// be resident).  The one-SM form:
//
// Output tile 128 (i) x 256 (j); both operands are read straight from row-major
// X by TMA as 64-token x 64-column boxes with 128-byte swizzle, which is the
// MN-major layout tcgen05 consumes (no transpose pass over X).  Per CTA:
//   warp 0      TMA producer (4-stage ring, 48 KB per stage)
//   warp 1      TMEM allocator and MMA issuer (tcgen05.mma kind::f16, M=128 N=256 K=16)
//   warps 2-9   epilogue: two warps per TMEM lane quadrant, 128 columns each
//
// Precision: the tensor core's fp32 accumulation does not round to nearest, so
// a long accumulation chain inside TMEM drifts (about 1e-4 relative over 20k
// tokens; about 2e-6 with 512-token segments, 1e-6 with 256, at 262144 tokens and
// C = 3072).  The MMA therefore accumulates SEG token steps (512 tokens) into one
// of two TMEM buffers, and the epilogue adds each segment into a register
// accumulator with ordinary round-to-nearest fp32 adds while the MMA fills the
// other buffer.  At the end of a work item the registers are added into H with
// vector red.global.add.
//
// Work items are (tile, token split) pairs handed out round-robin to a
// persistent grid of one CTA per SM; items in flight together share token
// ranges, so X is re-read from L2 rather than HBM.  H's upper triangle has been
// scaled by the running-mean factor beforehand, so every item adds its sum.
#include <algorithm>
#include <cmath>
#include <mutex>

#include "kernels.h"
#include "tc_common.cuh"

namespace gptq {

namespace {

constexpr int BM = 128, BN = 256, BK = 64;   // tile and tokens per stage
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;         // 16 KB
constexpr int B_BYTES = BN * BK * 2;         // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int BOX_BYTES = 64 * BK * 2;       // one 64-column x 64-token box, 8 KB
constexpr int THREADS = 320;                 // 2 control warps + 8 epilogue warps
constexpr int SEG = 8;                       // token steps (of 64) per TMEM segment
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t TMEM_COLS = 2 * BN;

constexpr int GJ = 8;            // j-tiles per group of the tile order (below)
constexpr int MAX_GROUPS = 64;   // groups with a precomputed start (C <= 131072)

struct Sched {
  int C, T, S, kt, ntj, vec;
  uint32_t wait_limit;           // polls of an mbarrier wait before it gives up
  int ng;                        // groups of GJ j-tiles
  int gstart[MAX_GROUPS + 1];    // first tile of each group (host-computed)
};

// Upper tiles: tile (it, jt) exists iff it < min(nti, 2 jt + 2), i.e. jt >= it / 2.
// They are ordered in groups of GJ j-tiles (GJ * 256 columns); inside a group by
// i-tile, then j-tile.  The tiles in flight together (one per SM) then cover about
// 18 i-tiles x GJ j-tiles, 4.4k columns of X at 49152 columns instead of 19k for a
// j-band order, so each token's columns come from HBM about four times less often.
// Inside group g (j-tiles jb0 .. jb1-1) i-tile it holds jb1 - max(jb0, it/2) tiles:
// jb1 - jb0 for every it < 2 jb0, then one fewer every two i-tiles.
__device__ __forceinline__ void tile_coords(const Sched& s, int t, int& i0, int& j0) {
  int g = 0;
  if (s.ng <= MAX_GROUPS) {
    while (g + 1 < s.ng && t >= s.gstart[g + 1]) ++g;
    t -= s.gstart[g];
  } else {
    const int nti = (s.C + BM - 1) / BM;
    for (; g < s.ng - 1; ++g) {
      const int jb0 = g * GJ, jb1 = min(jb0 + GJ, s.ntj), imax = min(nti, 2 * jb1);
      int n = 0;
      for (int it = 0; it < imax; ++it) n += jb1 - max(jb0, it / 2);
      if (t < n) break;
      t -= n;
    }
  }
  const int jb0 = g * GJ, jb1 = min(jb0 + GJ, s.ntj), w = jb1 - jb0;
  int it = 0;
  if (t < 2 * jb0 * w) {          // the i-tiles with a full row of w j-tiles
    it = t / w;
    t -= it * w;
  } else {
    it = 2 * jb0;
    t -= 2 * jb0 * w;
    for (;; ++it) {
      const int n = jb1 - max(jb0, it / 2);
      if (t < n) break;
      t -= n;
    }
  }
  i0 = it * BM;
  j0 = (max(jb0, it / 2) + t) * BN;
}

__device__ __forceinline__ void item_range(const Sched& s, int w, int& t, int& k0, int& k1) {
  const int sp = w / s.T;
  t = w % s.T;
  k0 = int((int64_t(s.kt) * sp) / s.S);
  k1 = int((int64_t(s.kt) * (sp + 1)) / s.S);
}

__global__ void __launch_bounds__(THREADS, 1)
k_hess_syrk_tc(const __grid_constant__ CUtensorMap xmap, float* H, Sched s, float beta,
               uint32_t idesc, int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = s.S * s.T;

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
        int t, k0, k1, i0, j0;
        item_range(s, w, t, k0, k1);
        tile_coords(s, t, i0, j0);
        for (int k = k0; k < k1; ++k) {
          if (!tc::mbar_wait(empty + stage, phase ^ 1u, abort_flag, s.wait_limit)) { ok = false; break; }
          uint8_t* a = smem + stage * STAGE_BYTES;
          uint8_t* b = a + A_BYTES;
          tc::mbar_expect_tx(full + stage, STAGE_BYTES);
          const int y = k * BK;
#pragma unroll
          for (int q = 0; q < BM / 64; ++q) tc::tma_load_2d(a + q * BOX_BYTES, &xmap, i0 + 64 * q, y, full + stage);
#pragma unroll
          for (int q = 0; q < BN / 64; ++q) tc::tma_load_2d(b + q * BOX_BYTES, &xmap, j0 + 64 * q, y, full + stage);
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
        int t, k0, k1;
        item_range(s, w, t, k0, k1);
        for (int ks = k0; ks < k1 && ok; ks += SEG) {
          const int ke = min(ks + SEG, k1);
          if (!tc::mbar_wait(acc_empty + acc, acc_phase ^ 1u, abort_flag, s.wait_limit)) { ok = false; break; }
          tc::fence_after_sync();
          const uint32_t d = tmem_base + uint32_t(acc * BN);
          for (int k = ks; k < ke; ++k) {
            if (!tc::mbar_wait(full + stage, phase, abort_flag, s.wait_limit)) { ok = false; break; }
            tc::fence_after_sync();
            const uint8_t* a = smem + stage * STAGE_BYTES;
            const uint8_t* b = a + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              // 16 tokens = 16 rows of 128 B inside each swizzled box
              const uint64_t ad = tc::smem_desc_sw128(a + kk * 2048, BOX_BYTES, 1024);
              const uint64_t bd = tc::smem_desc_sw128(b + kk * 2048, BOX_BYTES, 1024);
              tc::mma_f16(d, ad, bd, idesc, (k > ks || kk > 0) ? 1u : 0u);
            }
            tc::mma_commit(empty + stage);
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          }
          if (!ok) break;
          tc::mma_commit(acc_full + acc);
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
    const bool vec = s.vec != 0;
    bool ok = true;
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      int t, k0, k1, i0, j0;
      item_range(s, w, t, k0, k1);
      tile_coords(s, t, i0, j0);
      float r[128];
#pragma unroll
      for (int q = 0; q < 128; ++q) r[q] = 0.f;
      for (int ks = k0; ks < k1; ks += SEG) {
        if (!tc::mbar_wait(acc_full + acc, acc_phase, abort_flag, s.wait_limit)) { ok = false; break; }
        tc::fence_after_sync();
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t v[16];
          tc::tmem_ld_32x16(tmem_base + (uint32_t(lane_base) << 16) +
                                uint32_t(acc * BN + half * 128 + c * 16), v);
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
      const int gi = i0 + lane_base + lane;
      if (gi < s.C) {
        float* hrow = H + int64_t(gi) * s.C;
        const int jb = j0 + half * 128;
#pragma unroll
        for (int q = 0; q < 128; q += 4) {
          const int gj = jb + q;
          const float x0 = beta * r[q], x1 = beta * r[q + 1];
          const float x2 = beta * r[q + 2], x3 = beta * r[q + 3];
          if (vec && gj >= gi && gj + 3 < s.C) {
            tc::red_add_v4(hrow + gj, x0, x1, x2, x3);
          } else {
            if (gj >= gi && gj < s.C) atomicAdd(hrow + gj, x0);
            if (gj + 1 >= gi && gj + 1 < s.C) atomicAdd(hrow + gj + 1, x1);
            if (gj + 2 >= gi && gj + 2 < s.C) atomicAdd(hrow + gj + 2, x2);
            if (gj + 3 >= gi && gj + 3 < s.C) atomicAdd(hrow + gj + 3, x3);
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

// ---------------------------------------------------------------------------
// The same contraction on CTA pairs: a cluster of two CTAs computes a 256 x 256
// tile with one tcgen05.mma of cta_group::2 (M = 256, N = 256, K = 16) per 16
// tokens.  Rank 0 loads X's columns i0 .. i0+127 (A) and j0 .. j0+127 (B), rank 1
// columns i0+128 .. i0+255 and j0+128 .. j0+255, each into its own shared memory,
// with the completion of both counted on rank 0's barrier; rank 0 issues the MMAs,
// whose accumulator rows i0 .. i0+127 land in rank 0's TMEM and i0+128 .. i0+255
// in rank 1's.  Per SM a stage is 32 KB for the same 512 MMA cycles that cost
// 48 KB on one SM with a 128 x 256 tile, and the six-stage ring holds 3k cycles
// of work.  Segments, epilogue and write-back are those of the kernel above,
// each CTA draining its own half of the accumulator.
namespace pair {

constexpr int BT = 256;                      // pair tile (both sides)
constexpr int HT = 128;                      // each CTA's half
constexpr int STAGES = 6;
constexpr int A_BYTES = HT * BK * 2;         // 16 KB
constexpr int B_BYTES = HT * BK * 2;         // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 512 /*barriers*/;
constexpr int GJ = 8;                        // j-tiles per group of the tile order

struct Sched {
  int C, T, S, kt, nt, vec;
  uint32_t wait_limit;
};

// Upper tiles (it <= jt) of nt x nt, in groups of GJ j-tiles; inside a group by
// i-tile, then j-tile.  Group g (j-tiles jb0 .. jb0+w-1) holds jb0 w + w (w+1) / 2
// tiles: w for each i-tile below jb0, then w, w-1, .., 1.
__device__ __forceinline__ void tile_coords(const Sched& s, int t, int& i0, int& j0) {
  int jb0 = 0, w = min(GJ, s.nt);
  for (;;) {
    const int n = jb0 * w + w * (w + 1) / 2;
    if (t < n || jb0 + w >= s.nt) break;
    t -= n;
    jb0 += GJ;
    w = min(GJ, s.nt - jb0);
  }
  int it, jt;
  if (t < jb0 * w) {
    it = t / w;
    jt = jb0 + (t - it * w);
  } else {
    t -= jb0 * w;
    it = jb0;
    int n = w;
    while (t >= n) { t -= n; ++it; --n; }
    jt = it + t;
  }
  i0 = it * BT;
  j0 = jt * BT;
}

__device__ __forceinline__ void item_range(const Sched& s, int w, int& t, int& k0, int& k1) {
  const int sp = w / s.T;
  t = w % s.T;
  k0 = int((int64_t(s.kt) * sp) / s.S);
  k1 = int((int64_t(s.kt) * (sp + 1)) / s.S);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
k_hess_syrk_pair(const __grid_constant__ CUtensorMap xmap, float* H, Sched s, float beta,
                 uint32_t idesc, int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* issued_slot = tmem_slot + 2;       // the partner's fill count (abort path)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = tc::cluster_rank();
  const int pair_id = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int n_items = s.S * s.T;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      tc::mbar_init(full + i, 1);
      tc::mbar_init(empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(acc_full + i, 1);
      tc::mbar_init(acc_empty + i, 16);        // 8 epilogue warps of each CTA
    }
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    *issued_slot = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tc::tmem_relinquish_pair();
  }
  tc::fence_before_sync();
  tc::cluster_sync();                          // both CTAs' barriers and TMEM ready
  tc::fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t peer_flag = tc::cluster_addr(const_cast<int*>(abort_flag), rank ^ 1u);
  int64_t issued = 0;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int w = pair_id; w < n_items && ok; w += n_pairs) {
        int t, k0, k1, i0, j0;
        item_range(s, w, t, k0, k1);
        tile_coords(s, t, i0, j0);
        const int ia = i0 + HT * int(rank), jb = j0 + HT * int(rank);
        for (int k = k0; k < k1; ++k) {
          if (!tc::mbar_wait_pair(empty + stage, phase ^ 1u, abort_flag, peer_flag, s.wait_limit)) { ok = false; break; }
          uint8_t* a = smem + stage * STAGE_BYTES;
          uint8_t* b = a + A_BYTES;
          if (rank == 0) tc::mbar_expect_tx(full + stage, 2 * STAGE_BYTES);
          const uint32_t cbar = tc::cluster_addr(full + stage, 0);
          const int y = k * BK;
          tc::tma_load_2d_pair(a, &xmap, ia, y, cbar);
          tc::tma_load_2d_pair(a + BOX_BYTES, &xmap, ia + 64, y, cbar);
          tc::tma_load_2d_pair(b, &xmap, jb, y, cbar);
          tc::tma_load_2d_pair(b + BOX_BYTES, &xmap, jb + 64, y, cbar);
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // every fill consumed: the MMA's last arrivals on this CTA's empty barriers
      // have landed before the CTA can exit
      if (ok)
        for (int st = 0; st < STAGES; ++st) {
          const int64_t n = issued / STAGES + (st < issued % STAGES ? 1 : 0);
          if (n > 0 && !tc::mbar_wait_pair(empty + st, uint32_t((n - 1) & 1), abort_flag, peer_flag, s.wait_limit))
            break;
        }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int w = pair_id; w < n_items && ok; w += n_pairs) {
        int t, k0, k1;
        item_range(s, w, t, k0, k1);
        for (int ks = k0; ks < k1 && ok; ks += SEG) {
          const int ke = min(ks + SEG, k1);
          if (!tc::mbar_wait_pair(acc_empty + acc, acc_phase ^ 1u, abort_flag, peer_flag, s.wait_limit, true)) { ok = false; break; }
          tc::fence_after_sync();
          const uint32_t d = tmem_base + uint32_t(acc * BN);
          for (int k = ks; k < ke; ++k) {
            if (!tc::mbar_wait_pair(full + stage, phase, abort_flag, peer_flag, s.wait_limit)) { ok = false; break; }
            tc::fence_after_sync();
            const uint8_t* a = smem + stage * STAGE_BYTES;
            const uint8_t* b = a + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t ad = tc::smem_desc_sw128(a + kk * 2048, BOX_BYTES, 1024);
              const uint64_t bd = tc::smem_desc_sw128(b + kk * 2048, BOX_BYTES, 1024);
              tc::mma_f16_pair(d, ad, bd, idesc, (k > ks || kk > 0) ? 1u : 0u);
            }
            tc::mma_commit_pair(empty + stage, 0x3);
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          }
          if (!ok) break;
          tc::mma_commit_pair(acc_full + acc, 0x3);
          if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
      }
    }
  } else {
    // epilogue warps 2..9: TMEM lanes 32*(warp % 4) .. +31 (rows i0 + 128 rank + lane),
    // columns 128*half .. +127
    const int lane_base = (warp & 3) * 32;
    const int half = (warp - 2) >> 2;
    const uint32_t acc_empty0 = tc::cluster_addr(acc_empty, 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    const bool vec = s.vec != 0;
    bool ok = true;
    for (int w = pair_id; w < n_items && ok; w += n_pairs) {
      int t, k0, k1, i0, j0;
      item_range(s, w, t, k0, k1);
      tile_coords(s, t, i0, j0);
      float r[128];
#pragma unroll
      for (int q = 0; q < 128; ++q) r[q] = 0.f;
      for (int ks = k0; ks < k1; ks += SEG) {
        if (!tc::mbar_wait_pair(acc_full + acc, acc_phase, abort_flag, peer_flag, s.wait_limit)) { ok = false; break; }
        tc::fence_after_sync();
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t v[16];
          tc::tmem_ld_32x16(tmem_base + (uint32_t(lane_base) << 16) +
                                uint32_t(acc * BN + half * 128 + c * 16), v);
          tc::tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 16; ++q) r[c * 16 + q] += __uint_as_float(v[q]);
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive_cluster(acc_empty0 + uint32_t(acc * 8));
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) break;
      const int gi = i0 + HT * int(rank) + lane_base + lane;
      if (gi < s.C) {
        float* hrow = H + int64_t(gi) * s.C;
        const int jc = j0 + half * 128;
#pragma unroll
        for (int q = 0; q < 128; q += 4) {
          const int gj = jc + q;
          const float x0 = beta * r[q], x1 = beta * r[q + 1];
          const float x2 = beta * r[q + 2], x3 = beta * r[q + 3];
          if (vec && gj >= gi && gj + 3 < s.C) {
            tc::red_add_v4(hrow + gj, x0, x1, x2, x3);
          } else {
            if (gj >= gi && gj < s.C) atomicAdd(hrow + gj, x0);
            if (gj + 1 >= gi && gj + 1 < s.C) atomicAdd(hrow + gj + 1, x1);
            if (gj + 2 >= gi && gj + 2 < s.C) atomicAdd(hrow + gj + 2, x2);
            if (gj + 3 >= gi && gj + 3 < s.C) atomicAdd(hrow + gj + 3, x3);
          }
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::cluster_sync();          // both CTAs out of their loops: the abort flags are final
  if (*abort_flag) {
    // A wait gave up in one of the CTAs, which raised both flags.  (1) rank 0's MMAs
    // land; (2) the producers exchange their fill counts and the one behind fills
    // the phases the other filled (a box at the origin), so every phase of rank 0's
    // full barriers that either CTA loaded into completes; (3) rank 0 waits for
    // them, i.e. for both CTAs' copies; (4) neither CTA exits before that.
    if (warp == 1 && lane == 0 && rank == 0) {
      tc::mma_commit_pair(drain, 0x1);
      tc::mbar_drain(drain, 0);
    }
    if (warp == 0 && lane == 0)
      tc::st_cluster_u32(tc::cluster_addr(issued_slot, rank ^ 1u), uint32_t(issued));
    tc::fence_before_sync();
    tc::cluster_sync();
    if (warp == 0 && lane == 0) {
      const int64_t other = int64_t(*issued_slot);
      for (int64_t f = issued; f < other; ++f) {
        const int st = int(f % STAGES);
        uint8_t* a = smem + st * STAGE_BYTES;
        if (rank == 0) tc::mbar_expect_tx(full + st, 2 * STAGE_BYTES);
        const uint32_t cbar = tc::cluster_addr(full + st, 0);
        tc::tma_load_2d_pair(a, &xmap, 0, 0, cbar);
        tc::tma_load_2d_pair(a + BOX_BYTES, &xmap, 0, 0, cbar);
        tc::tma_load_2d_pair(a + A_BYTES, &xmap, 0, 0, cbar);
        tc::tma_load_2d_pair(a + A_BYTES + BOX_BYTES, &xmap, 0, 0, cbar);
      }
      if (rank == 0) tc::drain_tma_ring(full, STAGES, other > issued ? other : issued);
    }
    tc::fence_before_sync();
    tc::cluster_sync();
    if (threadIdx.x == 0 && rank == 0) raise_status(status, GPTQ_ERR_TIMEOUT);
  }
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace pair

}  // namespace

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

static bool tc_supported_device() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  return major == 10 && minor == 0;
}

// Token splits per tile: the fewest that keep the last wave of the persistent
// grid at least 95% full, and that keep every work item at or below 16384
// token steps (a few ms) so no wait in the kernel comes near its limit.
static int choose_splits(int T, int P, int kt) {
  const int smin = std::max(1, (kt + 16383) / 16384);
  int best = smin;
  for (int S = smin; S <= smin + 64; ++S) {
    if (S > kt) break;
    const double items = double(S) * T;
    const double waves = items / P;
    const double eff = waves / std::ceil(waves);
    best = S;
    if (eff >= 0.95) break;
  }
  return best;
}

// CTA pairs that can be resident at once for the pair kernel on the current device
// (0: clusters of two unavailable, use the one-SM kernel).  Queried once per device.
static int pair_slots() {
  static std::mutex mu;
  static int cached[64];
  static bool known[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (!known[dev]) {
    int n = 0;
    if (cudaFuncSetAttribute(pair::k_hess_syrk_pair, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             pair::SMEM_BYTES) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * 74, 1, 1);
      cfg.blockDim = dim3(THREADS, 1, 1);
      cfg.dynamicSmemBytes = pair::SMEM_BYTES;
      if (cudaOccupancyMaxActiveClusters(&n, pair::k_hess_syrk_pair, &cfg) != cudaSuccess) n = 0;
    }
    (void)cudaGetLastError();
    cached[dev] = n;
    known[dev] = true;
  }
  return cached[dev];
}

gptq_status hessian_syrk_tc(cudaStream_t st, float* H, const void* X, int dt, int64_t m, int C,
                            int64_t ldx, float beta, int32_t* status) {
  if (dt != GPTQ_F16 && dt != GPTQ_BF16) return GPTQ_ERR_UNSUPPORTED;
  if ((ldx % 8) != 0 || (reinterpret_cast<uintptr_t>(X) & 15) != 0) return GPTQ_ERR_UNSUPPORTED;
  if (m > (int64_t(1) << 31) - BK || !tc_supported_device()) return GPTQ_ERR_UNSUPPORTED;
  EncodeTiledFn enc = encode_tiled_fn();
  const int P = sm_count();
  if (!enc || P <= 0) return GPTQ_ERR_UNSUPPORTED;

  CUtensorMap map;
  const cuuint64_t dims[2] = {cuuint64_t(C), cuuint64_t(m)};
  const cuuint64_t strides[1] = {cuuint64_t(ldx) * 2};
  const cuuint32_t box[2] = {64, BK};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType ty =
      dt == GPTQ_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (enc(&map, ty, 2, const_cast<void*>(X), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return GPTQ_ERR_UNSUPPORTED;

  const uint32_t fmt = dt == GPTQ_F16 ? 0u : 1u;
  const int n_pairs = pair_slots();
  if (n_pairs > 0) {
    pair::Sched s;
    s.C = C;
    s.nt = (C + pair::BT - 1) / pair::BT;
    s.T = s.nt * (s.nt + 1) / 2;
    s.kt = int((m + BK - 1) / BK);
    s.S = choose_splits(s.T, n_pairs, s.kt);
    s.vec = ((C & 3) == 0 && (reinterpret_cast<uintptr_t>(H) & 15) == 0) ? 1 : 0;
    s.wait_limit = pipeline_wait_limit();
    const int pairs = int(std::min<int64_t>(n_pairs, int64_t(s.S) * s.T));
    // idesc: D f32, A/B f16 or bf16, both MN-major, N = 256, M = 256 (the pair's)
    const uint32_t idesc = (1u << 4) | (fmt << 7) | (fmt << 10) | (1u << 15) | (1u << 16) |
                           (uint32_t(pair::BT >> 3) << 17) | (uint32_t(pair::BT >> 4) << 24);
    GPTQ_LAUNCH(pair::k_hess_syrk_pair, 2 * pairs, THREADS, pair::SMEM_BYTES, st, map, H, s, beta,
                idesc, status);
    return GPTQ_OK;
  }

  Sched s;
  s.C = C;
  s.ntj = (C + BN - 1) / BN;
  const int nti = (C + BM - 1) / BM;
  s.T = 0;
  for (int jt = 0; jt < s.ntj; ++jt) s.T += std::min(nti, 2 * jt + 2);
  s.ng = (s.ntj + GJ - 1) / GJ;
  if (s.ng <= MAX_GROUPS) {
    int start = 0;
    for (int g = 0; g < s.ng; ++g) {
      s.gstart[g] = start;
      const int jb0 = g * GJ, jb1 = std::min(jb0 + GJ, s.ntj), imax = std::min(nti, 2 * jb1);
      for (int it = 0; it < imax; ++it) start += jb1 - std::max(jb0, it / 2);
    }
    s.gstart[s.ng] = start;
    if (start != s.T) return GPTQ_ERR_UNSUPPORTED;   // the two tile counts must agree
  }
  s.kt = int((m + BK - 1) / BK);
  s.S = choose_splits(s.T, P, s.kt);
  s.vec = ((C & 3) == 0 && (reinterpret_cast<uintptr_t>(H) & 15) == 0) ? 1 : 0;
  s.wait_limit = pipeline_wait_limit();
  const int items = s.S * s.T;
  const int grid = std::min(P, items);

  // idesc: D f32, A/B f16 or bf16, both MN-major, N = 256, M = 128
  const uint32_t idesc = (1u << 4) | (fmt << 7) | (fmt << 10) | (1u << 15) | (1u << 16) |
                         (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);
  GPTQ_CUDA(allow_smem(k_hess_syrk_tc, SMEM_BYTES));
  GPTQ_LAUNCH(k_hess_syrk_tc, grid, THREADS, SMEM_BYTES, st, map, H, s, beta, idesc, status);
  return GPTQ_OK;
}

}  // namespace gptq
