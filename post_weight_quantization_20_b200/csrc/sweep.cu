// The column sweep, GPTQ量化算法深度解析 §2.2 (OBS compensation), §2.4 (fixed order,
// lazy batch updates), §3.1 step 3-4.
//
// Data layout in HBM (workspace):
//   Wk    rows x C fp32   working copy of W in sweep order (columns gathered by perm)
//   Err   rows x 2048 fp32 (hi and lo parts) scaled errors (w - Q)/U[q][q]; panel p
//         writes columns 128 (p % 16) .. +128, so the errors of two consecutive
//         blocks of eight panels are held at once
//   cp    rows x C u8     codes in sweep order
//   lpart tiles x C fp32  per-row-tile partial column losses (summed in finalize)
//
// Rows are independent once U is known, so the in-panel sweep runs one row per
// SW_TPR threads: each thread keeps SW_CPT panel columns in registers, the
// column being quantized is broadcast with a warp shuffle, and every thread of
// the row applies the rank-1 compensation to its own columns using the panel's
// U block held in shared memory.  Group grids are warp-shuffle min/max
// reductions over the row's g columns.  The lazy trailing update
// W[:, end:] -= Err * U[panel, end:] is split three ways (see sweep_lookahead):
// the next panel's columns inside the next sweep (fp32, before it quantizes),
// the columns up to the end of the panel's block of eight on the tensor cores,
// and the columns beyond that once per block (K = 1024).
#include <algorithm>

#include "common.cuh"
#include "gemm_f32.cuh"
#include "kernels.h"

namespace gptq {

constexpr int SW_B = 128;                 // panel width (columns)
constexpr int SW_B2 = 1024;               // second level of the lazy update (8 panels)
constexpr int SW_ESLOTS = 2 * SW_B2 / SW_B;
constexpr int SW_LDERR = SW_ESLOTS * SW_B; // row stride of the error buffers
constexpr int SW_TPR = 8;                 // threads per row
constexpr int SW_CPT = SW_B / SW_TPR;     // panel columns owned by one thread (16)
constexpr int SW_ROWS = 16;               // rows per CTA
constexpr int SW_THREADS = SW_ROWS * SW_TPR;
constexpr int SW_LDU = SW_B + 4 * SW_TPR; // skewed U row: column c at c + 4*(c / SW_CPT)
constexpr int SW_LDE = SW_B + 1;           // staged error row (the previous panel's)
// U block, 1/U_qq, per-row losses of the panel (or the previous panel's errors)
constexpr int SW_SMEM = (SW_B * SW_LDU + SW_B + SW_ROWS * SW_LDE) * 4;

struct QuantLayout {
  float* Wk;
  float* Ehi;    // rows x SW_LDERR
  float* Elo;
  uint8_t* cp;
  float* lpart;
  float* Uhi;
  float* Ulo;
  int tiles;
};

static QuantLayout quant_layout(void* ws, int64_t R, int64_t C) {
  QuantLayout L{};
  L.tiles = int((R + SW_ROWS - 1) / SW_ROWS);
  char* p = static_cast<char*>(ws);
  L.Wk = reinterpret_cast<float*>(p);    p += align256(size_t(R) * C * 4);
  L.Ehi = reinterpret_cast<float*>(p);   p += align256(size_t(R) * SW_LDERR * 4);
  L.Elo = reinterpret_cast<float*>(p);   p += align256(size_t(R) * SW_LDERR * 4);
  L.cp = reinterpret_cast<uint8_t*>(p);  p += align256(size_t(R) * C);
  L.lpart = reinterpret_cast<float*>(p); p += align256(size_t(L.tiles) * C * 4);
  L.Uhi = reinterpret_cast<float*>(p);   p += align256(size_t(C) * C * 4);
  L.Ulo = reinterpret_cast<float*>(p);
  return L;
}

size_t quantize_ws_bytes(int64_t R, int64_t C, const gptq_config&) {
  const int64_t tiles = (R + SW_ROWS - 1) / SW_ROWS;
  return align256(size_t(R) * C * 4) + 2 * align256(size_t(R) * SW_LDERR * 4) +
         align256(size_t(R) * C) + align256(size_t(tiles) * C * 4) +
         2 * align256(size_t(C) * C * 4) + 256;
}

// Grid of a set of values with range [lo, hi] (lo <= 0 <= hi), all in IEEE fp32.
__device__ __forceinline__ void grid_params(float lo, float hi, float maxq, int sym, float& s,
                                            float& z) {
  if (sym) {
    float m = fmaxf(-lo, hi);
    if (m == 0.f) m = 1.f;
    s = __fdiv_rn(__fsub_rn(m, -m), maxq);
    z = (maxq + 1.f) * 0.5f;
  } else {
    if (lo == 0.f && hi == 0.f) { lo = -1.f; hi = 1.f; }
    s = __fdiv_rn(__fsub_rn(hi, lo), maxq);
    z = rintf(__fdiv_rn(-lo, s));
  }
}

// Wk[r][j] = W[r][perm[j]] as fp32.
__global__ void k_load_w(const void* W, int dt, int R, int C, int64_t ldw, const int32_t* perm,
                         float* Wk) {
  const int64_t total = int64_t(R) * C;
  for (int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; idx < total;
       idx += int64_t(gridDim.x) * blockDim.x) {
    const int r = int(idx / C), j = int(idx % C);
    int p = perm[j];
    p = min(max(p, 0), C - 1);
    Wk[idx] = load_f32(W, dt, int64_t(r) * ldw + p);
  }
}

// One grid per row from the uncompensated row (group_size 0): one warp per row.
__global__ void k_row_grid(const float* Wk, int R, int C, int bits, int sym, float* scales,
                           float* zeros) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= R) return;
  const float* row = Wk + int64_t(warp) * C;
  float lo = 0.f, hi = 0.f;
  for (int j = lane; j < C; j += 32) {
    lo = fminf(lo, row[j]);
    hi = fmaxf(hi, row[j]);
  }
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    float s, z;
    grid_params(lo, hi, float((1 << bits) - 1), sym, s, z);
    scales[warp] = s;
    zeros[warp] = z;
  }
}

// In-panel sweep of columns [i0, i0 + nb) for SW_ROWS rows per CTA.  Thread
// (row, t) owns panel columns 16t .. 16t + 15 of its row in registers.
__device__ __forceinline__ int uskew(int b) { return b + 4 * (b / SW_CPT); }

__global__ void __launch_bounds__(SW_THREADS)
k_sweep_panel(float* Wk, int R, int C, int i0, int nb, const float* U, int bits, int g, int sym,
              float* scales, float* zeros, int G, uint8_t* cp, float* Ehi, float* Elo,
              float* lpart, const float* Eph, const float* Epl, int ip) {
  constexpr int ldE = SW_LDERR;   // row stride of the error buffers
  extern __shared__ __align__(16) float sm[];
  float* Us = sm;                       // SW_B x SW_LDU
  float* dinv = Us + SW_B * SW_LDU;     // SW_B
  float* lrow = dinv + SW_B;            // SW_ROWS x SW_LDE
  const int tid = threadIdx.x, lane = tid & 31;
  const int t = tid % SW_TPR, rl = tid / SW_TPR;
  const int r = blockIdx.x * SW_ROWS + rl;
  const bool rv = r < R;
  const bool vec = ((C & 3) == 0) && (nb == SW_B) && ((reinterpret_cast<uintptr_t>(U) & 15) == 0);
  // U[a0 .. a0+128, i0 .. i0+nb) into the skewed layout, 16-byte loads
  const auto load_ublock = [&](int a0, int na) {
    if (vec) {
      // batches of 16 loads issued before their stores (a generic-pointer load
      // may not move past a shared store the compiler cannot tell apart from it)
      constexpr int NX = (SW_B * SW_B / 4) / SW_THREADS, BX = 16;
#pragma unroll 1
      for (int x0 = 0; x0 < NX; x0 += BX) {
        float4 v[BX];
#pragma unroll
        for (int x = 0; x < BX; ++x) {
          const int e4 = tid + SW_THREADS * (x0 + x);
          const int a = e4 / (SW_B / 4), b = 4 * (e4 % (SW_B / 4));
          v[x] = *reinterpret_cast<const float4*>(U + int64_t(a0 + a) * C + i0 + b);
        }
#pragma unroll
        for (int x = 0; x < BX; ++x) {
          const int e4 = tid + SW_THREADS * (x0 + x);
          const int a = e4 / (SW_B / 4), b = 4 * (e4 % (SW_B / 4));
          *reinterpret_cast<float4*>(Us + a * SW_LDU + uskew(b)) = v[x];
        }
      }
    } else {
      for (int e = tid; e < SW_B * SW_B; e += SW_THREADS) {
        const int a = e / SW_B, b = e % SW_B;
        Us[a * SW_LDU + uskew(b)] = (a < na && b < nb) ? U[int64_t(a0 + a) * C + i0 + b] : 0.f;
      }
    }
  };
  float w[SW_CPT];
  const float* wrow = Wk + int64_t(rv ? r : 0) * C + i0 + t * SW_CPT;
  if (rv && vec) {
#pragma unroll
    for (int q = 0; q < SW_CPT / 4; ++q) {
      const float4 v = *reinterpret_cast<const float4*>(wrow + 4 * q);
      w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int jj = 0; jj < SW_CPT; ++jj) w[jj] = (rv && t * SW_CPT + jj < nb) ? wrow[jj] : 0.f;
  }
  if (ip >= 0) {
    // the previous panel's lazy update restricted to this panel's columns, in fp32:
    // W[:, i0:i0+nb] -= Err_prev * U[ip:ip+128, i0:i0+nb]
    {
      // the CTA's rows of the previous errors: all loads in flight at once
      constexpr int NQ = SW_ROWS * SW_B / 4 / SW_THREADS;
      float4 hq[NQ], lq[NQ];
#pragma unroll
      for (int x = 0; x < NQ; ++x) {
        const int e4 = tid + SW_THREADS * x, rr = e4 / (SW_B / 4), k = 4 * (e4 % (SW_B / 4));
        const int row = blockIdx.x * SW_ROWS + rr;
        const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
        hq[x] = row < R ? *reinterpret_cast<const float4*>(Eph + int64_t(row) * ldE + k) : zero4;
        lq[x] = row < R ? *reinterpret_cast<const float4*>(Epl + int64_t(row) * ldE + k) : zero4;
      }
      load_ublock(ip, SW_B);
#pragma unroll
      for (int x = 0; x < NQ; ++x) {
        const int e4 = tid + SW_THREADS * x, rr = e4 / (SW_B / 4), k = 4 * (e4 % (SW_B / 4));
        float* d = lrow + rr * SW_LDE + k;
        d[0] = hq[x].x + lq[x].x;
        d[1] = hq[x].y + lq[x].y;
        d[2] = hq[x].z + lq[x].z;
        d[3] = hq[x].w + lq[x].w;
      }
    }
    __syncthreads();
    const float* erow = lrow + rl * SW_LDE;
#pragma unroll 4
    for (int k = 0; k < SW_B; ++k) {
      const float ek = erow[k];
      const float* urow = Us + k * SW_LDU + t * (SW_CPT + 4);
#pragma unroll
      for (int jj = 0; jj < SW_CPT; jj += 4) {
        const float4 u = *reinterpret_cast<const float4*>(urow + jj);
        w[jj + 0] = fmaf(-ek, u.x, w[jj + 0]);
        w[jj + 1] = fmaf(-ek, u.y, w[jj + 1]);
        w[jj + 2] = fmaf(-ek, u.z, w[jj + 2]);
        w[jj + 3] = fmaf(-ek, u.w, w[jj + 3]);
      }
    }
    __syncthreads();   // Us and lrow are reused below
  }
  // the panel's own U block (rows and columns i0 .. i0 + nb)
  load_ublock(i0, nb);
  if (tid < SW_B) dinv[tid] = tid < nb ? 1.f / U[int64_t(i0 + tid) * C + i0 + tid] : 0.f;
  __syncthreads();

  const float maxq = float((1 << bits) - 1);
  float s = 1.f, z = 0.f;
  if (g <= 0 && rv) { s = scales[r]; z = zeros[r]; }
  float inv_s = __frcp_rn(s), cmin = -z, cmax = maxq - z;
  const int gmask = g - 1;   // g divides 128, so it is a power of two
  float e[SW_CPT];
  uint32_t cw[SW_CPT / 4];
#pragma unroll
  for (int jj = 0; jj < SW_CPT; ++jj) e[jj] = 0.f;
#pragma unroll
  for (int jj = 0; jj < SW_CPT / 4; ++jj) cw[jj] = 0u;

  for (int c = 0; c < SW_TPR; ++c) {
#pragma unroll
    for (int qq = 0; qq < SW_CPT; ++qq) {
      const int q = c * SW_CPT + qq;
      if (q >= nb) break;
      if (g > 0 && (q & gmask) == 0) {
        float lo = 0.f, hi = 0.f;
#pragma unroll
        for (int jj = 0; jj < SW_CPT; ++jj) {
          const int col = t * SW_CPT + jj;
          if (col >= q && col < q + g && col < nb) {
            lo = fminf(lo, w[jj]);
            hi = fmaxf(hi, w[jj]);
          }
        }
#pragma unroll
        for (int o = 1; o < SW_TPR; o <<= 1) {
          lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
          hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        grid_params(lo, hi, maxq, sym, s, z);
        inv_s = __frcp_rn(s);
        cmin = -z;
        cmax = maxq - z;
        if (t == 0 && rv) {
          const int gi = (i0 + q) / g;
          scales[int64_t(r) * G + gi] = s;
          zeros[int64_t(r) * G + gi] = z;
        }
      }
      // code - z = clamp(rint(x / s), -z, maxq - z), with x / s taken as x * (1/s)
      // (within 2 ulp of the division); err = (x - s (code - z)) / U_qq, where the
      // fma rounds x - s (code - z) once
      const float dq = dinv[q];
      const float x = __shfl_sync(0xffffffffu, w[qq], (lane & ~(SW_TPR - 1)) | c);
      const float cq = fminf(fmaxf(rintf(x * inv_s), cmin), cmax);
      const float err = fmaf(-s, cq, x) * dq;
      const bool mine = (t == c);
      e[qq] = mine ? err : e[qq];
      cw[qq >> 2] |= mine ? (uint32_t(cq + z) << (8 * (qq & 3))) : 0u;
      const float* urow = Us + q * SW_LDU + t * (SW_CPT + 4);
#pragma unroll
      for (int jj = 0; jj < SW_CPT; jj += 4) {
        const float4 u = *reinterpret_cast<const float4*>(urow + jj);
        w[jj + 0] = fmaf(-err, u.x, w[jj + 0]);
        w[jj + 1] = fmaf(-err, u.y, w[jj + 1]);
        w[jj + 2] = fmaf(-err, u.z, w[jj + 2]);
        w[jj + 3] = fmaf(-err, u.w, w[jj + 3]);
      }
    }
  }

  // errors for the trailing update (split hi + lo, hi exact in tf32), codes, and
  // per-row losses for the column reduction
  if (rv) {
    float hv[SW_CPT], lv[SW_CPT];
#pragma unroll
    for (int jj = 0; jj < SW_CPT; ++jj) {
      hv[jj] = __uint_as_float(__float_as_uint(e[jj]) & 0xFFFFE000u);
      lv[jj] = e[jj] - hv[jj];
    }
    float4* hrow = reinterpret_cast<float4*>(Ehi + int64_t(r) * ldE + t * SW_CPT);
    float4* lrw = reinterpret_cast<float4*>(Elo + int64_t(r) * ldE + t * SW_CPT);
#pragma unroll
    for (int q = 0; q < SW_CPT / 4; ++q) {
      hrow[q] = make_float4(hv[4 * q], hv[4 * q + 1], hv[4 * q + 2], hv[4 * q + 3]);
      lrw[q] = make_float4(lv[4 * q], lv[4 * q + 1], lv[4 * q + 2], lv[4 * q + 3]);
    }
    uint8_t* crow = cp + int64_t(r) * C + i0 + t * SW_CPT;
    if (vec && ((reinterpret_cast<uintptr_t>(crow) & 15) == 0)) {
      *reinterpret_cast<uint4*>(crow) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    } else {
#pragma unroll
      for (int jj = 0; jj < SW_CPT; ++jj)
        if (t * SW_CPT + jj < nb) crow[jj] = uint8_t((cw[jj >> 2] >> (8 * (jj & 3))) & 0xffu);
    }
  }
#pragma unroll
  for (int jj = 0; jj < SW_CPT; ++jj) lrow[rl * SW_LDE + t * SW_CPT + jj] = rv ? 0.5f * e[jj] * e[jj] : 0.f;
  __syncthreads();
  if (tid < nb) {
    float l = 0.f;
#pragma unroll
    for (int i = 0; i < SW_ROWS; ++i) l += lrow[i * SW_LDE + tid];
    lpart[int64_t(blockIdx.x) * C + i0 + tid] = l;
  }
}

// Original column order: codes[r][perm[j]] = cp[r][j]; losses[perm[j]] = sum over
// row tiles; g_idx[perm[j]] = j / g.
__global__ void k_scatter_codes(const uint8_t* cp, int R, int C, const int32_t* perm,
                                uint8_t* codes) {
  const int64_t total = int64_t(R) * C;
  for (int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; idx < total;
       idx += int64_t(gridDim.x) * blockDim.x) {
    const int r = int(idx / C), j = int(idx % C);
    int p = perm[j];
    p = min(max(p, 0), C - 1);
    codes[int64_t(r) * C + p] = cp[idx];
  }
}

__global__ void k_finalize_cols(const float* lpart, int tiles, int C, const int32_t* perm, int g,
                                float* losses, int32_t* g_idx) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= C) return;
  float l = 0.f;
  for (int t = 0; t < tiles; ++t) l += lpart[int64_t(t) * C + j];
  int p = perm[j];
  p = min(max(p, 0), C - 1);
  losses[p] = l;
  g_idx[p] = g > 0 ? j / g : 0;
}

static int grid_for(int64_t n) { return int(std::min<int64_t>((n + 255) / 256, 148 * 32)); }

// One non-blocking side stream per host thread and device, created on first use.
static cudaStream_t side_stream(gptq_status& err) {
  static thread_local cudaStream_t streams[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) {
    note_error(e == cudaSuccess ? cudaErrorInvalidDevice : e, "side_stream");
    err = GPTQ_ERR_CUDA;
    return nullptr;
  }
  if (!streams[dev]) {
    e = cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking);
    if (e != cudaSuccess) {
      note_error(e, "cudaStreamCreateWithFlags");
      streams[dev] = nullptr;
      err = GPTQ_ERR_CUDA;
      return nullptr;
    }
  }
  err = GPTQ_OK;
  return streams[dev];
}

// The panels, with the lazy trailing update in two levels and a lookahead of one
// panel.  Panel p of block S (eight panels, SW_B2 columns, ending at column S_end):
//   * the sweep of p first applies panel p-1's update to its own columns (in
//     fp32, from the errors p-1 left in its slot), then sweeps;
//   * a side stream applies p's update (K = 128) to the columns from panel p+2
//     up to and including the first panel after block S;
//   * after the last panel of S, the side stream applies the update of all of S
//     (K = 1024) to the columns after that.
// So every panel receives exactly one update from every earlier panel, and the
// far columns are rewritten once per block instead of once per panel.  Order:
// side work for p starts after the sweep of p; the sweep of p waits for the side
// work enqueued after the sweep of p-2, which includes every side update that
// writes p's columns (side work runs in panel order on one stream).  Panel p's
// errors live in slot p % 16 of the error buffers; the slot is rewritten by the
// sweep of p+16, after the side work of p+14, so after every reader (the sweep
// of p+1 and the side updates of p and of its block).  The caller's stream joins
// the side stream before returning (event fork/join).  Every column receives its
// updates in panel order, so results are deterministic.
static gptq_status sweep_lookahead(cudaStream_t st, const QuantLayout& L, int R, int C,
                                   const float* U, const gptq_config& cfg, int g, int G,
                                   float* scales, float* zeros, int32_t* status) {
  gptq_status err = GPTQ_OK;
  cudaStream_t side = side_stream(err);
  if (err != GPTQ_OK) return err;
  cudaEvent_t ev[3] = {};   // swept, updated[2]
  cudaError_t ce = cudaSuccess;
  for (int i = 0; i < 3 && ce == cudaSuccess; ++i)
    ce = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
  if (ce != cudaSuccess) {
    for (cudaEvent_t e : ev)
      if (e) cudaEventDestroy(e);
    note_error(ce, "cudaEventCreateWithFlags");
    return GPTQ_ERR_CUDA;
  }
  cudaEvent_t swept = ev[0];
  // fork: the side stream starts after everything the caller enqueued so far
  ce = cudaEventRecord(swept, st);
  if (ce == cudaSuccess) ce = cudaStreamWaitEvent(side, swept, 0);
  bool upd[2] = {false, false};   // updated[b] holds the side work of an earlier panel
  const int np = (C + SW_B - 1) / SW_B, per = SW_B2 / SW_B;
  for (int p = 0; p < np && ce == cudaSuccess && err == GPTQ_OK; ++p) {
    const int i0 = p * SW_B, nb = min(SW_B, C - i0), b = p & 1;
    if (upd[b]) {   // the side work of p-2
      ce = cudaStreamWaitEvent(st, ev[1 + b], 0);
      if (ce != cudaSuccess) break;
      upd[b] = false;
    }
    const int slot = p % SW_ESLOTS, pslot = (p + SW_ESLOTS - 1) % SW_ESLOTS;
    k_sweep_panel<<<L.tiles, SW_THREADS, SW_SMEM, st>>>(
        L.Wk, R, C, i0, nb, U, cfg.bits, g, cfg.sym, scales, zeros, G, L.cp, L.Ehi + slot * SW_B,
        L.Elo + slot * SW_B, L.lpart, L.Ehi + pslot * SW_B, L.Elo + pslot * SW_B,
        p > 0 ? i0 - SW_B : -1);
    note_launch();
    ce = cudaGetLastError();
    if (ce != cudaSuccess) break;
    const int S0 = (p / per) * SW_B2, S_end = min(S0 + SW_B2, C);
    const bool last = (p % per == per - 1) || p == np - 1;
    const int e1 = i0 + nb + SW_B, c1 = min(S_end + SW_B, C);   // panel level
    const int e2 = S_end + SW_B;                                 // block level
    const bool lvl1 = e1 < c1, lvl2 = last && e2 < C;
    if (!lvl1 && !lvl2) continue;
    ce = cudaEventRecord(swept, st);
    if (ce == cudaSuccess) ce = cudaStreamWaitEvent(side, swept, 0);
    if (ce != cudaSuccess) break;
    // W[:, e:cend] -= Err[:, slot window] * U[panel rows, e:cend], with U read as its
    // transposed split Ut[n][k] = U[k][n]
    if (lvl1)
      err = gemm3_tf32(side, L.Wk, C, R, e1, c1, SW_B, L.Ehi, L.Elo, SW_LDERR, slot * SW_B,
                       L.Uhi, L.Ulo, C, C, i0, false, status);
    if (err == GPTQ_OK && lvl2)
      err = gemm3_tf32(side, L.Wk, C, R, e2, C, S_end - S0, L.Ehi, L.Elo, SW_LDERR,
                       ((p / per) % 2) * SW_B2, L.Uhi, L.Ulo, C, C, S0, false, status);
    if (err != GPTQ_OK) break;
    ce = cudaEventRecord(ev[1 + b], side);
    upd[b] = ce == cudaSuccess;
  }
  // join (also after an error, so that nothing is left running on the side stream
  // unordered with the caller's stream)
  if (cudaEventRecord(swept, side) == cudaSuccess) cudaStreamWaitEvent(st, swept, 0);
  for (cudaEvent_t e : ev) cudaEventDestroy(e);
  if (ce != cudaSuccess) {
    note_error(ce, "sweep_lookahead");
    return GPTQ_ERR_CUDA;
  }
  return err;
}

gptq_status quantize_run(cudaStream_t st, const void* W, int wdt, int R, int C, int64_t ldw,
                         const float* U, const int32_t* perm, const gptq_config& cfg,
                         uint8_t* codes, float* scales, float* zeros, int32_t* g_idx,
                         float* losses, void* ws, int32_t* status) {
  QuantLayout L = quant_layout(ws, R, C);
  const int g = cfg.group_size > 0 ? cfg.group_size : 0;
  const int G = g ? (C + g - 1) / g : 1;
  if (R == 0) {
    GPTQ_LAUNCH(k_finalize_cols, (C + 255) / 256, 256, 0, st, L.lpart, 0, C, perm, g, losses, g_idx);
    return GPTQ_OK;
  }
  GPTQ_CUDA(allow_smem(k_sweep_panel, SW_SMEM));
  GPTQ_LAUNCH(k_load_w, grid_for(int64_t(R) * C), 256, 0, st, W, wdt, R, C, ldw, perm, L.Wk);
  if (!g) {
    GPTQ_LAUNCH(k_row_grid, (R + 7) / 8, 256, 0, st, L.Wk, R, C, cfg.bits, cfg.sym, scales, zeros);
  }
  const bool tc = C > SW_B && trailing_tc_supported(C);
  if (tc) {
    GPTQ_TRY(split_tf32_t(st, U, C, L.Uhi, L.Ulo));
    GPTQ_TRY(sweep_lookahead(st, L, R, C, U, cfg, g, G, scales, zeros, status));
  } else {
    for (int i0 = 0; i0 < C; i0 += SW_B) {
      const int nb = min(SW_B, C - i0);
      GPTQ_LAUNCH(k_sweep_panel, L.tiles, SW_THREADS, SW_SMEM, st, L.Wk, R, C, i0, nb, U, cfg.bits,
                  g, cfg.sym, scales, zeros, G, L.cp, L.Ehi, L.Elo, L.lpart, nullptr, nullptr, -1);
      const int e = i0 + nb;
      if (e < C) {
        // W[:, e:] -= Err[:, 0:nb] * U[i0:e, e:]
        GPTQ_TRY(gemm_f32(st, R, C - e, nb, -1.f, L.Ehi, SW_LDERR, 1, U + int64_t(i0) * C + e, C,
                          1, 1.f, L.Wk + e, C, 0));
        GPTQ_TRY(gemm_f32(st, R, C - e, nb, -1.f, L.Elo, SW_LDERR, 1, U + int64_t(i0) * C + e, C,
                          1, 1.f, L.Wk + e, C, 0));
      }
    }
  }
  GPTQ_LAUNCH(k_scatter_codes, grid_for(int64_t(R) * C), 256, 0, st, L.cp, R, C, perm, codes);
  GPTQ_LAUNCH(k_finalize_cols, (C + 255) / 256, 256, 0, st, L.lpart, L.tiles, C, perm, g, losses,
              g_idx);
  return GPTQ_OK;
}

}  // namespace gptq
