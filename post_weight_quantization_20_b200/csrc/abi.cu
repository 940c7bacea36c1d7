// The C ABI of libgptq (include/gptq.h): argument validation and dispatch.
// Every host-checkable error is reported before anything is launched.
#include <atomic>
#include <climits>
#include <cmath>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

#include <cstdio>

namespace gptq {
static std::atomic<uint64_t> g_launches{0};
static std::atomic<uint32_t> g_wait_limit{0};   // 0: tc::WAIT_LIMIT
uint32_t pipeline_wait_limit() {
  const uint32_t v = g_wait_limit.load(std::memory_order_relaxed);
  return v ? v : tc::WAIT_LIMIT;
}
static thread_local char g_last_error[256] = "";
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
void note_error(cudaError_t e, const char* where) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", where, cudaGetErrorName(e),
                cudaGetErrorString(e));
}
}  // namespace gptq

using namespace gptq;


static bool valid_dtype(int dt) { return dt == GPTQ_F32 || dt == GPTQ_F16 || dt == GPTQ_BF16; }

namespace gptq {
gptq_status check_cfg(const gptq_config* cfg) {
  if (!cfg) return GPTQ_ERR_INVALID_ARG;
  if (cfg->bits != 2 && cfg->bits != 3 && cfg->bits != 4 && cfg->bits != 8)
    return GPTQ_ERR_INVALID_ARG;
  if (cfg->sym != 0 && cfg->sym != 1) return GPTQ_ERR_INVALID_ARG;
  if (cfg->act_order < GPTQ_ORDER_NATURAL || cfg->act_order > GPTQ_ORDER_GIVEN)
    return GPTQ_ERR_INVALID_ARG;
  if (!(cfg->damp >= 0.f) || !std::isfinite(cfg->damp)) return GPTQ_ERR_INVALID_ARG;
  if (cfg->block_size < 1) return GPTQ_ERR_INVALID_ARG;
  if (cfg->group_size < -1) return GPTQ_ERR_INVALID_ARG;
  return GPTQ_OK;
}
}  // namespace gptq

static gptq_status check_group(const gptq_config* cfg) {
  const int g = cfg->group_size;
  if (g <= 0) return GPTQ_OK;
  if (128 % g != 0) return GPTQ_ERR_UNSUPPORTED;
  const int B = cfg->block_size;
  if (g % B != 0 && B % g != 0) return GPTQ_ERR_UNSUPPORTED;
  return GPTQ_OK;
}

static bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

extern "C" {

size_t gptq_workspace_size(int op, int64_t rows, int64_t cols, const gptq_config* cfg) {
  if (cols <= 0 || cols > INT_MAX / 2 || rows < 0 || rows > INT_MAX) return 0;
  if (check_cfg(cfg) != GPTQ_OK) return 0;
  if (op == GPTQ_OP_PREPARE) return prepare_ws_bytes(cols);
  if (op == GPTQ_OP_QUANTIZE) return quantize_ws_bytes(rows, cols, *cfg);
  return 0;
}

gptq_status gptq_hessian_accumulate(float* H, int64_t* n_seen, const void* X, int xdtype,
                                    int64_t m_tokens, int64_t cols, int64_t ldx,
                                    int32_t* dev_status, void* stream) {
  CallRange range_("gptq_hessian_accumulate");
  if (!H || !n_seen || cols <= 0 || cols > INT_MAX / 2 || m_tokens < 0 || *n_seen < 0)
    return GPTQ_ERR_INVALID_ARG;
  if (!valid_dtype(xdtype) || ldx < cols) return GPTQ_ERR_INVALID_ARG;
  if (m_tokens == 0) return GPTQ_OK;
  if (!X) return GPTQ_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  const int64_t n = *n_seen;
  const double tot = double(n) + double(m_tokens);
  GPTQ_TRY(hessian_prescale(st, H, int(cols), double(n) / tot, n == 0));
  const float beta = float(2.0 / tot);
  gptq_status s = hessian_syrk_tc(st, H, X, xdtype, m_tokens, int(cols), ldx, beta, dev_status);
  if (s == GPTQ_ERR_UNSUPPORTED)
    s = hessian_syrk_simt(st, H, X, xdtype, m_tokens, int(cols), ldx, beta);
  if (s != GPTQ_OK) return s;
  *n_seen = n + m_tokens;
  return GPTQ_OK;
}

gptq_status gptq_prepare(const float* H, int64_t cols, const gptq_config* cfg, float* U,
                         int32_t* perm, void* ws, size_t ws_bytes, int32_t* dev_status,
                         void* stream) {
  CallRange range_("gptq_prepare");
  if (!H || !U || !perm || cols <= 0 || cols > INT_MAX / 2) return GPTQ_ERR_INVALID_ARG;
  GPTQ_TRY(check_cfg(cfg));
  if (!ws || !aligned256(ws)) return GPTQ_ERR_INVALID_ARG;
  if (ws_bytes < prepare_ws_bytes(cols)) return GPTQ_ERR_WORKSPACE;
  return prepare_run(as_stream(stream), H, int(cols), *cfg, U, perm, ws, dev_status);
}

gptq_status gptq_quantize_layer(const void* W, int wdtype, int64_t rows, int64_t cols,
                                int64_t ldw, const float* U, const int32_t* perm,
                                const gptq_config* cfg, uint8_t* codes, float* scales,
                                float* zeros, int32_t* g_idx, float* losses, void* ws,
                                size_t ws_bytes, int32_t* dev_status, void* stream) {
  CallRange range_("gptq_quantize_layer");
  if (cols <= 0 || cols > INT_MAX / 2 || rows < 0 || rows > INT_MAX) return GPTQ_ERR_INVALID_ARG;
  if (!U || !perm || !g_idx || !losses) return GPTQ_ERR_INVALID_ARG;
  if (rows > 0 && (!W || !codes || !scales || !zeros)) return GPTQ_ERR_INVALID_ARG;
  if (!valid_dtype(wdtype) || ldw < cols) return GPTQ_ERR_INVALID_ARG;
  GPTQ_TRY(check_cfg(cfg));
  GPTQ_TRY(check_group(cfg));
  if (!ws || !aligned256(ws)) return GPTQ_ERR_INVALID_ARG;
  if (ws_bytes < quantize_ws_bytes(rows, cols, *cfg)) return GPTQ_ERR_WORKSPACE;
  return quantize_run(as_stream(stream), W, wdtype, int(rows), int(cols), ldw, U, perm, *cfg,
                      codes, scales, zeros, g_idx, losses, ws, dev_status);
}

gptq_status gptq_pack(const uint8_t* codes, int64_t rows, int64_t cols, int bits,
                      uint32_t* packed, void* stream) {
  CallRange range_("gptq_pack");
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return GPTQ_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0) return GPTQ_ERR_INVALID_ARG;
  if (rows > 0 && cols > 0 && (!codes || !packed)) return GPTQ_ERR_INVALID_ARG;
  return pack_run(as_stream(stream), codes, rows, cols, bits, packed);
}

const char* gptq_status_string(int status) {
  switch (status) {
    case GPTQ_OK: return "GPTQ_OK";
    case GPTQ_ERR_INVALID_ARG: return "GPTQ_ERR_INVALID_ARG";
    case GPTQ_ERR_UNSUPPORTED: return "GPTQ_ERR_UNSUPPORTED";
    case GPTQ_ERR_WORKSPACE: return "GPTQ_ERR_WORKSPACE";
    case GPTQ_ERR_NOT_PD: return "GPTQ_ERR_NOT_PD";
    case GPTQ_ERR_NONFINITE: return "GPTQ_ERR_NONFINITE";
    case GPTQ_ERR_TIMEOUT: return "GPTQ_ERR_TIMEOUT";
    case GPTQ_ERR_CUDA: return "GPTQ_ERR_CUDA";
    default: return "GPTQ_ERR_<combined>";
  }
}

gptq_status gptq_selftest_timeout(int which, int32_t* dev_status, void* stream) {
  CallRange range_("gptq_selftest_timeout");
  if (!dev_status) return GPTQ_ERR_INVALID_ARG;
  if (which == GPTQ_SELFTEST_MBARRIER) return selftest_mbarrier(as_stream(stream), dev_status);
  if (which == GPTQ_SELFTEST_GRID_BARRIER)
    return selftest_grid_barrier(as_stream(stream), dev_status);
  return GPTQ_ERR_INVALID_ARG;
}

gptq_status gptq_repack_sweep_order(const uint32_t* packed, int64_t rows, int64_t cols, int bits,
                                    const int32_t* perm, uint32_t* out, void* stream) {
  CallRange range_("gptq_repack_sweep_order");
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return GPTQ_ERR_INVALID_ARG;
  if (rows < 0 || rows > INT_MAX || cols <= 0 || cols > INT_MAX / 2 || cols % 32 != 0)
    return GPTQ_ERR_INVALID_ARG;
  if (rows > 0 && (!packed || !out)) return GPTQ_ERR_INVALID_ARG;
  return repack_sweep_run(as_stream(stream), packed, int(rows), int(cols), bits, perm, out);
}

gptq_status gptq_dequant_matmul(const void* X, int xdtype, int64_t m_tokens, int64_t cols,
                                int64_t ldx, const uint32_t* qp, const float* scales,
                                const float* zeros, int bits, int group_size,
                                const int32_t* perm, float* Y, int64_t rows, int half_sums,
                                void* stream) {
  CallRange range_("gptq_dequant_matmul");
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return GPTQ_ERR_INVALID_ARG;
  if (rows < 0 || rows > INT_MAX || cols <= 0 || cols > INT_MAX / 2 || cols % 32 != 0)
    return GPTQ_ERR_INVALID_ARG;
  if (m_tokens < 1 || m_tokens > INT_MAX || !valid_dtype(xdtype) || ldx < cols)
    return GPTQ_ERR_INVALID_ARG;
  if (group_size != 0 && group_size != -1 && group_size != 32 && group_size != 64 &&
      group_size != 128)
    return GPTQ_ERR_UNSUPPORTED;
  if (!X || !Y) return GPTQ_ERR_INVALID_ARG;
  if (rows > 0 && (!qp || !scales || !zeros)) return GPTQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(qp) & 15) != 0) return GPTQ_ERR_INVALID_ARG;
  return dequant_matmul_run(as_stream(stream), X, xdtype, int(m_tokens), int(cols), ldx, qp,
                            scales, zeros, bits, group_size > 0 ? group_size : 0, perm, Y,
                            int(rows), half_sums != 0);
}

uint32_t gptq_debug_set_wait_limit(uint32_t polls) {
  const uint32_t old = g_wait_limit.exchange(polls, std::memory_order_relaxed);
  return old ? old : tc::WAIT_LIMIT;
}

uint64_t gptq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* gptq_last_error(void) { return g_last_error; }

}  // extern "C"
