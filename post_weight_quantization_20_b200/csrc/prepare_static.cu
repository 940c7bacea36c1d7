// gptq_prepare_static: gptq_prepare without a caller workspace.
//
// Some callers cannot allocate device memory where they call us: a plugin
// running inside a framework whose caching allocator has already reserved the
// device's memory, code handed a fixed memory budget up front, or a service that
// must not allocate after start-up because an allocation can block and
// synchronize the device.  This entry point serves them: its scratch memory is a
// fixed array compiled into the library, so the call allocates nothing.  The
// caller still provides H, U, perm and the status word.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds GPTQ_STATIC_SCRATCH_BYTES of it until the process exits.  In
// host code the array's name only stands in for the device variable; it is not
// a device address, and a kernel handed it would fault or read the wrong
// memory.  The device address is looked up with cudaGetSymbolAddress once per
// device, while that device is current, on the first call made on that device,
// and cached for later calls.
#include <cmath>
#include <mutex>

#include "kernels.h"

namespace gptq {

static __device__ __align__(256) unsigned char g_prepare_scratch[GPTQ_STATIC_SCRATCH_BYTES];

static constexpr int kMaxDevices = 64;
static std::mutex g_setup_mutex;
static void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_prepare_scratch on the current device (looked up on first use).
static gptq_status scratch_for_current_device(void** out) {
  int dev = -1;
  GPTQ_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return GPTQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    GPTQ_CUDA(cudaGetSymbolAddress(&p, g_prepare_scratch));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return GPTQ_OK;
}

}  // namespace gptq

using namespace gptq;

extern "C" gptq_status gptq_prepare_static(const float* H, int64_t cols, const gptq_config* cfg,
                                           float* U, int32_t* perm, int32_t* dev_status,
                                           void* stream) {
  gptq::CallRange range_("gptq_prepare_static");
  if (!H || !U || !perm || cols <= 0 || !cfg) return GPTQ_ERR_INVALID_ARG;
  if (cfg->bits != 2 && cfg->bits != 3 && cfg->bits != 4 && cfg->bits != 8)
    return GPTQ_ERR_INVALID_ARG;
  if (cfg->sym != 0 && cfg->sym != 1) return GPTQ_ERR_INVALID_ARG;
  if (cfg->act_order < GPTQ_ORDER_NATURAL || cfg->act_order > GPTQ_ORDER_GIVEN)
    return GPTQ_ERR_INVALID_ARG;
  if (!(cfg->damp >= 0.f) || !std::isfinite(cfg->damp)) return GPTQ_ERR_INVALID_ARG;
  if (cfg->block_size < 1 || cfg->group_size < -1) return GPTQ_ERR_INVALID_ARG;
  // sizes the built-in array cannot hold are refused before anything is launched
  if (cols > GPTQ_STATIC_MAX_COLS || prepare_ws_bytes(cols) > GPTQ_STATIC_SCRATCH_BYTES)
    return GPTQ_ERR_WORKSPACE;
  void* ws = nullptr;
  GPTQ_TRY(scratch_for_current_device(&ws));
  return prepare_run(as_stream(stream), H, int(cols), *cfg, U, perm, ws, dev_status);
}
