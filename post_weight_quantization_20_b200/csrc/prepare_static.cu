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
// memory.  The device address is looked up with cudaGetSymbolAddress while the
// device is current, on the first call made in a device's context, and cached
// together with that context's id: after a device reset the context (and the
// module holding the array) is a new one, its id differs, and the next call looks
// the address up again instead of using a stale one.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.h"

namespace gptq {

static __device__ __align__(256) unsigned char g_prepare_scratch[GPTQ_STATIC_SCRATCH_BYTES];

static constexpr int kMaxDevices = 64;

struct ScratchSlot {
  void* ptr;
  unsigned long long ctx_id;   // id of the context the address belongs to
  bool valid;
};

static std::mutex g_setup_mutex;
static ScratchSlot g_scratch[kMaxDevices] = {};

// The driver calls that name the current context, fetched at run time (the
// library does not link libcuda).
struct CtxFns {
  PFN_cuCtxGetCurrent get_current = nullptr;
  PFN_cuCtxGetId get_id = nullptr;
};

static const CtxFns& ctx_fns() {
  static CtxFns fns;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.get_current = reinterpret_cast<PFN_cuCtxGetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.get_id = reinterpret_cast<PFN_cuCtxGetId>(p);
  });
  return fns;
}

// Id of the calling thread's current context; false if there is none (or the
// driver cannot say).
static bool current_ctx_id(unsigned long long* id) {
  const CtxFns& f = ctx_fns();
  if (!f.get_current || !f.get_id) return false;
  CUcontext ctx = nullptr;
  if (f.get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return f.get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_prepare_scratch in the current device's context.
static gptq_status scratch_for_current_device(void** out) {
  int dev = -1;
  GPTQ_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return GPTQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  unsigned long long id = 0;
  ScratchSlot& slot = g_scratch[dev];
  if (slot.valid && current_ctx_id(&id) && id == slot.ctx_id) {
    *out = slot.ptr;
    return GPTQ_OK;
  }
  // first call in this context: the lookup also makes the device's primary
  // context current if nothing has yet
  void* p = nullptr;
  GPTQ_CUDA(cudaGetSymbolAddress(&p, g_prepare_scratch));
  slot.ptr = p;
  slot.valid = current_ctx_id(&id);   // without an id, look the address up every call
  slot.ctx_id = id;
  *out = p;
  return GPTQ_OK;
}

}  // namespace gptq

using namespace gptq;

extern "C" gptq_status gptq_prepare_static(const float* H, int64_t cols, const gptq_config* cfg,
                                           float* U, int32_t* perm, int32_t* dev_status,
                                           void* stream) {
  gptq::CallRange range_("gptq_prepare_static");
  if (!H || !U || !perm || cols <= 0) return GPTQ_ERR_INVALID_ARG;
  GPTQ_TRY(check_cfg(cfg));   // the same configuration rules as gptq_prepare
  // sizes the built-in array cannot hold are refused before anything is launched
  if (cols > GPTQ_STATIC_MAX_COLS || prepare_ws_bytes(cols) > GPTQ_STATIC_SCRATCH_BYTES)
    return GPTQ_ERR_WORKSPACE;
  void* ws = nullptr;
  GPTQ_TRY(scratch_for_current_device(&ws));
  return prepare_run(as_stream(stream), H, int(cols), *cfg, U, perm, ws, dev_status);
}
