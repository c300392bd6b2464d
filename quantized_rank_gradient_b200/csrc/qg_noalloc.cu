// qg_step_noalloc: the optimizer step with its scratch (P~ and N) held in a
// file-scope device array instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory for a workspace: for example a
// host program whose device memory is entirely owned by another allocator with
// a fixed budget (an extra cudaMalloc would break its accounting or fail), or a
// thread that must not pay the implicit device synchronisation that cudaMalloc
// and cudaFree can cause.  This entry point needs nothing but the layer's state,
// the weights and the gradient, which the caller already owns.
//
// The array is QG_NOALLOC_SCRATCH_BYTES large; every GPU that loads this library
// keeps it until the process exits.  In host code the array's name only stands
// for it: its device address is obtained with cudaGetSymbolAddress, with the
// device current, on the first call made in each CUDA context, and cached
// together with that context.  A call that finds another context current (the
// primary context was reset and built again, for example after
// cudaDeviceReset, which loads the module and its array anew) looks the
// address up again instead of using a stale one.  All calls share the array,
// so calls whose work overlaps on the GPU (other streams, other host threads)
// race on it; the step overwrites every byte it later reads, so nothing has to
// be cleared between calls.
#include <cuda.h>

#include <mutex>

#include "../../include/qgalore.h"
#include "qg_internal.h"

namespace {

static __device__ __align__(256) uint8_t g_step_scratch[QG_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// The driver's cuCtxGetCurrent, found once through the runtime.
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<CtxGetCurrentFn>(nullptr);
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  return fn;
}

// Device address of g_step_scratch in the current device's current context,
// looked up once per context.  A thread on which the runtime has not yet made a
// context current sees none; the lookup itself makes the device's primary
// context current, and the address is cached with that context.
cudaError_t scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  CtxGetCurrentFn get = ctx_get_current();
  if (!get) return cudaErrorDeviceUninitialized;
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!ctx || !g_scratch_ptr[dev] || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_step_scratch);
    if (e != cudaSuccess) return e;
    if (get(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorDeviceUninitialized;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

namespace qg {
// Defined in qg_api.cu: copies the layer's configuration.
qg_status layer_config(const qg_layer* layer, qg_config* out);
}  // namespace qg

extern "C" qg_status qg_step_noalloc(qg_layer* layer, const void* d_G, int64_t ldg, void* stream) {
  if (!layer || !d_G) return QG_EINVAL;
  qg_config cfg;
  if (qg::layer_config(layer, &cfg) != QG_OK) return QG_EINVAL;
  // Matrices whose scratch (P~ and N) does not fit the static array are refused.
  if (qg::step_scratch_bytes(cfg.m, cfg.n, cfg.r, cfg.proj_side) > QG_NOALLOC_SCRATCH_BYTES) return QG_ESHAPE;
  void* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return QG_ECUDA;
  // The regular step, with the static array as its workspace.
  return qg_step(layer, d_G, ldg, scratch, QG_NOALLOC_SCRATCH_BYTES, stream);
}
