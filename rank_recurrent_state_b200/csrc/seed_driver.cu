// seed_driver.cu -- CUDA driver entry points the launchers use, looked up once
// through the runtime (no link against libcuda), and the per-device launch facts
// the launchers cache.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "seed_launch.h"

namespace seed {

namespace {

struct DriverFns {
  PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  CUresult (*ctx_current)(CUcontext*) = nullptr;
  CUresult (*ctx_id)(CUcontext, unsigned long long*) = nullptr;
};

const DriverFns& driver_fns() {
  static std::once_flag once;
  static DriverFns fns;
  std::call_once(once, [] {
    auto get = [](const char* name) -> void* {
      void* p = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPointByVersion(name, &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess)
        return nullptr;
      return p;
    };
    fns.encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(get("cuTensorMapEncodeTiled"));
    fns.ctx_current = reinterpret_cast<CUresult (*)(CUcontext*)>(get("cuCtxGetCurrent"));
    fns.ctx_id = reinterpret_cast<CUresult (*)(CUcontext, unsigned long long*)>(get("cuCtxGetId"));
  });
  return fns;
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() { return driver_fns().encode; }

unsigned long long current_context_id() {
  const DriverFns& f = driver_fns();
  if (!f.ctx_current || !f.ctx_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (f.ctx_current(&ctx) != CUDA_SUCCESS || !ctx || f.ctx_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

int LaunchCache::prepare(const void* kernel, size_t max_dyn_smem, int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return SEED_ERR_CUDA;
  *dev_out = dev;
  if (sm_count[dev].load(std::memory_order_relaxed) == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      return SEED_ERR_CUDA;
    sm_count[dev].store(n, std::memory_order_relaxed);
  }
  if (max_dyn_smem > 48 * 1024) {
    // the opt-in belongs to the function in the current context: set it again
    // whenever the context has changed (a device reset loads the module afresh)
    const unsigned long long id = current_context_id();
    if (id == 0 || attr_ctx[dev].load(std::memory_order_acquire) != id) {
      if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)max_dyn_smem) !=
          cudaSuccess)
        return SEED_ERR_CUDA;
      attr_ctx[dev].store(id, std::memory_order_release);
    }
  }
  return SEED_OK;
}

}  // namespace seed
