// seed_noalloc.cu -- seed_decode_step for callers that cannot allocate device memory.
//
// Every other entry point takes a workspace that the caller allocated: 256 bytes
// holding the device status word the kernels raise flags in, plus counters.  Some
// callers cannot provide one: a host program that links libseed.so without a
// device allocator of its own (no torch, no CUDA memory pool), or a serving
// engine whose memory planner fixes every device buffer before serving starts
// and refuses allocations inside its decode loop.  seed_decode_step_noalloc runs
// the same decode kernel with its workspace in a fixed array that is part of the
// library's device image; the call itself allocates nothing.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/seed.h"

namespace {

// The decode step's workspace: only its first word (the status flags) is
// written by the decode kernel.  Zero at module load; every call clears the
// status word again after copying it out, so each call starts from zero.  One
// array per device, shared by every call on that device.
constexpr size_t kStaticWsBytes = 256;
static __device__ __align__(256) unsigned char g_seed_static_ws[kStaticWsBytes];

constexpr int kMaxDevices = 64;

// Per device: the array's device address and the unique id of the context it
// was looked up in.  A device reset (cudaDeviceReset, or the primary context
// being released and created again) gives the device a new context with a new
// id, in which the module is loaded again, possibly at another address; the
// next call sees the id change and looks the address up again, so no call
// writes through an address of a context that no longer exists.
struct StaticWsSlot {
  std::mutex mu;
  unsigned long long ctx_id = 0;   // 0: not looked up yet (context ids start at 1)
  void* ptr = nullptr;
};
StaticWsSlot g_slots[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// cuCtxGetCurrent and cuCtxGetId from the driver (CUDA 12.0 and later).
bool driver_ctx_fns(CtxGetCurrentFn* cur, CtxGetIdFn* id) {
  static std::once_flag once;
  static CtxGetCurrentFn s_cur = nullptr;
  static CtxGetIdFn s_id = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      s_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      s_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  *cur = s_cur;
  *id = s_id;
  return s_cur && s_id;
}

// Device address of g_seed_static_ws in the current device's current context:
// looked up once per device (with that device current) and again only when the
// device's context has changed since.  The first lookup may load the library's
// module onto the device.
int static_ws_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SEED_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SEED_ERR_INVALID_ARG;
  CtxGetCurrentFn get_cur;
  CtxGetIdFn get_id;
  if (!driver_ctx_fns(&get_cur, &get_id)) return SEED_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS) return SEED_ERR_CUDA;
  if (!ctx) {
    // no context is current on this thread yet: since CUDA 12.0 cudaSetDevice
    // creates the device's primary context and makes it current
    if (cudaSetDevice(dev) != cudaSuccess || get_cur(&ctx) != CUDA_SUCCESS || !ctx) return SEED_ERR_CUDA;
  }
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS || id == 0) return SEED_ERR_CUDA;
  StaticWsSlot& slot = g_slots[dev];
  std::lock_guard<std::mutex> lock(slot.mu);
  if (slot.ctx_id != id || !slot.ptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_seed_static_ws) != cudaSuccess || !ptr) return SEED_ERR_CUDA;
    slot.ptr = ptr;
    slot.ctx_id = id;
  }
  *out = slot.ptr;
  return SEED_OK;
}

}  // namespace

extern "C" {

size_t seed_noalloc_workspace_bytes(void) { return kStaticWsBytes; }

int seed_decode_step_noalloc(const seed_dims* dims, const seed_state* state, int32_t layer,
                             const float* q, const float* k, const float* v, const float* alpha,
                             const float* beta, float* o, uint32_t* status_out, void* stream) {
  if (!dims) return SEED_ERR_INVALID_ARG;
  if (seed_workspace_bytes(dims) > kStaticWsBytes) return SEED_ERR_WORKSPACE;
  if (status_out && (reinterpret_cast<uintptr_t>(status_out) & 3u)) return SEED_ERR_ALIGN;
  void* ws = nullptr;
  int rc = static_ws_address(&ws);
  if (rc != SEED_OK) return rc;
  // validates every argument before it enqueues anything
  rc = seed_decode_step(dims, state, layer, q, k, v, alpha, beta, o, ws, kStaticWsBytes, stream);
  if (rc != SEED_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (status_out &&
      cudaMemcpyAsync(status_out, ws, sizeof(uint32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return SEED_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), st) != cudaSuccess) return SEED_ERR_CUDA;
  return SEED_OK;
}

}  // extern "C"
