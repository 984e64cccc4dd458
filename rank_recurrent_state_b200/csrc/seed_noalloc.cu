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
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/seed.h"

namespace {

// The decode step's workspace: only its first word (the status flags) is
// written by the decode kernel.  Zero at module load; every call clears the
// status word again after copying it out, so each call starts from zero.  One
// array per device, shared by every call on that device.
constexpr size_t kStaticWsBytes = 256;
static __device__ __align__(256) unsigned char g_seed_static_ws[kStaticWsBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_static_ws_ptr[kMaxDevices];

// Device address of g_seed_static_ws on the current device, looked up once per
// device.  The first lookup may load the library's module onto the device.
int static_ws_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SEED_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SEED_ERR_INVALID_ARG;
  void* ptr = g_static_ws_ptr[dev].load(std::memory_order_acquire);
  if (!ptr) {
    if (cudaGetSymbolAddress(&ptr, g_seed_static_ws) != cudaSuccess || !ptr) return SEED_ERR_CUDA;
    g_static_ws_ptr[dev].store(ptr, std::memory_order_release);
  }
  *out = ptr;
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
