// seed_launch.h -- host launchers behind the C ABI (internal to libseed).
// Arguments are validated by seed_abi.cu before any of these is called.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/seed.h"
#include "../../include/seed_synth.h"

namespace seed {

constexpr int kMaxDev = 64;

// Index (32-bit words from the status word) of the workspace word that turns on the
// injected wait fault of the timeout tests (kWsWaitFaultWord in seed_common.cuh).
constexpr int kWsWaitFaultWordHost = 8;

// cuTensorMapEncodeTiled from the driver, looked up once (nullptr if unavailable).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Unique id of the calling thread's current CUDA context; 0 if there is none.
unsigned long long current_context_id();

// Blocks of a persistent grid of at most max_blocks that deal `units` units round
// robin so that every block takes the same number of units, up to one: with
// k = ceil(units / max_blocks) units per block, ceil(units / k) blocks.  (A grid of
// max_blocks itself would leave a last round in which only units mod max_blocks
// blocks work.)
inline int balanced_grid(int units, int max_blocks) {
  if (units <= 0) return 1;
  if (max_blocks < 1) max_blocks = 1;
  const int k = (units + max_blocks - 1) / max_blocks;
  return (units + k - 1) / k;
}

// Per kernel instantiation and device: the SM count, and the context in which the
// kernel's dynamic shared-memory opt-in was last set (a device reset loads the
// module afresh, so the opt-in is set again in the new context).  Atomics: host
// threads that launch at the same time for the first time store equal values.
struct LaunchCache {
  std::atomic<int> sm_count[kMaxDev];
  std::atomic<unsigned long long> attr_ctx[kMaxDev];
  // Current device into *dev; sets the opt-in for max_dyn_smem bytes when above
  // the default 48 KB and not yet set in this context.
  int prepare(const void* kernel, size_t max_dyn_smem, int* dev);
};

// Per-unit length of seed_state.scale: d_k for KDA (the decay product P), else
// R + W rounded up to a multiple of 4 (column scales, 16-byte aligned per unit).
inline int scale_len(const seed_dims& d) {
  return d.form == SEED_KDA ? d.d_k : ((d.R + d.W + 3) & ~3);
}

// Bytes of one element of U and V.
inline int factor_bytes(const seed_dims& d) { return d.factors == SEED_FACTORS_F32 ? 4 : 2; }

// f(T{}) with T the element type of U and V (float, __half or __nv_bfloat16).
template <typename F>
int with_factor_type(const seed_dims& d, F&& f) {
  switch (d.factors) {
    case SEED_FACTORS_F32: return f(float{});
    case SEED_FACTORS_F16: return f(__half{});
    case SEED_FACTORS_BF16: return f(__nv_bfloat16{});
  }
  return SEED_ERR_INVALID_ARG;
}

bool decode_dims_supported(int dk, int dv);

// overlap: seed_decode_step_overlapped (the one-warp kernels, R + W <= 65, are then
// launched with programmatic stream serialization; the four-warp kernel as usual).
int launch_decode_step(const seed_dims& d, const seed_state& s, int layer, const float* q,
                       const float* k, const float* v, const float* alpha, const float* beta,
                       float* o, uint32_t* status, cudaStream_t st, bool overlap = false);

bool compress_fast_supported(const seed_dims& d);
int launch_compress_fast(const seed_dims& d, const seed_state& s, int layer, float* sigma_out,
                         uint32_t* status, cudaStream_t st);

// 32 < R + W <= 64, R <= 32 (seed_compress_wide.cu).
bool compress_wide_supported(const seed_dims& d);
int launch_compress_wide(const seed_dims& d, const seed_state& s, int layer, float* sigma_out,
                         uint32_t* status, cudaStream_t st);

int launch_compress(const seed_dims& d, const seed_state& s, int layer, float* sigma_out,
                    uint32_t* status, cudaStream_t st);

// The Householder compression alone (the units still holding R + W columns).
int launch_compress_householder(const seed_dims& d, const seed_state& s, int layer, float* sigma_out,
                                uint32_t* status, cudaStream_t st);

// The decode step of one layer with the compression of the units it brings to
// R + W columns (seed_decode_fused.cu).
bool decode_compress_fused_supported(const seed_dims& d);
int launch_decode_compress(const seed_dims& d, const seed_state& s, int layer, const float* q, const float* k,
                           const float* v, const float* alpha, const float* beta, float* o, float* sigma_out,
                           uint32_t* status, cudaStream_t st);

int launch_init_from_dense(const seed_dims& d, const seed_state& s, int layer, const float* S,
                           float* sigma_out, uint32_t* status, cudaStream_t st);

int launch_to_dense(const seed_dims& d, const seed_state& s, int layer, const int32_t* units,
                    int n_units, float* S_out, uint32_t* status, cudaStream_t st);

int launch_state_energy(const seed_dims& d, const seed_state& s, int layer, const int32_t* units,
                        int n_units, float* out, uint32_t* status, cudaStream_t st);

int launch_state_spectrum(const seed_dims& d, const seed_state& s, int layer, const int32_t* units, int n_units,
                          float* sigma_state, float* sigma_content, float* cos_top, int32_t* ranks,
                          uint32_t* status, cudaStream_t st);

int launch_dense_step(const seed_dims& d, float* S, int layer, const float* q, const float* k,
                      const float* v, const float* alpha, const float* beta, float* o,
                      uint32_t* status, cudaStream_t st);

int launch_synth_vbar(const seed_dims& d, const seed_synth_key& key, float* vbar, cudaStream_t st);

int launch_synth_token_inputs(const seed_dims& d, const seed_synth_key& key, int phase, int t,
                              int layer, const float* vbar, float* q, float* k, float* v,
                              float* alpha, float* beta, cudaStream_t st);

int launch_synth_dense_prefill(const seed_dims& d, const seed_synth_key& key, int n_tokens,
                               int layer, const float* vbar, float* S_out, cudaStream_t st);

}  // namespace seed
