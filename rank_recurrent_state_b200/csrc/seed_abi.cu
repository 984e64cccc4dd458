// seed_abi.cu -- the extern "C" entry points of libseed.so: argument validation,
// then one kernel launch on the caller's stream.  No entry point allocates.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "../../include/seed.h"
#include "../../include/seed_synth.h"
#include "seed_launch.h"

namespace {

constexpr size_t kWorkspaceBytes = 256;   // the device status word and counters, padded
constexpr int kDiagCounters = 6;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_dims(const seed_dims* d) {
  if (!d) return SEED_ERR_INVALID_ARG;
  if (d->form < SEED_GDN || d->form > SEED_MAMBA2) return SEED_ERR_INVALID_ARG;
  if (d->factors < SEED_FACTORS_F32 || d->factors > SEED_FACTORS_BF16) return SEED_ERR_INVALID_ARG;
  if (d->batch < 1 || d->layers < 1 || d->heads < 1 || d->R < 1 || d->W < 1)
    return SEED_ERR_INVALID_ARG;
  if (!seed::decode_dims_supported(d->d_k, d->d_v)) return SEED_ERR_SHAPE;
  const int m = d->R + d->W;
  if (m > SEED_MAX_COLS) return SEED_ERR_SHAPE;
  if (m > d->d_k || m > d->d_v) return SEED_ERR_SHAPE;
  const long long blocks = (long long)d->batch * d->heads * d->layers;
  if (blocks > 0x7fffffffLL) return SEED_ERR_SHAPE;
  return SEED_OK;
}

int check_layer(const seed_dims* d, int32_t layer, bool allow_all) {
  if (layer == SEED_ALL_LAYERS) return allow_all ? SEED_OK : SEED_ERR_INVALID_ARG;
  return (layer >= 0 && layer < d->layers) ? SEED_OK : SEED_ERR_INVALID_ARG;
}

int check_ptr(const void* p) {
  if (!p) return SEED_ERR_INVALID_ARG;
  return aligned16(p) ? SEED_OK : SEED_ERR_ALIGN;
}

int check_opt_ptr(const void* p) { return p ? check_ptr(p) : SEED_OK; }

int check_ws(void* ws, size_t ws_bytes) {
  if (!ws || ws_bytes < kWorkspaceBytes) return SEED_ERR_WORKSPACE;
  return aligned16(ws) ? SEED_OK : SEED_ERR_ALIGN;
}

int check_state(const seed_state* s) {
  if (!s) return SEED_ERR_INVALID_ARG;
  int rc;
  if ((rc = check_ptr(s->a)) || (rc = check_ptr(s->U)) || (rc = check_ptr(s->V)) ||
      (rc = check_ptr(s->scale)) || (rc = check_ptr(s->ncols)) || (rc = check_ptr(s->vbar)))
    return rc;
  return SEED_OK;
}

#define SEED_TRY(x)          \
  do {                       \
    const int rc_ = (x);     \
    if (rc_) return rc_;     \
  } while (0)

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline uint32_t* status_word(void* ws) { return reinterpret_cast<uint32_t*>(ws); }

}  // namespace

extern "C" {

int32_t seed_scale_len(const seed_dims* dims) {
  if (check_dims(dims)) return -1;
  return seed::scale_len(*dims);
}

size_t seed_workspace_bytes(const seed_dims* dims) {
  (void)dims;
  return kWorkspaceBytes;
}

int seed_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  SEED_TRY(check_ws(ws, ws_bytes));
  return cudaMemsetAsync(ws, 0, kWorkspaceBytes, as_stream(stream)) == cudaSuccess ? SEED_OK
                                                                                     : SEED_ERR_CUDA;
}

int seed_state_init_from_dense(const seed_dims* dims, const seed_state* state, int32_t layer,
                               const float* S_dense, float* sigma_out, void* ws, size_t ws_bytes,
                               void* stream) {
  SEED_TRY(check_dims(dims));
  SEED_TRY(check_layer(dims, layer, true));
  SEED_TRY(check_state(state));
  SEED_TRY(check_ptr(S_dense));
  SEED_TRY(check_opt_ptr(sigma_out));
  SEED_TRY(check_ws(ws, ws_bytes));
  return seed::launch_init_from_dense(*dims, *state, layer, S_dense, sigma_out, status_word(ws),
                                      as_stream(stream));
}

int seed_decode_step(const seed_dims* dims, const seed_state* state, int32_t layer, const float* q,
                     const float* k, const float* v, const float* alpha, const float* beta,
                     float* o, void* ws, size_t ws_bytes, void* stream) {
  SEED_TRY(check_dims(dims));
  SEED_TRY(check_layer(dims, layer, false));
  SEED_TRY(check_state(state));
  SEED_TRY(check_ptr(q));
  SEED_TRY(check_ptr(k));
  SEED_TRY(check_ptr(v));
  SEED_TRY(check_ptr(alpha));
  SEED_TRY(check_ptr(beta));
  SEED_TRY(check_ptr(o));
  SEED_TRY(check_ws(ws, ws_bytes));
  return seed::launch_decode_step(*dims, *state, layer, q, k, v, alpha, beta, o, status_word(ws),
                                  as_stream(stream));
}

int seed_decode_step_overlapped(const seed_dims* dims, const seed_state* state, int32_t layer, const float* q,
                                const float* k, const float* v, const float* alpha, const float* beta,
                                float* o, void* ws, size_t ws_bytes, void* stream) {
  SEED_TRY(check_dims(dims));
  SEED_TRY(check_layer(dims, layer, false));
  SEED_TRY(check_state(state));
  SEED_TRY(check_ptr(q));
  SEED_TRY(check_ptr(k));
  SEED_TRY(check_ptr(v));
  SEED_TRY(check_ptr(alpha));
  SEED_TRY(check_ptr(beta));
  SEED_TRY(check_ptr(o));
  SEED_TRY(check_ws(ws, ws_bytes));
  return seed::launch_decode_step(*dims, *state, layer, q, k, v, alpha, beta, o, status_word(ws),
                                  as_stream(stream), true);
}

int seed_decode_step_compress(const seed_dims* dims, const seed_state* state, int32_t layer, const float* q,
                              const float* k, const float* v, const float* alpha, const float* beta, float* o,
                              float* sigma_out, void* ws, size_t ws_bytes, void* stream) {
  SEED_TRY(check_dims(dims));
  SEED_TRY(check_layer(dims, layer, false));
  SEED_TRY(check_state(state));
  SEED_TRY(check_ptr(q));
  SEED_TRY(check_ptr(k));
  SEED_TRY(check_ptr(v));
  SEED_TRY(check_ptr(alpha));
  SEED_TRY(check_ptr(beta));
  SEED_TRY(check_ptr(o));
  SEED_TRY(check_opt_ptr(sigma_out));
  SEED_TRY(check_ws(ws, ws_bytes));
  return seed::launch_decode_compress(*dims, *state, layer, q, k, v, alpha, beta, o, sigma_out, status_word(ws),
                                      as_stream(stream));
}

int seed_compress(const seed_dims* dims, const seed_state* state, int32_t layer, float* sigma_out,
                  void* ws, size_t ws_bytes, void* stream) {
  SEED_TRY(check_dims(dims));
  SEED_TRY(check_layer(dims, layer, true));
  SEED_TRY(check_state(state));
  SEED_TRY(check_opt_ptr(sigma_out));
  SEED_TRY(check_ws(ws, ws_bytes));
  return seed::launch_compress(*dims, *state, layer, sigma_out, status_word(ws), as_stream(stream));
}

int seed_state_to_dense(const seed_dims* dims, const seed_state* state, int32_t layer,
                        const int32_t* units, int32_t n_units, float* S_out, void* ws,
                        size_t ws_bytes, void* stream) {
  SEED_TRY(check_dims(dims));
  SEED_TRY(check_layer(dims, layer, true));
  SEED_TRY(check_state(state));
  SEED_TRY(check_ptr(S_out));
  SEED_TRY(check_ws(ws, ws_bytes));
  const long long scope = (long long)dims->batch * dims->heads * (layer < 0 ? dims->layers : 1);
  if (units) {
    if (n_units < 0 || n_units > scope) return SEED_ERR_INVALID_ARG;
    if (n_units == 0) return SEED_OK;
    SEED_TRY(check_ptr(units));
  } else {
    n_units = (int32_t)scope;
  }
  return seed::launch_to_dense(*dims, *state, layer, units, n_units, S_out, status_word(ws),
                               as_stream(stream));
}

int seed_state_energy(const seed_dims* dims, const seed_state* state, int32_t layer,
                      const int32_t* units, int32_t n_units, float* out, void* ws, size_t ws_bytes,
                      void* stream) {
  SEED_TRY(check_dims(dims));
  SEED_TRY(check_layer(dims, layer, true));
  SEED_TRY(check_state(state));
  SEED_TRY(check_ptr(out));
  SEED_TRY(check_ws(ws, ws_bytes));
  const long long scope = (long long)dims->batch * dims->heads * (layer < 0 ? dims->layers : 1);
  if (units) {
    if (n_units < 0 || n_units > scope) return SEED_ERR_INVALID_ARG;
    if (n_units == 0) return SEED_OK;
    SEED_TRY(check_ptr(units));
  } else {
    n_units = (int32_t)scope;
  }
  return seed::launch_state_energy(*dims, *state, layer, units, n_units, out, status_word(ws),
                                   as_stream(stream));
}

int seed_state_spectrum(const seed_dims* dims, const seed_state* state, int32_t layer, const int32_t* units,
                        int32_t n_units, float* sigma_state, float* sigma_content, float* cos_top,
                        int32_t* ranks, void* ws, size_t ws_bytes, void* stream) {
  SEED_TRY(check_dims(dims));
  SEED_TRY(check_layer(dims, layer, true));
  SEED_TRY(check_state(state));
  SEED_TRY(check_ptr(sigma_state));
  SEED_TRY(check_ptr(sigma_content));
  SEED_TRY(check_ptr(cos_top));
  SEED_TRY(check_ptr(ranks));
  SEED_TRY(check_ws(ws, ws_bytes));
  const long long scope = (long long)dims->batch * dims->heads * (layer < 0 ? dims->layers : 1);
  if (units) {
    if (n_units < 0 || n_units > scope) return SEED_ERR_INVALID_ARG;
    if (n_units == 0) return SEED_OK;
    SEED_TRY(check_ptr(units));
  } else {
    n_units = (int32_t)scope;
  }
  return seed::launch_state_spectrum(*dims, *state, layer, units, n_units, sigma_state, sigma_content, cos_top,
                                     ranks, status_word(ws), as_stream(stream));
}

int seed_dense_step(const seed_dims* dims, float* S, int32_t layer, const float* q, const float* k,
                    const float* v, const float* alpha, const float* beta, float* o, void* ws,
                    size_t ws_bytes, void* stream) {
  SEED_TRY(check_dims(dims));
  SEED_TRY(check_layer(dims, layer, false));
  SEED_TRY(check_ptr(S));
  SEED_TRY(check_ptr(q));
  SEED_TRY(check_ptr(k));
  SEED_TRY(check_ptr(v));
  SEED_TRY(check_ptr(alpha));
  SEED_TRY(check_ptr(beta));
  SEED_TRY(check_ptr(o));
  SEED_TRY(check_ws(ws, ws_bytes));
  return seed::launch_dense_step(*dims, S, layer, q, k, v, alpha, beta, o, status_word(ws),
                                 as_stream(stream));
}

int seed_get_status(void* ws, void* stream, uint32_t* flags) {
  if (!flags) return SEED_ERR_INVALID_ARG;
  SEED_TRY(check_ws(ws, kWorkspaceBytes));
  cudaStream_t st = as_stream(stream);
  uint32_t host = 0;
  if (cudaMemcpyAsync(&host, ws, sizeof(uint32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return SEED_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), st) != cudaSuccess) return SEED_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SEED_ERR_CUDA;
  *flags = host;
  return SEED_OK;
}

int seed_get_diagnostics(void* ws, void* stream, uint32_t* counters) {
  if (!counters) return SEED_ERR_INVALID_ARG;
  SEED_TRY(check_ws(ws, kWorkspaceBytes));
  cudaStream_t st = as_stream(stream);
  uint32_t host[kDiagCounters] = {0};
  uint32_t* dev = status_word(ws) + 1;
  if (cudaMemcpyAsync(host, dev, sizeof(host), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return SEED_ERR_CUDA;
  if (cudaMemsetAsync(dev, 0, sizeof(host), st) != cudaSuccess) return SEED_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SEED_ERR_CUDA;
  for (int i = 0; i < kDiagCounters; ++i) counters[i] = host[i];
  return SEED_OK;
}

int seed_debug_wait_fault(void* ws, size_t ws_bytes, int32_t enable, void* stream) {
  SEED_TRY(check_ws(ws, ws_bytes));
  uint32_t* word = status_word(ws) + seed::kWsWaitFaultWordHost;
  return cudaMemsetAsync(word, enable ? 1 : 0, sizeof(uint32_t), as_stream(stream)) == cudaSuccess
             ? SEED_OK
             : SEED_ERR_CUDA;
}

const char* seed_status_string(int status) {
  switch (status) {
    case SEED_OK: return "ok";
    case SEED_ERR_INVALID_ARG: return "invalid argument";
    case SEED_ERR_SHAPE: return "unsupported shape";
    case SEED_ERR_ALIGN: return "pointer not 16-byte aligned";
    case SEED_ERR_CUDA: return "CUDA error";
    case SEED_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

// ------------------------------------------------------------------ synthetic workloads
int seed_synth_vbar(const seed_dims* dims, seed_synth_key key, float* vbar, void* stream) {
  SEED_TRY(check_dims(dims));
  SEED_TRY(check_ptr(vbar));
  return seed::launch_synth_vbar(*dims, key, vbar, as_stream(stream));
}

int seed_synth_token_inputs(const seed_dims* dims, seed_synth_key key, int32_t phase, int32_t t,
                            int32_t layer, const float* vbar, float* q, float* k, float* v,
                            float* alpha, float* beta, void* stream) {
  SEED_TRY(check_dims(dims));
  SEED_TRY(check_layer(dims, layer, false));
  if (phase != SEED_PHASE_PREFILL && phase != SEED_PHASE_DECODE && phase != SEED_PHASE_LEADIN)
    return SEED_ERR_INVALID_ARG;
  if (t < 0 || key.b0 < 0) return SEED_ERR_INVALID_ARG;
  SEED_TRY(check_ptr(vbar));
  SEED_TRY(check_opt_ptr(q));
  SEED_TRY(check_ptr(k));
  SEED_TRY(check_ptr(v));
  SEED_TRY(check_ptr(alpha));
  SEED_TRY(check_ptr(beta));
  return seed::launch_synth_token_inputs(*dims, key, phase, t, layer, vbar, q, k, v, alpha, beta,
                                         as_stream(stream));
}

int seed_synth_dense_prefill(const seed_dims* dims, seed_synth_key key, int32_t n_tokens,
                             int32_t layer, const float* vbar, float* S_out, void* stream) {
  SEED_TRY(check_dims(dims));
  SEED_TRY(check_layer(dims, layer, true));
  if (n_tokens < 0 || key.b0 < 0) return SEED_ERR_INVALID_ARG;
  SEED_TRY(check_ptr(vbar));
  SEED_TRY(check_ptr(S_out));
  return seed::launch_synth_dense_prefill(*dims, key, n_tokens, layer, vbar, S_out,
                                          as_stream(stream));
}

}  // extern "C"
