// seed_decode_fused.cu -- the fused decode-and-compress entry: the fused launch
// where the fast compression applies, else a decode launch and a compression
// launch (kernels in seed_decode_fused.cuh, one translation unit per factor type).
#include "seed_decode_fused.cuh"

namespace seed {

bool decode_compress_fused_supported(const seed_dims& d) {
  return d.R + d.W - 1 <= 32 && compress_fast_supported(d);
}

int launch_decode_compress(const seed_dims& d, const seed_state& s, int layer, const float* q, const float* k,
                           const float* v, const float* alpha, const float* beta, float* o, float* sigma_out,
                           uint32_t* status, cudaStream_t st) {
  if (!decode_compress_fused_supported(d)) {
    const int rc = launch_decode_step(d, s, layer, q, k, v, alpha, beta, o, status, st);
    return rc != SEED_OK ? rc : launch_compress(d, s, layer, sigma_out, status, st);
  }
  DecodeParams p{q, k, v, alpha, beta, o, s.a, s.U, s.V, s.scale, s.ncols, s.vbar, status,
                 d.batch, d.layers, d.heads, layer, d.R, d.W, scale_len(d)};
  FastParams fp{s.U, s.V, s.scale, s.ncols, sigma_out, status, d.batch, d.layers, d.heads, layer, d.R, d.W,
                scale_len(d)};
  int rc = SEED_ERR_INVALID_ARG;
  switch (d.factors) {
    case SEED_FACTORS_F32: rc = launch_fused_f32(d, p, fp, st); break;
    case SEED_FACTORS_F16: rc = launch_fused_f16(d, p, fp, st); break;
    case SEED_FACTORS_BF16: rc = launch_fused_bf16(d, p, fp, st); break;
  }
  return rc != SEED_OK ? rc : launch_compress_householder(d, s, layer, sigma_out, status, st);
}

}  // namespace seed
