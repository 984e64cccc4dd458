// seed_compress_wide.cu -- the wide compression entry, 32 < R + W <= 64 (the kernel
// and the per-unit device function are in seed_compress_wide.cuh, instantiated in one
// translation unit per factor type).
#include "seed_compress_wide.cuh"

namespace seed {

bool compress_wide_supported(const seed_dims& d) {
  const int m = d.R + d.W;
  return m > 32 && m <= kWideMP && d.R <= kWideMaxR && (d.d_k == 64 || d.d_k == 128) &&
         (d.d_v == 64 || d.d_v == 128);
}

int launch_compress_wide(const seed_dims& d, const seed_state& s, int layer, float* sigma_out,
                         uint32_t* status, cudaStream_t st) {
  FastParams p{s.U, s.V, s.scale, s.ncols, sigma_out, status,
               d.batch, d.layers, d.heads, layer, d.R, d.W, scale_len(d)};
  const int blocks = d.batch * d.heads * (layer < 0 ? d.layers : 1);
  switch (d.factors) {
    case SEED_FACTORS_F32: return launch_wide_f32(d, p, blocks, st);
    case SEED_FACTORS_F16: return launch_wide_f16(d, p, blocks, st);
    case SEED_FACTORS_BF16: return launch_wide_bf16(d, p, blocks, st);
  }
  return SEED_ERR_INVALID_ARG;
}

}  // namespace seed
