// seed_decode_fused_bf16.cu -- the fused decode-and-compress kernels for __nv_bfloat16 factors.
#include "seed_decode_fused.cuh"

namespace seed {

int launch_fused_bf16(const seed_dims& d, const DecodeParams& p, const FastParams& fp, cudaStream_t st) {
  return launch_fused_typed<__nv_bfloat16>(d, p, fp, st);
}

}  // namespace seed
