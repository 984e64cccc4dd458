// seed_decode_fused_f16.cu -- the fused decode-and-compress kernels for __half factors.
#include "seed_decode_fused.cuh"

namespace seed {

int launch_fused_f16(const seed_dims& d, const DecodeParams& p, const FastParams& fp, cudaStream_t st) {
  return launch_fused_typed<__half>(d, p, fp, st);
}

}  // namespace seed
