// seed_compress_wide_bf16.cu -- the wide compression kernels for __nv_bfloat16 factors.
#include "seed_compress_wide.cuh"

namespace seed {

int launch_wide_bf16(const seed_dims& d, const FastParams& p, int blocks, cudaStream_t st) {
  return launch_wide_typed<__nv_bfloat16>(d, p, blocks, st);
}

}  // namespace seed
