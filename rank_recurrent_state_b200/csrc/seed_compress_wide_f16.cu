// seed_compress_wide_f16.cu -- the wide compression kernels for __half factors.
#include "seed_compress_wide.cuh"

namespace seed {

int launch_wide_f16(const seed_dims& d, const FastParams& p, int blocks, cudaStream_t st) {
  return launch_wide_typed<__half>(d, p, blocks, st);
}

}  // namespace seed
