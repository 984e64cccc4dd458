// seed_compress_wide_f32.cu -- the wide compression kernels for float factors.
#include "seed_compress_wide.cuh"

namespace seed {

int launch_wide_f32(const seed_dims& d, const FastParams& p, int blocks, cudaStream_t st) {
  return launch_wide_typed<float>(d, p, blocks, st);
}

}  // namespace seed
