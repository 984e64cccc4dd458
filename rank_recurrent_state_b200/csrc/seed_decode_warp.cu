// seed_decode_warp.cu -- launch of the one-warp-per-unit decode step with a whole-unit
// stage (the kernel body is in seed_decode_warp.cuh), for 16-bit factors.
//
// With 16-bit factors a unit's stored columns fit one stage of half the float32 size,
// and one bulk copy per factor and unit costs fewer instructions per byte than the
// ring's 8-column chunks (seed_decode_ring.cuh), whose per-chunk waits and refills
// bound the 16-bit step; float32 factors stream through the ring.
#include "seed_decode_warp.cuh"

namespace seed {

template <int FORM, int DK, int DV, int MAXC, typename TS>
__global__ void __launch_bounds__(32) decode_warp_kernel(const DecodeParams p) {
  decode_warp_run<FORM, DK, DV, MAXC, TS, false, 16>(p, nullptr, nullptr, nullptr);
}

template <int FORM, int DK, int DV, int MAXC, typename TS>
static int launch_warp_t(const DecodeParams& p, cudaStream_t st) {
  auto kern = decode_warp_kernel<FORM, DK, DV, MAXC, TS>;
  const int maxc = p.R + p.W - 1;
  if (maxc > MAXC) return SEED_ERR_CUDA;
  const size_t smem = warp_stage_bytes(maxc, DK, DV, sizeof(TS)) + coef_floats(MAXC) * sizeof(float) + 16;
  const size_t smax = warp_stage_bytes(MAXC, DK, DV, sizeof(TS)) + coef_floats(MAXC) * sizeof(float) + 16;
  // per device: the shared-memory opt-in for the largest stage, and the resident
  // blocks per SM for each stage size
  static LaunchCache cache;
  static std::atomic<int> grid_per_sm[kMaxDev][MAXC + 1];
  int dev = 0;
  if (const int rc = cache.prepare(reinterpret_cast<const void*>(kern), smax, &dev)) return rc;
  int per_sm = grid_per_sm[dev][maxc].load(std::memory_order_relaxed);
  if (per_sm == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 32, smem) != cudaSuccess) return SEED_ERR_CUDA;
    per_sm = n > 0 ? n : 1;
    grid_per_sm[dev][maxc].store(per_sm, std::memory_order_relaxed);
  }
  const int units = p.B * p.H;
  const int grid = balanced_grid(units, per_sm * cache.sm_count[dev].load(std::memory_order_relaxed));
  if (!p.overlap) {
    kern<<<grid, 32, smem, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg = {};   // programmatic stream serialization, as the ring kernel
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p) == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
}

template <int FORM, int DK, int DV, typename TS>
static int launch_warp_maxc(const DecodeParams& p, cudaStream_t st) {
  const int maxc = p.R + p.W - 1;
  if (maxc <= 8) return launch_warp_t<FORM, DK, DV, 8, TS>(p, st);
  if (maxc <= 16) return launch_warp_t<FORM, DK, DV, 16, TS>(p, st);
  if (maxc <= 32) return launch_warp_t<FORM, DK, DV, 32, TS>(p, st);
  return launch_warp_t<FORM, DK, DV, 64, TS>(p, st);
}

template <int FORM, int DK, int DV>
static int launch_warp_dims(const DecodeParams& p, int factors, cudaStream_t st) {
  switch (factors) {
    case SEED_FACTORS_F16: return launch_warp_maxc<FORM, DK, DV, __half>(p, st);
    case SEED_FACTORS_BF16: return launch_warp_maxc<FORM, DK, DV, __nv_bfloat16>(p, st);
  }
  return SEED_ERR_INVALID_ARG;
}

int launch_decode_warp16(const DecodeParams& p, int form, int dk, int dv, int factors, cudaStream_t st) {
#define SEED_WARP_DIMS(FORM)                                                              \
  do {                                                                                    \
    if (dk == 16 && dv == 16) return launch_warp_dims<FORM, 16, 16>(p, factors, st);      \
    if (dk == 32 && dv == 32) return launch_warp_dims<FORM, 32, 32>(p, factors, st);      \
    if (dk == 64 && dv == 64) return launch_warp_dims<FORM, 64, 64>(p, factors, st);      \
    if (dk == 128 && dv == 128) return launch_warp_dims<FORM, 128, 128>(p, factors, st);  \
    if (dk == 128 && dv == 64) return launch_warp_dims<FORM, 128, 64>(p, factors, st);    \
    if (dk == 64 && dv == 128) return launch_warp_dims<FORM, 64, 128>(p, factors, st);    \
    return SEED_ERR_SHAPE;                                                                \
  } while (0)
  switch (form) {
    case SEED_GDN: SEED_WARP_DIMS(SEED_GDN);
    case SEED_KDA: SEED_WARP_DIMS(SEED_KDA);
    case SEED_MAMBA2: SEED_WARP_DIMS(SEED_MAMBA2);
  }
#undef SEED_WARP_DIMS
  return SEED_ERR_INVALID_ARG;
}

}  // namespace seed
