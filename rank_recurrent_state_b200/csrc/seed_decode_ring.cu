// seed_decode_ring.cu -- launch of the one-warp-per-unit decode step with a ring of
// column chunks (the kernel body is in seed_decode_ring.cuh).
#include "seed_decode_ring.cuh"

namespace seed {

// Slots per warp: about 16 KB of chunks (at least 3, at most 8), so that 13 to 14
// warps share an SM.
constexpr int kRingBytes = 16384;   // shared memory of one warp's ring

template <int DK, int DV, typename TS>
constexpr int ring_slots() {
  constexpr int slot_bytes = kRingChunk * (DK > DV ? DK : DV) * (int)sizeof(TS);
  constexpr int n = kRingBytes / slot_bytes;
  return n < 3 ? 3 : (n > 8 ? 8 : n);
}

template <int FORM, int DK, int DV, int MAXC, typename TS>
__global__ void __launch_bounds__(32) decode_ring_kernel(const DecodeParams p) {
  decode_ring_run<FORM, DK, DV, MAXC, ring_slots<DK, DV, TS>(), TS>(p);
}

template <int FORM, int DK, int DV, int MAXC, typename TS>
static int launch_ring_t(const DecodeParams& p, cudaStream_t st) {
  constexpr int NSLOT = ring_slots<DK, DV, TS>();
  auto kern = decode_ring_kernel<FORM, DK, DV, MAXC, TS>;
  const size_t smem = (size_t)NSLOT * kRingChunk * (DK > DV ? DK : DV) * sizeof(TS) + 2 * MAXC * sizeof(float);
  static LaunchCache cache;
  static std::atomic<int> grid_per_sm[kMaxDev];
  if (p.R + p.W - 1 > MAXC) return SEED_ERR_CUDA;
  int dev = 0;
  if (const int rc = cache.prepare(reinterpret_cast<const void*>(kern), smem, &dev)) return rc;
  int per_sm = grid_per_sm[dev].load(std::memory_order_relaxed);
  if (per_sm == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 32, smem) != cudaSuccess) return SEED_ERR_CUDA;
    per_sm = n > 0 ? n : 1;
    grid_per_sm[dev].store(per_sm, std::memory_order_relaxed);
  }
  const int units = p.B * p.H;
  const int grid = balanced_grid(units, per_sm * cache.sm_count[dev].load(std::memory_order_relaxed));
  if (!p.overlap) {
    kern<<<grid, 32, smem, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
  }
  // programmatic stream serialization: the launch may start as the previous kernel on
  // the stream retires its blocks; the kernel waits for it (griddep_wait) before it
  // reads the step's inputs
  cudaLaunchConfig_t cfg = {};
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
static int launch_ring_maxc(const DecodeParams& p, cudaStream_t st) {
  const int maxc = p.R + p.W - 1;
  if (maxc <= 8) return launch_ring_t<FORM, DK, DV, 8, TS>(p, st);
  if (maxc <= 16) return launch_ring_t<FORM, DK, DV, 16, TS>(p, st);
  if (maxc <= 32) return launch_ring_t<FORM, DK, DV, 32, TS>(p, st);
  return launch_ring_t<FORM, DK, DV, 64, TS>(p, st);
}

template <int FORM, int DK, int DV>
static int launch_ring_dims(const DecodeParams& p, int factors, cudaStream_t st) {
  switch (factors) {
    case SEED_FACTORS_F32: return launch_ring_maxc<FORM, DK, DV, float>(p, st);
    case SEED_FACTORS_F16: return launch_ring_maxc<FORM, DK, DV, __half>(p, st);
    case SEED_FACTORS_BF16: return launch_ring_maxc<FORM, DK, DV, __nv_bfloat16>(p, st);
  }
  return SEED_ERR_INVALID_ARG;
}

int launch_decode_ring(const DecodeParams& p, int form, int dk, int dv, int factors, cudaStream_t st) {
#define SEED_RING_DIMS(FORM)                                                              \
  do {                                                                                    \
    if (dk == 16 && dv == 16) return launch_ring_dims<FORM, 16, 16>(p, factors, st);      \
    if (dk == 32 && dv == 32) return launch_ring_dims<FORM, 32, 32>(p, factors, st);      \
    if (dk == 64 && dv == 64) return launch_ring_dims<FORM, 64, 64>(p, factors, st);      \
    if (dk == 128 && dv == 128) return launch_ring_dims<FORM, 128, 128>(p, factors, st);  \
    if (dk == 128 && dv == 64) return launch_ring_dims<FORM, 128, 64>(p, factors, st);    \
    if (dk == 64 && dv == 128) return launch_ring_dims<FORM, 64, 128>(p, factors, st);    \
    return SEED_ERR_SHAPE;                                                                \
  } while (0)
  switch (form) {
    case SEED_GDN: SEED_RING_DIMS(SEED_GDN);
    case SEED_KDA: SEED_RING_DIMS(SEED_KDA);
    case SEED_MAMBA2: SEED_RING_DIMS(SEED_MAMBA2);
  }
#undef SEED_RING_DIMS
  return SEED_ERR_INVALID_ARG;
}

}  // namespace seed
