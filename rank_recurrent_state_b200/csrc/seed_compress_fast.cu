// seed_compress_fast.cu -- launch of the fast compression (the algorithm and the
// per-unit device function are in seed_compress_fast.cuh).
#include "seed_compress_fast.cuh"

namespace seed {

// One warp per block and per unit of the scope.  The kernel has no static shared
// memory, so its dynamic shared memory starts the block's window, which is
// allocated without alignment slack (more blocks per SM); a block that finds it
// off a 1 KB boundary leaves its unit to the Householder kernel (counted with the
// units the fast path declines) rather than misplace the swizzled buffers.
template <int FORM, int DK, int DV, int MP, typename TS>
__global__ void __launch_bounds__(32)
    compress_fast_kernel(const FastParams p, const __grid_constant__ CUtensorMap tmU,
                         const __grid_constant__ CUtensorMap tmV) {
  using Lay = FastLayout<FORM, DK, DV, MP>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  if (smem_addr(smem_raw) & 1023u) {
    if (threadIdx.x == 0) {
      const int per = p.layer < 0 ? p.L * p.H : p.H;
      const int b = blockIdx.x / per, rest = blockIdx.x - b * per;
      const long long unit = p.layer < 0 ? (long long)blockIdx.x : ((long long)b * p.L + p.layer) * p.H + rest;
      if (p.ncols[unit] == p.R + p.W) atomicAdd(p.status + 6, 1u);
    }
    return;
  }
  float* sA = reinterpret_cast<float*>(smem_raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem_raw + Lay::BAR_OFF);
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  __syncwarp();
  uint32_t uses[2] = {0u, 0u};
  compress_fast_unit<FORM, DK, DV, MP, TS>(p, tmU, tmV, blockIdx.x, sA, bar, uses);
}

// A factor array [units][m][D] as a 3-D float tensor {D, m, units}; boxes of 32 rows
// of MP columns of one unit, 128-byte swizzle, zero fill outside (columns >= m).
bool make_panel_map(CUtensorMap* tm, const float* base, int D, int m, long long units, int MP) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)m, (cuuint64_t)units};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)m * D * 4};
  const cuuint32_t box[3] = {32, (cuuint32_t)MP, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int FORM, int DK, int DV, int MP, typename TS>
static int launch_fast_t(const FastParams& p, int blocks, cudaStream_t st) {
  using Lay = FastLayout<FORM, DK, DV, MP>;
  auto kern = compress_fast_kernel<FORM, DK, DV, MP, TS>;
  static LaunchCache cache;
  int dev = 0;
  if (const int rc = cache.prepare(reinterpret_cast<const void*>(kern), Lay::bytes, &dev)) return rc;
  const long long units = (long long)p.B * p.L * p.H;
  const int m = p.R + p.W;
  CUtensorMap tmU, tmV;
  memset(&tmU, 0, sizeof(tmU));
  memset(&tmV, 0, sizeof(tmV));
  if (std::is_same<TS, float>::value &&
      (!make_panel_map(&tmU, static_cast<const float*>(p.U), DK, m, units, MP) ||
       !make_panel_map(&tmV, static_cast<const float*>(p.V), DV, m, units, MP)))
    return SEED_ERR_CUDA;
  kern<<<blocks, 32, Lay::bytes, st>>>(p, tmU, tmV);
  return cudaGetLastError() == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
}

template <int FORM, int DK, int DV, typename TS>
static int launch_fast_mt(const FastParams& p, int blocks, cudaStream_t st) {
  const int m = p.R + p.W;
  if (m <= 16) return launch_fast_t<FORM, DK, DV, 16, TS>(p, blocks, st);
  return launch_fast_t<FORM, DK, DV, 32, TS>(p, blocks, st);
}

template <int FORM, int DK, int DV>
static int launch_fast_m(const FastParams& p, int blocks, int factors, cudaStream_t st) {
  switch (factors) {
    case SEED_FACTORS_F32: return launch_fast_mt<FORM, DK, DV, float>(p, blocks, st);
    case SEED_FACTORS_F16: return launch_fast_mt<FORM, DK, DV, __half>(p, blocks, st);
    case SEED_FACTORS_BF16: return launch_fast_mt<FORM, DK, DV, __nv_bfloat16>(p, blocks, st);
  }
  return SEED_ERR_INVALID_ARG;
}

// R <= 16: the R new columns are accumulated in registers in one pass over the
// old ones, so that no output overwrites a column before it was read.
bool compress_fast_supported(const seed_dims& d) {
  const int m = d.R + d.W;
  return m <= 32 && d.R <= kFastMaxR && (d.d_k == 64 || d.d_k == 128) &&
         (d.d_v == 64 || d.d_v == 128);
}

int launch_compress_fast(const seed_dims& d, const seed_state& s, int layer, float* sigma_out,
                         uint32_t* status, cudaStream_t st) {
  FastParams p{s.U, s.V, s.scale, s.ncols, sigma_out, status,
               d.batch, d.layers, d.heads, layer, d.R, d.W, scale_len(d)};
  const int blocks = d.batch * d.heads * (layer < 0 ? d.layers : 1);
#define SEED_FAST_DIMS(FORM)                                                                       \
  do {                                                                                             \
    if (d.d_k == 128 && d.d_v == 128) return launch_fast_m<FORM, 128, 128>(p, blocks, d.factors, st);          \
    if (d.d_k == 128 && d.d_v == 64) return launch_fast_m<FORM, 128, 64>(p, blocks, d.factors, st);            \
    if (d.d_k == 64 && d.d_v == 128) return launch_fast_m<FORM, 64, 128>(p, blocks, d.factors, st);            \
    if (d.d_k == 64 && d.d_v == 64) return launch_fast_m<FORM, 64, 64>(p, blocks, d.factors, st);              \
    return SEED_ERR_SHAPE;                                                                         \
  } while (0)
  switch (d.form) {
    case SEED_GDN: SEED_FAST_DIMS(SEED_GDN);
    case SEED_KDA: SEED_FAST_DIMS(SEED_KDA);
    case SEED_MAMBA2: SEED_FAST_DIMS(SEED_MAMBA2);
  }
#undef SEED_FAST_DIMS
  return SEED_ERR_INVALID_ARG;
}

}  // namespace seed
