// seed_decode_fused.cuh -- the decode step with the compression fused into it.
//
// "Shallow Encoding Emits Deep Memories", SEED figures & tables (thelatestinai.com),
// Figure 1(b): each decode step appends a column pair and, every W steps, the
// factors are compressed back to rank R.  Here the step that brings a unit to
// R + W columns also compresses it, in the same launch and by the same warp
// (decode_warp_run with FUSE, seed_decode_warp.cuh; the compression is
// compress_fast_unit, seed_compress_fast.cuh): the unit's columns were staged for
// the step a moment before and are read again from L2 rather than HBM, and the
// separate compression launch over all units disappears.  Units the fast
// compression declines keep R + W columns and are compressed by the Householder
// kernel in a second launch over the layer.
#pragma once

#include "seed_decode_warp.cuh"

namespace seed {

// At most 168 registers a thread (12 warps per SM where shared memory allows, as
// the compression wants); the body fits without spills.
template <int FORM, int DK, int DV, int MAXC, typename TS, int MP>
__global__ void __launch_bounds__(32, 12)
    decode_compress_warp_kernel(const DecodeParams p, const FastParams fp, const __grid_constant__ CUtensorMap tmU,
                                const __grid_constant__ CUtensorMap tmV) {
  decode_warp_run<FORM, DK, DV, MAXC, TS, true, MP>(p, &fp, &tmU, &tmV);
}

// Dynamic shared memory: the larger of the decode stage (with the coefficients) and
// the compression's layout (which carries its own 1 KB alignment slack).
template <int FORM, int DK, int DV, int MP, typename TS>
static size_t fused_smem(int maxc) {
  const size_t dec = warp_stage_bytes(maxc, DK, DV, sizeof(TS)) + kCoefFloats * sizeof(float) + 16;
  const size_t cmp = FastLayout<FORM, DK, DV, MP>::bytes_aligned;
  return dec > cmp ? dec : cmp;
}

template <int FORM, int DK, int DV, int MAXC, typename TS, int MP>
static int launch_fused_t(const DecodeParams& p, const FastParams& fp, cudaStream_t st) {
  auto kern = decode_compress_warp_kernel<FORM, DK, DV, MAXC, TS, MP>;
  const int m = p.R + p.W, maxc = m - 1;
  const size_t smem = fused_smem<FORM, DK, DV, MP, TS>(maxc);
  static LaunchCache cache;
  static std::atomic<int> grid_per_sm[kMaxDev][MAXC + 1];
  if (maxc > MAXC) return SEED_ERR_CUDA;
  int dev = 0;
  if (const int rc = cache.prepare(reinterpret_cast<const void*>(kern), fused_smem<FORM, DK, DV, MP, TS>(MAXC), &dev))
    return rc;
  int per_sm = grid_per_sm[dev][maxc].load(std::memory_order_relaxed);
  if (per_sm == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 32, smem) != cudaSuccess) return SEED_ERR_CUDA;
    per_sm = n > 0 ? n : 1;
    grid_per_sm[dev][maxc].store(per_sm, std::memory_order_relaxed);
  }
  CUtensorMap tmU, tmV;
  memset(&tmU, 0, sizeof(tmU));
  memset(&tmV, 0, sizeof(tmV));
  const long long all_units = (long long)p.B * p.L * p.H;
  if (std::is_same<TS, float>::value &&
      (!make_panel_map(&tmU, static_cast<const float*>(p.U), DK, m, all_units, MP) ||
       !make_panel_map(&tmV, static_cast<const float*>(p.V), DV, m, all_units, MP)))
    return SEED_ERR_CUDA;
  const int units = p.B * p.H;
  const int grid = balanced_grid(units, per_sm * cache.sm_count[dev].load(std::memory_order_relaxed));
  kern<<<grid, 32, smem, st>>>(p, fp, tmU, tmV);
  return cudaGetLastError() == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
}

// (stage bucket, compression tile) pairs: MP = 16 needs R + W <= 16.
template <int FORM, int DK, int DV, typename TS>
static int launch_fused_ts(const DecodeParams& p, const FastParams& fp, cudaStream_t st) {
  const int m = p.R + p.W, maxc = m - 1;
  if (maxc <= 8) return launch_fused_t<FORM, DK, DV, 8, TS, 16>(p, fp, st);
  if (maxc <= 16) {
    if (m <= 16) return launch_fused_t<FORM, DK, DV, 16, TS, 16>(p, fp, st);
    return launch_fused_t<FORM, DK, DV, 16, TS, 32>(p, fp, st);
  }
  return launch_fused_t<FORM, DK, DV, 32, TS, 32>(p, fp, st);
}

template <int FORM, typename TS>
static int launch_fused_form(const seed_dims& d, const DecodeParams& p, const FastParams& fp, cudaStream_t st) {
  if (d.d_k == 128 && d.d_v == 128) return launch_fused_ts<FORM, 128, 128, TS>(p, fp, st);
  if (d.d_k == 128 && d.d_v == 64) return launch_fused_ts<FORM, 128, 64, TS>(p, fp, st);
  if (d.d_k == 64 && d.d_v == 128) return launch_fused_ts<FORM, 64, 128, TS>(p, fp, st);
  if (d.d_k == 64 && d.d_v == 64) return launch_fused_ts<FORM, 64, 64, TS>(p, fp, st);
  return SEED_ERR_SHAPE;
}

// The fused launch for factor type TS (one translation unit per type).
template <typename TS>
int launch_fused_typed(const seed_dims& d, const DecodeParams& p, const FastParams& fp, cudaStream_t st) {
  switch (d.form) {
    case SEED_GDN: return launch_fused_form<SEED_GDN, TS>(d, p, fp, st);
    case SEED_KDA: return launch_fused_form<SEED_KDA, TS>(d, p, fp, st);
    case SEED_MAMBA2: return launch_fused_form<SEED_MAMBA2, TS>(d, p, fp, st);
  }
  return SEED_ERR_INVALID_ARG;
}

int launch_fused_f32(const seed_dims& d, const DecodeParams& p, const FastParams& fp, cudaStream_t st);
int launch_fused_f16(const seed_dims& d, const DecodeParams& p, const FastParams& fp, cudaStream_t st);
int launch_fused_bf16(const seed_dims& d, const DecodeParams& p, const FastParams& fp, cudaStream_t st);

}  // namespace seed
