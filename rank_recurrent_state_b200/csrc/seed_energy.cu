// seed_energy.cu -- energies of the stored states: the sink's share and the content.
//
// "Shallow Encoding Emits Deep Memories", SEED figures & tables (thelatestinai.com),
// Figure 3 (f)-(g) and Figure 12 (f): the state S = a vbar^T + U V^T splits into the
// sink a vbar^T and the content C = U V^T, and the pages report the sink's share
// of ||S||_F^2, the two Frobenius norms, and the share of the content energy beyond
// rank R.  Per unit this kernel returns
//     ||a vbar^T||_F^2 = (a^T a)(vbar^T vbar)
//     ||U V^T||_F^2    = sum_ij (U^T U)_ij (V^T V)_ij          (true U, scales applied)
//     2 <a vbar^T, U V^T>_F = 2 sum_j (a^T u_j)(v_j^T vbar)
//     ||S||_F^2        = the sum of the three
// (the cross term is zero up to rounding when V^T vbar = 0, which every update of
// the library keeps).  With the kept singular values that the conversion and the
// compression return, the content energy beyond rank R follows on the host.  One
// block per unit; the true columns are staged in shared memory (rows padded by one
// float so that the Gram loops read without bank conflicts).
#include "seed_common.cuh"
#include "seed_launch.h"

namespace seed {

struct EnergyParams {
  const float* a;
  const void* U;   // element type: the kernel's factor type
  const void* V;
  const float* scale;
  const int32_t* ncols;
  const float* vbar;
  const int32_t* units;
  float* out;
  uint32_t* status;
  int B, L, H, layer, R, W, form, slen, factors;
};

constexpr int kEnergyThreads = 128;

template <int NT>
SEED_DEV float block_sum(float v, float* red) {
  v = group_sum<32>(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();   // red may still be read by a previous call
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) t += red[w];
  return t;
}

template <int DK, int DV, typename TS>
__global__ void __launch_bounds__(kEnergyThreads) energy_kernel(const EnergyParams p) {
  constexpr int NT = kEnergyThreads, LU = DK + 1, LV = DV + 1;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const int m = p.R + p.W;
  float* sU = reinterpret_cast<float*>(smem_raw);   // m x LU, true columns
  float* sV = sU + m * LU;                           // m x LV
  float* s_a = sV + m * LV;
  float* s_vb = s_a + DK;
  __shared__ float red[NT / 32];
  const int per = p.layer < 0 ? p.L * p.H : p.H;
  const int scope = p.units ? p.units[blockIdx.x] : (int)blockIdx.x;
  if (scope < 0 || scope >= p.B * per) {   // the unit list lives on the device: check it here
    if (threadIdx.x == 0) raise_flag(p.status, SEED_FLAG_BADINDEX);
    return;
  }
  const int b = scope / per, rest = scope - b * per;
  const int l = p.layer < 0 ? rest / p.H : p.layer;
  const int h = p.layer < 0 ? rest - (rest / p.H) * p.H : rest;
  const long long unit = ((long long)b * p.L + l) * p.H + h;
  const bool kda = p.form == SEED_KDA;
  int c = p.ncols[unit];
  if (c < 0 || c > m) {
    if (threadIdx.x == 0) raise_flag(p.status, SEED_FLAG_BADCOLS);
    c = 0;
  }
  for (int idx = threadIdx.x; idx < c * DK; idx += NT) {
    const int j = idx / DK, i = idx - j * DK;
    const float sc = kda ? p.scale[unit * DK + i] : p.scale[unit * p.slen + j];
    sU[j * LU + i] = sc * fac_to_f(static_cast<const TS*>(p.U)[unit * (long long)m * DK + idx]);
  }
  for (int idx = threadIdx.x; idx < c * DV; idx += NT) {
    const int j = idx / DV, i = idx - j * DV;
    sV[j * LV + i] = fac_to_f(static_cast<const TS*>(p.V)[unit * (long long)m * DV + idx]);
  }
  for (int i = threadIdx.x; i < DK; i += NT) s_a[i] = p.a[unit * DK + i];
  for (int i = threadIdx.x; i < DV; i += NT) s_vb[i] = p.vbar[((long long)l * p.H + h) * DV + i];
  __syncthreads();

  // content: sum over column pairs i <= j of (u_i . u_j)(v_i . v_j), off-diagonal twice
  float content = 0.f;
  const int pairs = c * (c + 1) / 2;
  for (int t = threadIdx.x; t < pairs; t += NT) {
    int j = (int)((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);   // row of the upper triangle
    while ((j + 1) * (j + 2) / 2 <= t) ++j;
    while (j * (j + 1) / 2 > t) --j;
    const int i = t - j * (j + 1) / 2;   // i <= j
    float gu = 0.f, gv = 0.f;
    for (int r = 0; r < DK; ++r) gu = fmaf(sU[i * LU + r], sU[j * LU + r], gu);
    for (int r = 0; r < DV; ++r) gv = fmaf(sV[i * LV + r], sV[j * LV + r], gv);
    content = fmaf(i == j ? 1.f : 2.f, gu * gv, content);
  }
  // cross: sum_j (a . u_j)(v_j . vbar)
  float cross = 0.f;
  for (int j = threadIdx.x; j < c; j += NT) {
    float za = 0.f, wv = 0.f;
    for (int r = 0; r < DK; ++r) za = fmaf(s_a[r], sU[j * LU + r], za);
    for (int r = 0; r < DV; ++r) wv = fmaf(sV[j * LV + r], s_vb[r], wv);
    cross = fmaf(za, wv, cross);
  }
  float aa = 0.f, vv = 0.f;
  for (int i = threadIdx.x; i < DK; i += NT) aa = fmaf(s_a[i], s_a[i], aa);
  for (int i = threadIdx.x; i < DV; i += NT) vv = fmaf(s_vb[i], s_vb[i], vv);
  content = block_sum<NT>(content, red);
  cross = 2.f * block_sum<NT>(cross, red);
  aa = block_sum<NT>(aa, red);
  vv = block_sum<NT>(vv, red);
  if (threadIdx.x == 0) {
    const float sink = aa * vv;
    float* o = p.out + (long long)blockIdx.x * 4;
    o[0] = sink;
    o[1] = content;
    o[2] = cross;
    o[3] = sink + content + cross;
    if (!(isfinite(sink) && isfinite(content) && isfinite(cross))) raise_flag(p.status, SEED_FLAG_NONFINITE);
  }
}

template <int DK, int DV, typename TS>
static int launch_energy_tt(const EnergyParams& p, int blocks, cudaStream_t st) {
  const size_t smem = ((size_t)(p.R + p.W) * (DK + 1 + DV + 1) + DK + DV) * sizeof(float);
  auto kern = energy_kernel<DK, DV, TS>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SEED_ERR_CUDA;
  kern<<<blocks, kEnergyThreads, smem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
}

template <int DK, int DV>
static int launch_energy_t(const EnergyParams& p, int blocks, cudaStream_t st) {
  switch (p.factors) {
    case SEED_FACTORS_F32: return launch_energy_tt<DK, DV, float>(p, blocks, st);
    case SEED_FACTORS_F16: return launch_energy_tt<DK, DV, __half>(p, blocks, st);
    case SEED_FACTORS_BF16: return launch_energy_tt<DK, DV, __nv_bfloat16>(p, blocks, st);
  }
  return SEED_ERR_INVALID_ARG;
}

int launch_state_energy(const seed_dims& d, const seed_state& s, int layer, const int32_t* units,
                        int n_units, float* out, uint32_t* status, cudaStream_t st) {
  EnergyParams p{s.a, s.U, s.V, s.scale, s.ncols, s.vbar, units, out, status,
                 d.batch, d.layers, d.heads, layer, d.R, d.W, d.form, scale_len(d), d.factors};
  if (d.d_k == 16 && d.d_v == 16) return launch_energy_t<16, 16>(p, n_units, st);
  if (d.d_k == 32 && d.d_v == 32) return launch_energy_t<32, 32>(p, n_units, st);
  if (d.d_k == 64 && d.d_v == 64) return launch_energy_t<64, 64>(p, n_units, st);
  if (d.d_k == 128 && d.d_v == 128) return launch_energy_t<128, 128>(p, n_units, st);
  if (d.d_k == 128 && d.d_v == 64) return launch_energy_t<128, 64>(p, n_units, st);
  if (d.d_k == 64 && d.d_v == 128) return launch_energy_t<64, 128>(p, n_units, st);
  return SEED_ERR_SHAPE;
}

}  // namespace seed
