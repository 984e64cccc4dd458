// seed_spectrum.cu -- singular spectra and the top output direction of stored states.
//
// "Shallow Encoding Emits Deep Memories", SEED figures & tables (thelatestinai.com):
// Figure 3 (e), the singular spectra of the state S = a vbar^T + U V^T and of the
// content C = U V^T, divided by the head's top singular value; Figure 3 (h), |cos|
// between the head's top output direction v* and vbar; Figure 13 (a), the energy share
// of the state's i-th singular direction; Figure 13 (d), the rank that holds 90% and
// 99% of the content's energy.  Per listed unit, one block of 256 threads forms S
// explicitly (d_k x d_v, from the stored factors with their scales) in shared memory
// and runs the one-sided Jacobi SVD of seed_common.cuh over its shorter side, the
// right rotations accumulated: then v*, the right singular vector of the largest
// singular value (the read-out o = S^T q lies in the span of the right singular
// vectors), is the rotation's column (over the columns of S) or the normalised
// rotated column (over the columns of S^T).  The content C is formed and
// decomposed the same way.  A diagnostic: not on the decode path, not timed.
#include "seed_common.cuh"
#include "seed_launch.h"

namespace seed {

struct SpectrumParams {
  const float* a;
  const void* U;   // element type: the kernel's factor type
  const void* V;
  const float* scale;
  const int32_t* ncols;
  const float* vbar;
  const int32_t* units;
  float* sigma_state;     // [n][R + W + 1]
  float* sigma_content;   // [n][R + W + 1]
  float* cos_top;         // [n]
  int32_t* ranks;         // [n][2]
  uint32_t* status;
  int B, L, H, layer, R, W, form, slen;
};

constexpr int kSpectrumThreads = 256;

// sC <- the explicit matrix (with_sink: S, else C) of the unit, stored as NC columns of
// length NR (over the columns of S when d_k >= d_v, else over the columns of S^T).
template <int DK, int DV, typename TS>
SEED_DEV void form_dense(const SpectrumParams& p, long long unit, int l, int h, int c, bool with_sink,
                         float* sC, int LDC) {
  constexpr bool COLS = DK >= DV;
  const int m = p.R + p.W;
  const bool kda = p.form == SEED_KDA;
  const TS* Ug = static_cast<const TS*>(p.U) + unit * (long long)m * DK;
  const TS* Vg = static_cast<const TS*>(p.V) + unit * (long long)m * DV;
  const float* vb = p.vbar + ((long long)l * p.H + h) * DV;
  for (int idx = threadIdx.x; idx < DK * DV; idx += kSpectrumThreads) {
    const int j = idx / DK, i = idx - j * DK;   // consecutive threads: consecutive rows i
    float s = with_sink ? p.a[unit * DK + i] * vb[j] : 0.f;
    const float pi = kda ? p.scale[unit * DK + i] : 1.f;
    for (int r = 0; r < c; ++r) {
      const float gr = kda ? 1.f : p.scale[unit * p.slen + r];
      s = fmaf(pi * gr * fac_to_f(Ug[(long long)r * DK + i]), fac_to_f(Vg[(long long)r * DV + j]), s);
    }
    if (COLS) sC[j * LDC + i] = s;   // column j of S
    else sC[i * LDC + j] = s;        // column i of S^T
  }
}

// Singular values of the NC rotated columns, descending, into out[0 .. n_out-1]
// (zeros past NC); returns the index of the largest column through top.
template <int NC, int NR>
SEED_DEV void sorted_norms(const float* sC, int LDC, float* nrm, float* out, int n_out, int* top) {
  for (int j = threadIdx.x; j < NC; j += kSpectrumThreads) {
    float s2 = 0.f;
    for (int i = 0; i < NR; ++i) s2 = fmaf(sC[j * LDC + i], sC[j * LDC + i], s2);
    nrm[j] = sqrtf(s2);
  }
  __syncthreads();
  for (int j = threadIdx.x; j < NC; j += kSpectrumThreads) {
    const float s = nrm[j];
    int rank = 0;
    for (int k = 0; k < NC; ++k) rank += (nrm[k] > s) || (nrm[k] == s && k < j);
    if (rank < n_out) out[rank] = s;
    if (rank == 0) *top = j;
  }
  for (int r = NC + threadIdx.x; r < n_out; r += kSpectrumThreads) out[r] = 0.f;
  __syncthreads();
}

template <int DK, int DV, typename TS>
__global__ void __launch_bounds__(kSpectrumThreads) spectrum_kernel(const SpectrumParams p) {
  constexpr int NT = kSpectrumThreads, NW = NT / 32;
  constexpr bool COLS = DK >= DV;
  constexpr int NC = COLS ? DV : DK;
  constexpr int NR = COLS ? DK : DV;
  constexpr int LDC = NR + 1, LDZ = NC + 1;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  float* sC = reinterpret_cast<float*>(smem_raw);   // NC x LDC
  float* sZ = sC + NC * LDC;                         // NC x LDZ
  float* nrm = sZ + NC * LDZ;                        // NC
  float* red = nrm + NC;                             // NW
  __shared__ int top;
  const int m = p.R + p.W, n_out = m + 1;
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
  int c = p.ncols[unit];
  if (c < 0 || c > m) {
    if (threadIdx.x == 0) raise_flag(p.status, SEED_FLAG_BADCOLS);
    c = 0;
  }
  const float tol = 8.f * sqrtf((float)NR) * 5.9604645e-8f;
  float* sigS = p.sigma_state + (long long)blockIdx.x * n_out;
  float* sigC = p.sigma_content + (long long)blockIdx.x * n_out;
  bool conv = true;

  // the state, with the right rotations for v*
  form_dense<DK, DV, TS>(p, unit, l, h, c, true, sC, LDC);
  __syncthreads();
  conv &= jacobi_svd<NT>(sC, LDC, NR, sZ, LDZ, NC, tol, 60, red, 1e-12f) <= 60;
  sorted_norms<NC, NR>(sC, LDC, nrm, sigS, n_out, &top);
  {
    // v*: COLS -> column `top` of Z; else the rotated column `top` of S^T Z, normalised
    const float* vs = COLS ? sZ + top * LDZ : sC + top * LDC;
    const float* vb = p.vbar + ((long long)l * p.H + h) * DV;
    float d = 0.f, vv = 0.f, bb = 0.f;
    for (int j = threadIdx.x; j < DV; j += NT) {
      d = fmaf(vs[j], vb[j], d);
      vv = fmaf(vs[j], vs[j], vv);
      bb = fmaf(vb[j], vb[j], bb);
    }
    d = group_sum<32>(d);
    vv = group_sum<32>(vv);
    bb = group_sum<32>(bb);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __shared__ float part[3][NW];
    if (lane == 0) {
      part[0][warp] = d;
      part[1][warp] = vv;
      part[2][warp] = bb;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float D = 0.f, VV = 0.f, BB = 0.f;
      for (int w = 0; w < NW; ++w) {
        D += part[0][w];
        VV += part[1][w];
        BB += part[2][w];
      }
      const float den = sqrtf(VV) * sqrtf(BB);
      const float cs = den > 0.f ? fabsf(D) / den : 0.f;
      p.cos_top[blockIdx.x] = cs;
      if (!isfinite(cs)) raise_flag(p.status, SEED_FLAG_NONFINITE);
      if (!(BB > 0.f)) raise_flag(p.status, SEED_FLAG_ZERO_VBAR);
    }
    __syncthreads();
  }

  // the content
  form_dense<DK, DV, TS>(p, unit, l, h, c, false, sC, LDC);
  __syncthreads();
  conv &= jacobi_svd<NT>(sC, LDC, NR, sZ, LDZ, NC, tol, 60, red, 1e-12f) <= 60;
  sorted_norms<NC, NR>(sC, LDC, nrm, sigC, n_out, &top);
  if (threadIdx.x == 0) {
    // ranks holding 90% and 99% of the content's energy: the smallest k whose k
    // largest singular values hold that share (0 for a zero content)
    float tot = 0.f;
    for (int k = NC - 1; k >= 0; --k) tot = fmaf(nrm[k], nrm[k], tot);   // any order: the total
    int k90 = 0, k99 = 0;
    if (tot > 0.f) {
      float cum = 0.f;
      for (int k = 0; k < n_out && k < NC; ++k) {
        cum = fmaf(sigC[k], sigC[k], cum);
        if (k90 == 0 && cum >= 0.9f * tot) k90 = k + 1;
        if (k99 == 0 && cum >= 0.99f * tot) k99 = k + 1;
      }
      if (k90 == 0) k90 = n_out < NC ? n_out : NC;
      if (k99 == 0) k99 = n_out < NC ? n_out : NC;
    }
    p.ranks[2 * (long long)blockIdx.x] = k90;
    p.ranks[2 * (long long)blockIdx.x + 1] = k99;
    if (!conv) raise_flag(p.status, SEED_FLAG_NOCONVERGE);
  }
}

template <int DK, int DV, typename TS>
static int launch_spectrum_tt(const SpectrumParams& p, int blocks, cudaStream_t st) {
  constexpr bool COLS = DK >= DV;
  constexpr int NC = COLS ? DV : DK, NR = COLS ? DK : DV;
  const size_t smem = ((size_t)NC * (NR + 1) + (size_t)NC * (NC + 1) + NC + kSpectrumThreads / 32) * sizeof(float);
  auto kern = spectrum_kernel<DK, DV, TS>;
  static LaunchCache cache;
  int dev = 0;
  if (const int rc = cache.prepare(reinterpret_cast<const void*>(kern), smem, &dev)) return rc;
  kern<<<blocks, kSpectrumThreads, smem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
}

template <int DK, int DV>
static int launch_spectrum_t(const SpectrumParams& p, int blocks, int factors, cudaStream_t st) {
  switch (factors) {
    case SEED_FACTORS_F32: return launch_spectrum_tt<DK, DV, float>(p, blocks, st);
    case SEED_FACTORS_F16: return launch_spectrum_tt<DK, DV, __half>(p, blocks, st);
    case SEED_FACTORS_BF16: return launch_spectrum_tt<DK, DV, __nv_bfloat16>(p, blocks, st);
  }
  return SEED_ERR_INVALID_ARG;
}

int launch_state_spectrum(const seed_dims& d, const seed_state& s, int layer, const int32_t* units, int n_units,
                          float* sigma_state, float* sigma_content, float* cos_top, int32_t* ranks,
                          uint32_t* status, cudaStream_t st) {
  SpectrumParams p{s.a, s.U, s.V, s.scale, s.ncols, s.vbar, units, sigma_state, sigma_content, cos_top, ranks,
                   status, d.batch, d.layers, d.heads, layer, d.R, d.W, d.form, scale_len(d)};
  if (n_units == 0) return SEED_OK;
  if (d.d_k == 16 && d.d_v == 16) return launch_spectrum_t<16, 16>(p, n_units, d.factors, st);
  if (d.d_k == 32 && d.d_v == 32) return launch_spectrum_t<32, 32>(p, n_units, d.factors, st);
  if (d.d_k == 64 && d.d_v == 64) return launch_spectrum_t<64, 64>(p, n_units, d.factors, st);
  if (d.d_k == 128 && d.d_v == 128) return launch_spectrum_t<128, 128>(p, n_units, d.factors, st);
  if (d.d_k == 128 && d.d_v == 64) return launch_spectrum_t<128, 64>(p, n_units, d.factors, st);
  if (d.d_k == 64 && d.d_v == 128) return launch_spectrum_t<64, 128>(p, n_units, d.factors, st);
  return SEED_ERR_SHAPE;
}

}  // namespace seed
