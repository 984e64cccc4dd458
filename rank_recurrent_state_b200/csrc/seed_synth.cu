// seed_synth.cu -- seeded synthetic inputs and dense prefill states on the device.
//
// Not part of the method.  Values are addressed by Philox4x32-10 counters
// (block, field | phase << 8, t, unit) under the key (seed, workload); each
// transform is evaluated in float64 with explicitly rounded operations (no
// contraction into fused multiply-adds) and rounded to float32 once, so that an
// independent host implementation of the same definitions reproduces the values.
#include "seed_common.cuh"
#include "seed_launch.h"

namespace seed {

enum : uint32_t { F_Q = 0, F_K = 1, F_V = 2, F_ALPHA = 3, F_BETA = 4, F_VBAR_DIR = 8,
                  F_VBAR_NORM = 9, F_A = 10 };

SEED_DEV uint4 philox_words(const seed_synth_key& key, uint32_t unit, uint32_t t, uint32_t field,
                            uint32_t phase, uint32_t block) {
  return philox4x32_10(make_uint4(block, field | (phase << 8), t, unit), key.seed, key.workload);
}

SEED_DEV double softplus_d(double x) { return log1p(exp(x)); }
SEED_DEV double sigmoid_d(double x) { return __ddiv_rn(1.0, __dadd_rn(1.0, exp(-x))); }

// Deterministic sum of n doubles in shared memory by one warp (fixed tree order).
SEED_DEV double warp_sum_d(const double* x, int n) {
  const int lane = threadIdx.x & 31;
  double s = 0.0;
  for (int i = lane; i < n; i += 32) s = __dadd_rn(s, __dmul_rn(x[i], x[i]));
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) s = __dadd_rn(s, __shfl_xor_sync(0xffffffffu, s, off));
  return s;
}

// ------------------------------------------------------------------ vbar
__global__ void synth_vbar_kernel(seed_synth_key key, int H, int DV, float* vbar) {
  extern __shared__ double sd[];   // DV (rounded up to 4)
  __shared__ double s_sum;
  const int head = blockIdx.x;   // l * H + h
  const int nb = (DV + 3) / 4;
  for (int blk = threadIdx.x; blk < nb; blk += blockDim.x) {
    double z[4];
    block_normals(philox_words(key, (uint32_t)head, 0, F_VBAR_DIR, SEED_PHASE_PREFILL, blk), z);
    for (int e = 0; e < 4; ++e) sd[4 * blk + e] = z[e];
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const double s = warp_sum_d(sd, DV);
    if (threadIdx.x == 0) s_sum = s;
  }
  __syncthreads();
  double nrm = 1.0;
  if (!key.vbar_unit) {
    double u[4];
    block_uniforms(philox_words(key, (uint32_t)head, 0, F_VBAR_NORM, SEED_PHASE_PREFILL, 0), u);
    nrm = __dadd_rn(1.0, __dmul_rn(3.0, u[0]));
  }
  const double root = sqrt(s_sum);
  for (int i = threadIdx.x; i < DV; i += blockDim.x)
    vbar[(long long)head * DV + i] = __double2float_rn(__dmul_rn(__ddiv_rn(sd[i], root), nrm));
  (void)H;
}

int launch_synth_vbar(const seed_dims& d, const seed_synth_key& key, float* vbar, cudaStream_t st) {
  const int nb = (d.d_v + 3) / 4;
  synth_vbar_kernel<<<d.layers * d.heads, 64, nb * 4 * sizeof(double), st>>>(key, d.heads, d.d_v,
                                                                              vbar);
  return cudaGetLastError() == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
}

// ------------------------------------------------------------------ per-token generation
// Generates the inputs of one unit and token into shared memory, float32:
// k[DK], q[DK] (optional), v[DV], alpha (scalar or [DK]), beta.  Called by all
// threads of the block; `zbuf` holds 2*DK + DV + DK doubles of scratch.
struct TokenSmem {
  double* zk;
  double* zq;
  double* zv;
  double* za;   // KDA alpha uniforms
  double* scal; // [0] beta-field normal, [1] alpha-field normal, [2] |k|^2, [3] |q|^2
  float* k;
  float* q;
  float* v;
  float* alpha;
  float* beta;  // [0] beta / Delta; [1] scalar alpha
};

template <int FORM, int DK, int DV>
SEED_DEV void gen_token(const seed_synth_key& key, uint32_t unit, uint32_t head, uint32_t t,
                        uint32_t phase, bool want_q, const float* vb, double A, TokenSmem s) {
  constexpr int NBK = DK / 4, NBV = DV / 4;
  constexpr bool KDA = FORM == SEED_KDA;
  constexpr bool M2 = FORM == SEED_MAMBA2;
  const int ntask = NBK + (want_q ? NBK : 0) + NBV + 1 + (KDA ? NBK : (M2 ? 0 : 1));
  for (int task = threadIdx.x; task < ntask; task += blockDim.x) {
    int x = task;
    double z[4];
    if (x < NBK) {
      block_normals(philox_words(key, unit, t, F_K, phase, x), z);
      for (int e = 0; e < 4; ++e) s.zk[4 * x + e] = z[e];
      continue;
    }
    x -= NBK;
    if (want_q) {
      if (x < NBK) {
        block_normals(philox_words(key, unit, t, F_Q, phase, x), z);
        for (int e = 0; e < 4; ++e) s.zq[4 * x + e] = z[e];
        continue;
      }
      x -= NBK;
    }
    if (x < NBV) {
      block_normals(philox_words(key, unit, t, F_V, phase, x), z);
      for (int e = 0; e < 4; ++e) s.zv[4 * x + e] = z[e];
      continue;
    }
    x -= NBV;
    if (x == 0) {
      block_normals(philox_words(key, unit, t, F_BETA, phase, 0), z);
      s.scal[0] = z[0];
      continue;
    }
    x -= 1;
    if (KDA) {
      double u[4];
      block_uniforms(philox_words(key, unit, t, F_ALPHA, phase, x), u);
      for (int e = 0; e < 4; ++e) s.za[4 * x + e] = u[e];
    } else {
      block_normals(philox_words(key, unit, t, F_ALPHA, phase, 0), z);
      s.scal[1] = z[0];
    }
  }
  __syncthreads();
  if (!M2) {
    if (threadIdx.x < 32) {
      const double sk = warp_sum_d(s.zk, DK);
      if (threadIdx.x == 0) s.scal[2] = sk;
    }
    if (want_q && threadIdx.x >= 32 && threadIdx.x < 64) {
      const double sq = warp_sum_d(s.zq, DK);
      if (threadIdx.x == 32) s.scal[3] = sq;
    }
  }
  __syncthreads();
  const double scale_m2 = __ddiv_rn(1.0, sqrt((double)DK));
  const double rk = M2 ? 0.0 : sqrt(s.scal[2]);
  const double rq = (M2 || !want_q) ? 0.0 : sqrt(s.scal[3]);
  for (int i = threadIdx.x; i < DK; i += blockDim.x) {
    s.k[i] = __double2float_rn(M2 ? __dmul_rn(s.zk[i], scale_m2) : __ddiv_rn(s.zk[i], rk));
    if (want_q) s.q[i] = __double2float_rn(M2 ? __dmul_rn(s.zq[i], scale_m2) : __ddiv_rn(s.zq[i], rq));
    if (KDA) s.alpha[i] = __double2float_rn(__dadd_rn(0.85, __dmul_rn(0.15, s.za[i])));
  }
  for (int i = threadIdx.x; i < DV; i += blockDim.x) {
    const double vbd = (double)vb[i];
    s.v[i] = __double2float_rn(M2 ? __dadd_rn(vbd, __dmul_rn(0.5, s.zv[i]))
                                  : __dadd_rn(__dmul_rn(3.0, vbd), __dmul_rn(0.3, s.zv[i])));
  }
  if (threadIdx.x == 0) {
    if (M2) {
      const double delta = softplus_d(__dadd_rn(-2.0, __dmul_rn(0.5, s.scal[0])));
      s.beta[0] = __double2float_rn(delta);
      s.beta[1] = __double2float_rn(exp(__dmul_rn(-delta, A)));
    } else {
      s.beta[0] = __double2float_rn(sigmoid_d(s.scal[0]));
      if (!KDA) s.beta[1] = __double2float_rn(exp(-softplus_d(__dadd_rn(-3.0, __dmul_rn(0.5, s.scal[1])))));
    }
  }
  __syncthreads();
  (void)head;
}

SEED_DEV double mamba2_A(const seed_synth_key& key, uint32_t head) {
  double u[4];
  block_uniforms(philox_words(key, head, 0, F_A, SEED_PHASE_PREFILL, 0), u);
  return __dadd_rn(1.0, __dmul_rn(15.0, u[0]));
}

template <int FORM, int DK, int DV>
struct SynthSmem {
  double zk[DK], zq[DK], zv[DV], za[FORM == SEED_KDA ? DK : 4], scal[4];
  float k[DK], q[DK], v[DV], alpha[FORM == SEED_KDA ? DK : 4], beta[2], vb[DV];
  __device__ TokenSmem view() { return TokenSmem{zk, zq, zv, za, scal, k, q, v, alpha, beta}; }
};

template <int FORM, int DK, int DV>
__global__ void synth_token_kernel(seed_synth_key key, int L, int H, int layer, int phase, int t,
                                   const float* vbar, float* q, float* k, float* v, float* alpha,
                                   float* beta) {
  __shared__ SynthSmem<FORM, DK, DV> sm;
  const int bh = blockIdx.x;
  const int b = bh / H, h = bh - b * H;
  const uint32_t head = (uint32_t)(layer * H + h);
  const uint32_t unit = (uint32_t)(((long long)(key.b0 + b) * L + layer) * H + h);
  for (int i = threadIdx.x; i < DV; i += blockDim.x) sm.vb[i] = vbar[(long long)head * DV + i];
  __syncthreads();
  const double A = FORM == SEED_MAMBA2 ? mamba2_A(key, head) : 0.0;
  gen_token<FORM, DK, DV>(key, unit, head, (uint32_t)t, (uint32_t)phase, q != nullptr, sm.vb, A,
                          sm.view());
  for (int i = threadIdx.x; i < DK; i += blockDim.x) {
    k[(long long)bh * DK + i] = sm.k[i];
    if (q) q[(long long)bh * DK + i] = sm.q[i];
    if (FORM == SEED_KDA) alpha[(long long)bh * DK + i] = sm.alpha[i];
  }
  for (int i = threadIdx.x; i < DV; i += blockDim.x) v[(long long)bh * DV + i] = sm.v[i];
  if (threadIdx.x == 0) {
    beta[bh] = sm.beta[0];
    if (FORM != SEED_KDA) alpha[bh] = sm.beta[1];
  }
}

// ------------------------------------------------------------------ dense prefill
// One CTA of max(32, DV) threads per unit; thread j < DV keeps column j of S (DK
// floats) in registers for the whole prefill and applies the form's dense recurrence.
template <int FORM, int DK, int DV>
__global__ void __launch_bounds__(DV < 32 ? 32 : DV) synth_prefill_kernel(seed_synth_key key, int L, int H,
                                                           int layer, int n_tokens,
                                                           const float* vbar, float* S_out) {
  __shared__ SynthSmem<FORM, DK, DV> sm;
  const int per = layer < 0 ? L * H : H;
  const int b = blockIdx.x / per, rest = blockIdx.x - b * per;
  const int l = layer < 0 ? rest / H : layer;
  const int h = layer < 0 ? rest - (rest / H) * H : rest;
  const uint32_t head = (uint32_t)(l * H + h);
  const uint32_t unit = (uint32_t)(((long long)(key.b0 + b) * L + l) * H + h);
  for (int i = threadIdx.x; i < DV; i += blockDim.x) sm.vb[i] = vbar[(long long)head * DV + i];
  __syncthreads();
  const double A = FORM == SEED_MAMBA2 ? mamba2_A(key, head) : 0.0;
  const int j = threadIdx.x < DV ? threadIdx.x : DV - 1;   // extra lanes mirror the last column
  float col[DK];
#pragma unroll
  for (int i = 0; i < DK; ++i) col[i] = 0.f;
  for (int t = 0; t < n_tokens; ++t) {
    gen_token<FORM, DK, DV>(key, unit, head, (uint32_t)t, SEED_PHASE_PREFILL, false, sm.vb, A,
                            sm.view());
    const float be = sm.beta[0];
    const float vj = sm.v[j];
    if (FORM == SEED_MAMBA2) {
      const float al = sm.beta[1];
      const float w = be * vj;
#pragma unroll
      for (int i = 0; i < DK; ++i) col[i] = fmaf(al, col[i], sm.k[i] * w);
    } else if (FORM == SEED_KDA) {
      float ks = 0.f;
#pragma unroll
      for (int i = 0; i < DK; ++i) ks = fmaf(sm.k[i] * sm.alpha[i], col[i], ks);
      const float w = be * (vj - ks);
#pragma unroll
      for (int i = 0; i < DK; ++i) col[i] = fmaf(sm.alpha[i], col[i], sm.k[i] * w);
    } else {
      const float g = sm.beta[1];
      float ks = 0.f;
#pragma unroll
      for (int i = 0; i < DK; ++i) ks = fmaf(sm.k[i], col[i], ks);
      const float w = be * (vj - g * ks);
#pragma unroll
      for (int i = 0; i < DK; ++i) col[i] = fmaf(g, col[i], sm.k[i] * w);
    }
  }
  float* S = S_out + (long long)blockIdx.x * DK * DV;
  if (threadIdx.x < DV) {
#pragma unroll
    for (int i = 0; i < DK; ++i) S[(long long)i * DV + j] = col[i];
  }
}

#define SEED_SYNTH_DIMS(LAUNCH)                       \
  do {                                                \
    if (d.d_k == 16 && d.d_v == 16) { LAUNCH(16, 16) }              \
    else if (d.d_k == 32 && d.d_v == 32) { LAUNCH(32, 32) }         \
    else if (d.d_k == 64 && d.d_v == 64) { LAUNCH(64, 64) }         \
    else if (d.d_k == 128 && d.d_v == 128) { LAUNCH(128, 128) }     \
    else if (d.d_k == 128 && d.d_v == 64) { LAUNCH(128, 64) }       \
    else if (d.d_k == 64 && d.d_v == 128) { LAUNCH(64, 128) }       \
    else return SEED_ERR_SHAPE;                       \
  } while (0)

int launch_synth_token_inputs(const seed_dims& d, const seed_synth_key& key, int phase, int t,
                              int layer, const float* vbar, float* q, float* k, float* v,
                              float* alpha, float* beta, cudaStream_t st) {
  const int blocks = d.batch * d.heads;
#define SEED_TOK(K, V)                                                                      \
  switch (d.form) {                                                                         \
    case SEED_GDN:                                                                          \
      synth_token_kernel<SEED_GDN, K, V><<<blocks, 64, 0, st>>>(key, d.layers, d.heads, layer, \
                                                                phase, t, vbar, q, k, v, alpha, beta); \
      break;                                                                                \
    case SEED_KDA:                                                                          \
      synth_token_kernel<SEED_KDA, K, V><<<blocks, 64, 0, st>>>(key, d.layers, d.heads, layer, \
                                                                phase, t, vbar, q, k, v, alpha, beta); \
      break;                                                                                \
    default:                                                                                \
      synth_token_kernel<SEED_MAMBA2, K, V><<<blocks, 64, 0, st>>>(                         \
          key, d.layers, d.heads, layer, phase, t, vbar, q, k, v, alpha, beta);             \
  }
  SEED_SYNTH_DIMS(SEED_TOK);
#undef SEED_TOK
  return cudaGetLastError() == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
}

int launch_synth_dense_prefill(const seed_dims& d, const seed_synth_key& key, int n_tokens,
                               int layer, const float* vbar, float* S_out, cudaStream_t st) {
  const int blocks = d.batch * d.heads * (layer < 0 ? d.layers : 1);
#define SEED_PRE(K, V)                                                                       \
  switch (d.form) {                                                                          \
    case SEED_GDN:                                                                           \
      synth_prefill_kernel<SEED_GDN, K, V><<<blocks, (V < 32 ? 32 : V), 0, st>>>(key, d.layers, d.heads, layer, \
                                                                 n_tokens, vbar, S_out);     \
      break;                                                                                 \
    case SEED_KDA:                                                                           \
      synth_prefill_kernel<SEED_KDA, K, V><<<blocks, (V < 32 ? 32 : V), 0, st>>>(key, d.layers, d.heads, layer, \
                                                                 n_tokens, vbar, S_out);     \
      break;                                                                                 \
    default:                                                                                 \
      synth_prefill_kernel<SEED_MAMBA2, K, V><<<blocks, (V < 32 ? 32 : V), 0, st>>>(key, d.layers, d.heads,  \
                                                                    layer, n_tokens, vbar, S_out); \
  }
  SEED_SYNTH_DIMS(SEED_PRE);
#undef SEED_PRE
  return cudaGetLastError() == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
}

}  // namespace seed
