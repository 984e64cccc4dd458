// seed_dense.cu -- the dense-state decode step SEED replaces (in-run comparison).
//
// Every decode step of the original model loads and stores whole recurrent
// states ("Shallow Encoding Emits Deep Memories", abstract (readsearch.ai)).  One
// CTA per (request, head): the d_k x d_v state is read once into registers
// (coalesced float4 rows), the two reductions S^T k and S^T q are formed, the
// state is updated in registers and streamed back, and o = S+^T q is written:
//   GDN      S+ = g (S - beta k (k^T S)) + beta k v^T
//            o  = g S^T q - g beta (k^T q) S^T k + beta (k^T q) v
//   KDA      S+ = D S - beta k (k^T D S) + beta k v^T,  D = Diag(alpha)
//            o  = S^T (alpha (.) q) - beta (k^T q) S^T (alpha (.) k) + beta (k^T q) v
//   Mamba-2  S+ = alpha S + Delta k v^T,  o = alpha S^T q + Delta (k^T q) v
#include "seed_common.cuh"
#include "seed_launch.h"

namespace seed {

struct DenseParams {
  float* S;
  const float* q;
  const float* k;
  const float* v;
  const float* alpha;
  const float* beta;
  float* o;
  uint32_t* status;
  int B, L, H, layer;
};

template <int FORM, int DK, int DV, int NT>
__global__ void __launch_bounds__(NT) dense_step_kernel(const DenseParams p) {
  constexpr int CQ = DV / 4;        // column quads
  constexpr int RG = NT / CQ;       // row groups
  constexpr int RPT = DK / RG;      // rows per thread
  static_assert(RPT >= 1 && RG * CQ == NT, "tile");
  constexpr bool KDA = FORM == SEED_KDA;
  __shared__ __align__(16) float s_k[DK], s_q[DK], s_v[DV], s_al[KDA ? DK : 4];
  __shared__ __align__(16) float s_pk[RG][DV], s_pq[RG][DV];
  __shared__ float s_kq;

  const int tid = threadIdx.x;
  const int cq = tid % CQ, rg = tid / CQ;
  const int bh = blockIdx.x;
  const int b = bh / p.H, h = bh - b * p.H;
  const long long unit = ((long long)b * p.L + p.layer) * p.H + h;
  float* S = p.S + unit * (long long)DK * DV;

  float4 sr[RPT];
#pragma unroll
  for (int t = 0; t < RPT; ++t) sr[t] = ld_stream4(S + (long long)(rg + RG * t) * DV + 4 * cq);
  for (int i = tid; i < DK; i += NT) {
    s_k[i] = p.k[(long long)bh * DK + i];
    s_q[i] = p.q[(long long)bh * DK + i];
    if constexpr (KDA) s_al[i] = p.alpha[(long long)bh * DK + i];
  }
  for (int i = tid; i < DV; i += NT) s_v[i] = p.v[(long long)bh * DV + i];
  if (tid < 32) {
    float x = 0.f;
    for (int i = tid; i < DK; i += 32) x = fmaf(p.k[(long long)bh * DK + i], p.q[(long long)bh * DK + i], x);
    x = group_sum<32>(x);
    if (tid == 0) s_kq = x;
  }
  const float g = KDA ? 1.f : p.alpha[bh];
  const float be = p.beta[bh];
  __syncthreads();

  float4 pk = zero4(), pq = zero4();
#pragma unroll
  for (int t = 0; t < RPT; ++t) {
    const int i = rg + RG * t;
    const float wk = KDA ? s_k[i] * s_al[i] : s_k[i];
    const float wq = KDA ? s_q[i] * s_al[i] : s_q[i];
    pk = fma4(wk, sr[t], pk);
    pq = fma4(wq, sr[t], pq);
  }
  st4(&s_pk[rg][4 * cq], pk);
  st4(&s_pq[rg][4 * cq], pq);
  __syncthreads();
  float kS[4], qS[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float a = 0.f, bq = 0.f;
#pragma unroll
    for (int r = 0; r < RG; ++r) {
      a += s_pk[r][4 * cq + e];
      bq += s_pq[r][4 * cq + e];
    }
    kS[e] = a;
    qS[e] = bq;
  }
  const float kq = s_kq;
  // per-column write coefficient w_j: S+[i][j] = (decay) S[i][j] + k_i w_j
  float w[4];
  const float vj[4] = {s_v[4 * cq], s_v[4 * cq + 1], s_v[4 * cq + 2], s_v[4 * cq + 3]};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    if constexpr (FORM == SEED_GDN) w[e] = be * (vj[e] - g * kS[e]);
    else if constexpr (KDA) w[e] = be * (vj[e] - kS[e]);
    else w[e] = be * vj[e];
  }
  bool bad = false;
#pragma unroll
  for (int t = 0; t < RPT; ++t) {
    const int i = rg + RG * t;
    const float ki = s_k[i];
    const float dec = KDA ? s_al[i] : g;
    float4 x = sr[t];
    x.x = fmaf(dec, x.x, ki * w[0]);
    x.y = fmaf(dec, x.y, ki * w[1]);
    x.z = fmaf(dec, x.z, ki * w[2]);
    x.w = fmaf(dec, x.w, ki * w[3]);
    st_stream4(S + (long long)i * DV + 4 * cq, x);
  }
  if (rg == 0) {
    float4 o;
    float* op = &o.x;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      // o_j = (decayed S)^T q + (k^T q) w_j
      op[e] = (KDA ? qS[e] : g * qS[e]) + kq * w[e];
      bad |= !isfinite(op[e]);
    }
    st4(p.o + (long long)bh * DV + 4 * cq, o);
  }
  if (bad) raise_flag(p.status, SEED_FLAG_NONFINITE);
}

template <int FORM, int DK, int DV>
static int launch_dense_t(const DenseParams& p, int blocks, cudaStream_t st) {
  constexpr int NT0 = DK * DV / 4 < 256 ? DK * DV / 4 : 256;
  dense_step_kernel<FORM, DK, DV, NT0><<<blocks, NT0, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
}

#define SEED_DENSE_DIMS(FORM)                                                           \
  do {                                                                                  \
    if (d.d_k == 16 && d.d_v == 16) return launch_dense_t<FORM, 16, 16>(p, blocks, st);   \
    if (d.d_k == 32 && d.d_v == 32) return launch_dense_t<FORM, 32, 32>(p, blocks, st);   \
    if (d.d_k == 64 && d.d_v == 64) return launch_dense_t<FORM, 64, 64>(p, blocks, st);   \
    if (d.d_k == 128 && d.d_v == 128) return launch_dense_t<FORM, 128, 128>(p, blocks, st); \
    if (d.d_k == 128 && d.d_v == 64) return launch_dense_t<FORM, 128, 64>(p, blocks, st); \
    if (d.d_k == 64 && d.d_v == 128) return launch_dense_t<FORM, 64, 128>(p, blocks, st); \
    return SEED_ERR_SHAPE;                                                              \
  } while (0)

int launch_dense_step(const seed_dims& d, float* S, int layer, const float* q, const float* k,
                      const float* v, const float* alpha, const float* beta, float* o,
                      uint32_t* status, cudaStream_t st) {
  DenseParams p{S, q, k, v, alpha, beta, o, status, d.batch, d.layers, d.heads, layer};
  const int blocks = d.batch * d.heads;
  switch (d.form) {
    case SEED_GDN: SEED_DENSE_DIMS(SEED_GDN);
    case SEED_KDA: SEED_DENSE_DIMS(SEED_KDA);
    case SEED_MAMBA2: SEED_DENSE_DIMS(SEED_MAMBA2);
  }
  return SEED_ERR_INVALID_ARG;
}

}  // namespace seed
