// seed_decode.cu -- the fused decode step of the sink-plus-low-rank state.
//
// "Shallow Encoding Emits Deep Memories", SEED summary (picx.dev), "Exact Update
// (Lemma 2)" with the sink recurrence of Lemma 1, and the read-out o = S+^T q.
// One CTA per (request, head) unit of the layer.  The step is HBM-bound: the unit's
// c stored columns of U and V are read once (coalesced float4, one warp-row per
// column), and only the touched bytes are written: the sink a, one new column of
// U and of V, the decay scales and the column count.
//
// Lazy decay.  Gated DeltaNet and Mamba-2 scale every old U column by the same
// scalar per step; instead of rewriting U the kernel keeps per-column scales
// gamma_j (true column = gamma_j * stored column) and updates only those.  KDA's
// decay is per channel (a row scaling of U), kept as a per-unit running product
// P (true U = Diag(P) * stored U); the new column is stored as k / P so that its
// true value is k.  Both are folded back into U by the compression.
#include "seed_common.cuh"
#include "seed_launch.h"

namespace seed {

struct DecodeParams {
  const float* q;
  const float* k;
  const float* v;
  const float* alpha;
  const float* beta;
  float* o;
  float* a;
  float* U;
  float* V;
  float* scale;
  int32_t* ncols;
  const float* vbar;
  uint32_t* status;
  int B, L, H, layer, R, W;
};

// FORM: seed_form; DK, DV: head dims; NW: warps per CTA; MAXC: bound on the
// column count c a unit may hold before the step (c <= R + W - 1 <= MAXC).
template <int FORM, int DK, int DV, int NW, int MAXC>
__global__ void __launch_bounds__(NW * 32) decode_step_kernel(const DecodeParams p) {
  constexpr int NT = NW * 32;
  constexpr int LK = DK / 4;            // lanes per U column (float4 each)
  constexpr int CPK = 32 / LK;          // U columns per warp pass
  constexpr int GK = NW * CPK;          // U column groups in the CTA
  constexpr int CU = (MAXC + GK - 1) / GK;
  constexpr int LV = DV / 4;
  constexpr int CPV = 32 / LV;
  constexpr int GV = NW * CPV;
  constexpr int CV = (MAXC + GV - 1) / GV;
  constexpr bool KDA = FORM == SEED_KDA;
  constexpr bool M2 = FORM == SEED_MAMBA2;

  __shared__ __align__(16) float s_a[DK];
  __shared__ __align__(16) float s_k[DK];
  __shared__ __align__(16) float s_q[DK];
  __shared__ __align__(16) float s_v[DV];
  __shared__ __align__(16) float s_vb[DV];
  __shared__ __align__(16) float s_al[KDA ? DK : 4];
  __shared__ __align__(16) float s_P[KDA ? DK : 4];
  __shared__ float s_dk[MAXC];
  __shared__ float s_dq[MAXC];
  __shared__ float s_gam[MAXC + 1];
  __shared__ __align__(16) float s_yk[NW][DV];
  __shared__ __align__(16) float s_yq[NW][DV];
  __shared__ float s_red[NW][5];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x;
  const int b = bh / p.H, h = bh - b * p.H;
  const long long unit = ((long long)b * p.L + p.layer) * p.H + h;
  const int m = p.R + p.W;
  const int c = p.ncols[unit];
  if (c < 0 || c >= m) {
    if (tid == 0) raise_flag(p.status, c == m ? SEED_FLAG_FULL : SEED_FLAG_BADCOLS);
    return;
  }

  // 1. issue the factor loads first: they are the bytes that bound the step
  const float* Uu = p.U + unit * (long long)m * DK;
  const float* Vu = p.V + unit * (long long)m * DV;
  const int gk = warp * CPK + lane / LK, lk = lane % LK;
  const int gv = warp * CPV + lane / LV, lv = lane % LV;
  float4 ur[CU], vr[CV];
#pragma unroll
  for (int i = 0; i < CU; ++i) {
    const int j = gk + GK * i;
    ur[i] = j < c ? ld_stream4(Uu + (long long)j * DK + 4 * lk) : zero4();
  }
#pragma unroll
  for (int i = 0; i < CV; ++i) {
    const int j = gv + GV * i;
    vr[i] = j < c ? ld_stream4(Vu + (long long)j * DV + 4 * lv) : zero4();
  }

  // 2. the unit's vectors and scalars
  for (int i = tid; i < DK / 4; i += NT) {
    st4(s_a + 4 * i, ld4(p.a + unit * DK + 4 * i));
    st4(s_k + 4 * i, ld4(p.k + (long long)bh * DK + 4 * i));
    st4(s_q + 4 * i, ld4(p.q + (long long)bh * DK + 4 * i));
    if constexpr (KDA) {
      st4(s_al + 4 * i, ld4(p.alpha + (long long)bh * DK + 4 * i));
      st4(s_P + 4 * i, ld4(p.scale + unit * DK + 4 * i));
    }
  }
  for (int i = tid; i < DV / 4; i += NT) {
    st4(s_v + 4 * i, ld4(p.v + (long long)bh * DV + 4 * i));
    st4(s_vb + 4 * i, ld4(p.vbar + ((long long)p.layer * p.H + h) * DV + 4 * i));
  }
  if constexpr (!KDA) {
    for (int j = tid; j < c; j += NT) s_gam[j] = p.scale[unit * m + j];
  }
  const float g = KDA ? 1.f : p.alpha[bh];   // GDN decay g / Mamba-2 alpha
  const float be = p.beta[bh];               // GDN/KDA beta / Mamba-2 Delta
  __syncthreads();

  // 3. dots of the stored U columns with k and q (KDA: with P+ (.) k, P+ (.) q,
  //    P+ = P (.) alpha, so that they are the dots of the decayed true columns)
  float4 kk = ld4(s_k + 4 * lk), qq = ld4(s_q + 4 * lk);
  if constexpr (KDA) {
    const float4 pp = mul4(ld4(s_P + 4 * lk), ld4(s_al + 4 * lk));
    kk = mul4(kk, pp);
    qq = mul4(qq, pp);
  }
  float dk[CU], dq[CU];
#pragma unroll
  for (int i = 0; i < CU; ++i) {
    dk[i] = dot4(ur[i], kk);
    dq[i] = dot4(ur[i], qq);
  }
#pragma unroll
  for (int i = 0; i < CU; ++i) {
    if constexpr (!M2) dk[i] = group_sum<LK>(dk[i]);
    dq[i] = group_sum<LK>(dq[i]);
  }
  if (lk == 0) {
#pragma unroll
    for (int i = 0; i < CU; ++i) {
      const int j = gk + GK * i;
      if (j < c) {
        s_dk[j] = dk[i];
        s_dq[j] = dq[i];
      }
    }
  }

  // scalars: k^T a', a'^T q, k^T q (a' = alpha (.) a for KDA), v^T vbar, vbar^T vbar
  float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f, r4 = 0.f;
  for (int i = tid; i < DK; i += NT) {
    const float ai = KDA ? s_al[i] * s_a[i] : s_a[i];
    r0 = fmaf(s_k[i], ai, r0);
    r1 = fmaf(ai, s_q[i], r1);
    r2 = fmaf(s_k[i], s_q[i], r2);
  }
  for (int i = tid; i < DV; i += NT) {
    r3 = fmaf(s_v[i], s_vb[i], r3);
    r4 = fmaf(s_vb[i], s_vb[i], r4);
  }
  r0 = group_sum<32>(r0);
  r1 = group_sum<32>(r1);
  r2 = group_sum<32>(r2);
  r3 = group_sum<32>(r3);
  r4 = group_sum<32>(r4);
  if (lane == 0) {
    s_red[warp][0] = r0;
    s_red[warp][1] = r1;
    s_red[warp][2] = r2;
    s_red[warp][3] = r3;
    s_red[warp][4] = r4;
  }
  __syncthreads();
  float ka = 0.f, aq = 0.f, kq = 0.f, vvb = 0.f, vbvb = 0.f;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    ka += s_red[w][0];
    aq += s_red[w][1];
    kq += s_red[w][2];
    vvb += s_red[w][3];
    vbvb += s_red[w][4];
  }
  if (!(vbvb > 0.f)) {
    if (tid == 0) raise_flag(p.status, SEED_FLAG_ZERO_VBAR);
    return;
  }
  const float omega = vvb / vbvb;

  // 4. V times the column coefficients: y_k = V (g gamma (.) U^T k) for the erase
  //    term, y_q = V (g gamma (.) U^T q) for the read-out (decayed true columns)
  float4 yk = zero4(), yq = zero4();
#pragma unroll
  for (int i = 0; i < CV; ++i) {
    const int j = gv + GV * i;
    if (j < c) {
      const float sc = KDA ? 1.f : g * s_gam[j];
      if constexpr (!M2) yk = fma4(sc * s_dk[j], vr[i], yk);
      yq = fma4(sc * s_dq[j], vr[i], yq);
    }
  }
#pragma unroll
  for (int off = LV; off < 32; off <<= 1) {
    yk.x += __shfl_xor_sync(0xffffffffu, yk.x, off);
    yk.y += __shfl_xor_sync(0xffffffffu, yk.y, off);
    yk.z += __shfl_xor_sync(0xffffffffu, yk.z, off);
    yk.w += __shfl_xor_sync(0xffffffffu, yk.w, off);
    yq.x += __shfl_xor_sync(0xffffffffu, yq.x, off);
    yq.y += __shfl_xor_sync(0xffffffffu, yq.y, off);
    yq.z += __shfl_xor_sync(0xffffffffu, yq.z, off);
    yq.w += __shfl_xor_sync(0xffffffffu, yq.w, off);
  }
  if (lane < LV) {
    st4(&s_yk[warp][4 * lane], yk);
    st4(&s_yq[warp][4 * lane], yq);
  }
  __syncthreads();

  // 5. sink update, new column pair, read-out
  float coef;   // a+ = a' + coef * k   (a' = g a, alpha (.) a, alpha a)
  if constexpr (FORM == SEED_GDN) coef = be * (omega - g * ka);
  else if constexpr (KDA) coef = be * (omega - ka);
  else coef = be * omega;
  const float apq = (KDA ? aq : g * aq) + coef * kq;   // a+^T q
  bool bad = false;
  float* Vnew = p.V + unit * (long long)m * DV + (long long)c * DV;
  float* Unew = p.U + unit * (long long)m * DK + (long long)c * DK;
  for (int i = tid; i < DV; i += NT) {
    float yki = 0.f, yqi = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      yki += s_yk[w][i];
      yqi += s_yq[w][i];
    }
    const float eps = s_v[i] - omega * s_vb[i];
    const float ncol = M2 ? be * eps : be * (eps - yki);
    const float oi = fmaf(s_vb[i], apq, yqi) + ncol * kq;
    bad |= !(isfinite(ncol) && isfinite(oi));
    Vnew[i] = ncol;
    p.o[(long long)bh * DV + i] = oi;
  }
  for (int i = tid; i < DK; i += NT) {
    const float ai = s_a[i];
    const float ki = s_k[i];
    float anew;
    if constexpr (KDA) {
      const float pn = s_P[i] * s_al[i];
      anew = fmaf(s_al[i], ai, coef * ki);
      const float us = ki / pn;
      bad |= !isfinite(us);
      Unew[i] = us;
      p.scale[unit * DK + i] = pn;
    } else {
      anew = fmaf(g, ai, coef * ki);
      Unew[i] = ki;
    }
    bad |= !isfinite(anew);
    p.a[unit * DK + i] = anew;
  }
  if constexpr (!KDA) {
    for (int j = tid; j <= c; j += NT) p.scale[unit * m + j] = j < c ? g * s_gam[j] : 1.f;
  }
  if (tid == 0) p.ncols[unit] = c + 1;
  if (bad) raise_flag(p.status, SEED_FLAG_NONFINITE);
}

template <int FORM, int DK, int DV, int NW, int MAXC>
static int launch_one(const DecodeParams& p, int blocks, cudaStream_t st) {
  decode_step_kernel<FORM, DK, DV, NW, MAXC><<<blocks, NW * 32, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
}

template <int FORM, int DK, int DV>
static int launch_cols(const DecodeParams& p, int blocks, cudaStream_t st) {
  const int maxc = p.R + p.W - 1;
  if (maxc <= 8) return launch_one<FORM, DK, DV, 4, 8>(p, blocks, st);
  if (maxc <= 16) return launch_one<FORM, DK, DV, 4, 16>(p, blocks, st);
  if (maxc <= 32) return launch_one<FORM, DK, DV, 4, 32>(p, blocks, st);
  if (maxc <= 64) return launch_one<FORM, DK, DV, 8, 64>(p, blocks, st);
  return launch_one<FORM, DK, DV, 12, 96>(p, blocks, st);
}

template <int FORM>
static int launch_dims(const DecodeParams& p, int dk, int dv, int blocks, cudaStream_t st) {
#define SEED_DIMS_CASE(K, V) \
  if (dk == K && dv == V) return launch_cols<FORM, K, V>(p, blocks, st);
  SEED_DIMS_CASE(16, 16)
  SEED_DIMS_CASE(32, 32)
  SEED_DIMS_CASE(64, 64)
  SEED_DIMS_CASE(128, 128)
  SEED_DIMS_CASE(128, 64)
  SEED_DIMS_CASE(64, 128)
#undef SEED_DIMS_CASE
  return SEED_ERR_SHAPE;
}

int launch_decode_step(const seed_dims& d, const seed_state& s, int layer, const float* q,
                       const float* k, const float* v, const float* alpha, const float* beta,
                       float* o, uint32_t* status, cudaStream_t st) {
  DecodeParams p{q, k, v, alpha, beta, o, s.a, s.U, s.V, s.scale, s.ncols, s.vbar, status,
                 d.batch, d.layers, d.heads, layer, d.R, d.W};
  const int blocks = d.batch * d.heads;
  switch (d.form) {
    case SEED_GDN: return launch_dims<SEED_GDN>(p, d.d_k, d.d_v, blocks, st);
    case SEED_KDA: return launch_dims<SEED_KDA>(p, d.d_k, d.d_v, blocks, st);
    case SEED_MAMBA2: return launch_dims<SEED_MAMBA2>(p, d.d_k, d.d_v, blocks, st);
  }
  return SEED_ERR_INVALID_ARG;
}

bool decode_dims_supported(int dk, int dv) {
  return (dk == dv && (dk == 16 || dk == 32 || dk == 64 || dk == 128)) ||
         (dk == 128 && dv == 64) || (dk == 64 && dv == 128);
}

}  // namespace seed
