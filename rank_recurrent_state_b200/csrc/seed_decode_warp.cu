// seed_decode_warp.cu -- the decode step with one warp per unit, for R + W <= 33.
//
// "Shallow Encoding Emits Deep Memories", SEED summary (picx.dev), "Exact Update
// (Lemma 2)" with the sink recurrence of Lemma 1, and the read-out o = S+^T q;
// the arithmetic is that of seed_decode.cu, organised differently.
//
// With at most 32 stored columns a unit is small enough for one warp, and a warp
// that owns a unit needs no block-level synchronisation at all.  Every warp of a
// persistent grid (one warp per block) owns NSW shared-memory stages; lane 0 fills
// a stage with TMA bulk copies (cp.async.bulk, completion on the stage's mbarrier,
// no multicast) for the warp's next unit as soon as the warp has finished reading
// it, so the copies of one warp overlap the arithmetic of the others.  Each lane
// holds d_k / 32 rows of every U column and d_v / 32 rows of every V column:
//   1. U^T q and U^T k by partial dot products over the lane's rows, summed over
//      the warp sixteen columns at a time by a transposed (recursive-halving)
//      reduction that leaves one dot per lane, which that lane scales into the
//      column's coefficient for step 3;
//   2. the scalars k^T a, a^T q, k^T q, v^T vbar, vbar^T vbar the same way;
//   3. y_k = V (g gamma (.) U^T k) and y_q = V (g gamma (.) U^T q), each lane for
//      its own rows, no reduction;
//   4. the sink update, the new column pair and the read-out, written straight
//      from registers.
#include "seed_common.cuh"
#include "seed_decode.cuh"
#include "seed_launch.h"
#include "seed_tma.cuh"

namespace seed {

// P consecutive floats at p (P = 4, 2 or 1; p aligned to 4 P bytes).
template <int P>
SEED_DEV void ldv(const float* p, float (&e)[P]) {
  if constexpr (P == 4) {
    const float4 t = ld4(p);
    e[0] = t.x; e[1] = t.y; e[2] = t.z; e[3] = t.w;
  } else if constexpr (P == 2) {
    const float2 t = *reinterpret_cast<const float2*>(p);
    e[0] = t.x; e[1] = t.y;
  } else {
    e[0] = *p;
  }
}

template <int P>
SEED_DEV void stv(float* p, const float (&e)[P]) {
  if constexpr (P == 4) {
    st4(p, make_float4(e[0], e[1], e[2], e[3]));
  } else if constexpr (P == 2) {
    *reinterpret_cast<float2*>(p) = make_float2(e[0], e[1]);
  } else {
    *p = e[0];
  }
}

template <int P>
SEED_DEV float dotv(const float (&a)[P], const float (&b)[P]) {
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < P; ++e) s = fmaf(a[e], b[e], s);
  return s;
}

SEED_DEV long long unit_index(const DecodeParams& p, int u) {
  const int b = u / p.H, h = u - b * p.H;
  return ((long long)b * p.L + p.layer) * p.H + h;
}

// Lane 0: the bulk copies of unit u (c stored columns) into stage S, completing on
// bar.  A unit with an invalid column count gets no copies (the wait still ends).
template <int FORM, int DK, int DV, int MAXC>
SEED_DEV void issue_unit(const DecodeParams& p, DecodeStage<FORM, DK, DV, MAXC>& S, uint64_t* bar,
                         int u, int c, int m) {
  constexpr bool KDA = FORM == SEED_KDA;
  const long long unit = unit_index(p, u);
  const int h = u % p.H;
  const bool valid = c >= 0 && c < m;
  uint32_t bytes = 0;
  if (valid) {
    bytes = (uint32_t)(c * (DK + DV) + 3 * DK + 2 * DV) * 4u;
    bytes += KDA ? 2u * DK * 4u : (uint32_t)((c + 3) & ~3) * 4u;
  }
  mbar_arrive_expect_tx(bar, bytes);
  if (!valid) return;
  if (c > 0) {
    bulk_g2s(S.U, p.U + unit * (long long)m * DK, (uint32_t)(c * DK * 4), bar);
    bulk_g2s(S.V, p.V + unit * (long long)m * DV, (uint32_t)(c * DV * 4), bar);
  }
  bulk_g2s(S.a, p.a + unit * DK, DK * 4, bar);
  bulk_g2s(S.k, p.k + (long long)u * DK, DK * 4, bar);
  bulk_g2s(S.q, p.q + (long long)u * DK, DK * 4, bar);
  bulk_g2s(S.v, p.v + (long long)u * DV, DV * 4, bar);
  bulk_g2s(S.vb, p.vbar + ((long long)p.layer * p.H + h) * DV, DV * 4, bar);
  if constexpr (KDA) {
    bulk_g2s(S.al, p.alpha + (long long)u * DK, DK * 4, bar);
    bulk_g2s(S.P, p.scale + unit * DK, DK * 4, bar);
  } else if (c > 0) {
    bulk_g2s(S.gam, p.scale + unit * p.slen, (uint32_t)((c + 3) & ~3) * 4u, bar);
  }
}

template <int FORM, int DK, int DV, int MAXC, int NSW>
struct WarpDecodeLayout {
  using Stage = DecodeStage<FORM, DK, DV, MAXC>;
  static constexpr int NCH = (MAXC + 31) / 32 * 4;   // coefficient pairs, in units of 8
  static constexpr size_t OFF_BAR = NSW * sizeof(Stage);
  static constexpr size_t OFF_DOT = OFF_BAR + 16 * ((NSW * 8 + 15) / 16);
  static constexpr size_t bytes = OFF_DOT + 2 * NCH * 8 * sizeof(float);
};

template <int FORM, int DK, int DV, int MAXC, int NSW>
__global__ void __launch_bounds__(32) decode_warp_kernel(const DecodeParams p) {
  using Lay = WarpDecodeLayout<FORM, DK, DV, MAXC, NSW>;
  using Stage = typename Lay::Stage;
  constexpr bool KDA = FORM == SEED_KDA;
  constexpr bool M2 = FORM == SEED_MAMBA2;
  constexpr int PK = DK >= 32 ? DK / 32 : 1;   // U rows per lane (d_k = 16: half the lanes)
  constexpr int PV = DV >= 32 ? DV / 32 : 1;
  constexpr int CPS = M2 ? 32 : 16;            // columns per warp reduction
  static_assert(NSW == 1 || NSW == 2, "one or two stages per warp");
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Stage* stages = reinterpret_cast<Stage*>(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw + Lay::OFF_BAR);
  float* s_f = reinterpret_cast<float*>(smem_raw + Lay::OFF_DOT);   // [MAXC][2]

  const int lane = threadIdx.x;
  const bool kact = DK >= 32 || lane < DK;
  const bool vact = DV >= 32 || lane < DV;
  const int n_units = p.B * p.H;
  const int m = p.R + p.W;
  const int stride = gridDim.x;
  const int u0 = blockIdx.x;
  if (lane == 0) {
    for (int s = 0; s < NSW; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  // prime the stages with the warp's first units
  int c_s0 = 0, c_s1 = 0;
#pragma unroll
  for (int k = 0; k < NSW; ++k) {
    const int u = u0 + k * stride;
    const int c = u < n_units ? p.ncols[unit_index(p, u)] : 0;
    if (k == 0) c_s0 = c;
    else c_s1 = c;
    if (lane == 0 && u < n_units) issue_unit<FORM, DK, DV, MAXC>(p, stages[k], &full[k], u, c, m);
  }
  int c_next = 0;   // column count of the unit that will refill the current stage
  {
    const int u = u0 + NSW * stride;
    if (u < n_units) c_next = p.ncols[unit_index(p, u)];
  }
  // the scalars of the current unit, loaded one unit ahead
  float g_cur = (KDA || u0 >= n_units) ? 1.f : p.alpha[u0];
  float b_cur = u0 < n_units ? p.beta[u0] : 0.f;

  for (int i = 0, u = u0; u < n_units; ++i, u += stride) {
    const int s = NSW == 1 ? 0 : (i & 1);
    const uint32_t ph = (uint32_t)(i / NSW) & 1u;
    const int c = s == 0 ? c_s0 : c_s1;
    const long long unit = unit_index(p, u);
    const float g = g_cur, be = b_cur;
    const int u_next = u + NSW * stride;
    const int u_after = u_next + stride;
    const int c_after = u_after < n_units ? p.ncols[unit_index(p, u_after)] : 0;
    if (u + stride < n_units) {
      g_cur = KDA ? 1.f : p.alpha[u + stride];
      b_cur = p.beta[u + stride];
    }

    if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full[s], ph, kWaitLimitNs))) {
      if (lane == 0) raise_flag(p.status, SEED_FLAG_TIMEOUT);
      for (int k = 0; k < NSW; ++k)   // let the copies in flight land before the block exits
        mbar_wait_bounded(&full[(s + k) % NSW], (uint32_t)((i + k) / NSW) & 1u, kWaitLimitNs);
      return;
    }
    const Stage& S = stages[s];
    if (c < 0 || c >= m) {
      if (lane == 0) raise_flag(p.status, c == m ? SEED_FLAG_FULL : SEED_FLAG_BADCOLS);
    } else {
      // 1. dots of the stored U columns with q and k (KDA: with P+ (.) q and P+ (.) k,
      //    P+ = P (.) alpha, the dots of the decayed true columns)
      float kr[PK], qr[PK], kk[PK], qq[PK], ar[PK], alr[PK], pr[PK];
#pragma unroll
      for (int e = 0; e < PK; ++e) kr[e] = qr[e] = ar[e] = 0.f, alr[e] = pr[e] = 1.f;
      if (kact) {
        ldv<PK>(S.k + lane * PK, kr);
        ldv<PK>(S.q + lane * PK, qr);
        ldv<PK>(S.a + lane * PK, ar);
        if constexpr (KDA) {
          ldv<PK>(S.al + lane * PK, alr);
          ldv<PK>(S.P + lane * PK, pr);
        }
      }
#pragma unroll
      for (int e = 0; e < PK; ++e) {
        const float pp = KDA ? pr[e] * alr[e] : 1.f;
        kk[e] = kr[e] * pp;
        qq[e] = qr[e] * pp;
      }
      // 16 columns per reduction (32 for Mamba-2, which has no erase): lane l ends up
      // with dot number l; it turns it into the column's y coefficient
      // g gamma_j (U^T q)_j or g gamma_j (U^T k)_j, stored as (q, k) pairs
      for (int c0 = 0; c0 < c; c0 += CPS) {
        float dv[32];
#pragma unroll
        for (int t = 0; t < CPS; ++t) {
          const int j = c0 + t;
          float ue[PK];
#pragma unroll
          for (int e = 0; e < PK; ++e) ue[e] = 0.f;
          if (j < c && kact) ldv<PK>(S.U + j * DK + lane * PK, ue);
          dv[t] = dotv<PK>(ue, qq);
          if constexpr (!M2) dv[16 + t] = dotv<PK>(ue, kk);
        }
        const float tot = warp_xreduce<32>(dv);
        const int j = c0 + (M2 ? lane : (lane & 15));
        if (j < c) {
          const float f = KDA ? 1.f : g * S.gam[j];
          s_f[2 * j + (M2 ? 0 : (lane >> 4))] = f * tot;
        }
      }
      // 2. scalars: k^T a', a'^T q, k^T q (a' = alpha (.) a for KDA), v^T vbar, vbar^T vbar
      float vr[PV], vbr[PV];
#pragma unroll
      for (int e = 0; e < PV; ++e) vr[e] = vbr[e] = 0.f;
      if (vact) {
        ldv<PV>(S.v + lane * PV, vr);
        ldv<PV>(S.vb + lane * PV, vbr);
      }
      float sc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int e = 0; e < PK; ++e) {
        const float ae = KDA ? alr[e] * ar[e] : ar[e];
        sc[0] = fmaf(kr[e], ae, sc[0]);
        sc[1] = fmaf(ae, qr[e], sc[1]);
        sc[2] = fmaf(kr[e], qr[e], sc[2]);
      }
#pragma unroll
      for (int e = 0; e < PV; ++e) {
        sc[3] = fmaf(vr[e], vbr[e], sc[3]);
        sc[4] = fmaf(vbr[e], vbr[e], sc[4]);
      }
      const float tot = warp_xreduce<8>(sc);   // lane 4 i holds scalar i
      const float ka = __shfl_sync(0xffffffffu, tot, 0);
      const float aq = __shfl_sync(0xffffffffu, tot, 4);
      const float kq = __shfl_sync(0xffffffffu, tot, 8);
      const float vvb = __shfl_sync(0xffffffffu, tot, 12);
      const float vbvb = __shfl_sync(0xffffffffu, tot, 16);
      __syncwarp();   // the column coefficients are in s_f
      if (!(vbvb > 0.f)) {
        if (lane == 0) raise_flag(p.status, SEED_FLAG_ZERO_VBAR);
      } else {
        const float omega = vvb / vbvb;
        // 3. y_k = V (g gamma (.) U^T k) for the erase, y_q = V (g gamma (.) U^T q)
        //    for the read-out (decayed true columns); each lane its own rows
        float yk[PV], yq[PV];
#pragma unroll
        for (int e = 0; e < PV; ++e) yk[e] = yq[e] = 0.f;
#pragma unroll 4
        for (int j = 0; j < c; ++j) {
          float ve[PV];
#pragma unroll
          for (int e = 0; e < PV; ++e) ve[e] = 0.f;
          if (vact) ldv<PV>(S.V + j * DV + lane * PV, ve);
          const float2 f2 = *reinterpret_cast<const float2*>(s_f + 2 * j);   // (q, k) coefficients
#pragma unroll
          for (int e = 0; e < PV; ++e) {
            if constexpr (!M2) yk[e] = fmaf(f2.y, ve[e], yk[e]);
            yq[e] = fmaf(f2.x, ve[e], yq[e]);
          }
        }
        // 4. sink update, new column pair, read-out
        float coef;   // a+ = a' + coef * k   (a' = g a, alpha (.) a, alpha a)
        if constexpr (FORM == SEED_GDN) coef = be * (omega - g * ka);
        else if constexpr (KDA) coef = be * (omega - ka);
        else coef = be * omega;
        const float apq = (KDA ? aq : g * aq) + coef * kq;   // a+^T q
        bool bad = false;
        if (vact) {
          float ncol[PV], oe[PV];
#pragma unroll
          for (int e = 0; e < PV; ++e) {
            const float eps = vr[e] - omega * vbr[e];
            ncol[e] = M2 ? be * eps : be * (eps - yk[e]);
            oe[e] = fmaf(vbr[e], apq, yq[e]) + ncol[e] * kq;
            bad |= !(isfinite(ncol[e]) && isfinite(oe[e]));
          }
          stv<PV>(p.V + unit * (long long)m * DV + (long long)c * DV + lane * PV, ncol);
          stv<PV>(p.o + (long long)u * DV + lane * PV, oe);
        }
        if (kact) {
          float anew[PK], unew[PK], pn[PK];
#pragma unroll
          for (int e = 0; e < PK; ++e) {
            if constexpr (KDA) {
              pn[e] = pr[e] * alr[e];
              anew[e] = fmaf(alr[e], ar[e], coef * kr[e]);
              unew[e] = kr[e] / pn[e];
              bad |= !isfinite(unew[e]);
            } else {
              anew[e] = fmaf(g, ar[e], coef * kr[e]);
              unew[e] = kr[e];
            }
            bad |= !isfinite(anew[e]);
          }
          stv<PK>(p.U + unit * (long long)m * DK + (long long)c * DK + lane * PK, unew);
          stv<PK>(p.a + unit * DK + lane * PK, anew);
          if constexpr (KDA) stv<PK>(p.scale + unit * DK + lane * PK, pn);
        }
        if constexpr (!KDA) {
          for (int j = lane; j <= c; j += 32) p.scale[unit * p.slen + j] = j < c ? g * S.gam[j] : 1.f;
        }
        if (lane == 0) p.ncols[unit] = c + 1;
        if (__any_sync(0xffffffffu, bad) && lane == 0) raise_flag(p.status, SEED_FLAG_NONFINITE);
      }
    }
    // every read of the stage (and of s_f) is above: refill the stage
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && u_next < n_units) issue_unit<FORM, DK, DV, MAXC>(p, stages[s], &full[s], u_next, c_next, m);
    if (s == 0) c_s0 = c_next;
    else c_s1 = c_next;
    c_next = c_after;
  }
}

template <int FORM, int DK, int DV, int MAXC, int NSW>
static int launch_warp_t(const DecodeParams& p, cudaStream_t st) {
  using Lay = WarpDecodeLayout<FORM, DK, DV, MAXC, NSW>;
  auto kern = decode_warp_kernel<FORM, DK, DV, MAXC, NSW>;
  constexpr int kMaxDev = 64;
  static int grid_per_sm[kMaxDev] = {0};
  static int sm_count[kMaxDev] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return SEED_ERR_CUDA;
  if (grid_per_sm[dev] == 0) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lay::bytes) !=
        cudaSuccess)
      return SEED_ERR_CUDA;
    int n = 0, sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return SEED_ERR_CUDA;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 32, Lay::bytes) != cudaSuccess)
      return SEED_ERR_CUDA;
    sm_count[dev] = sms;
    grid_per_sm[dev] = n > 0 ? n : 1;
  }
  const int units = p.B * p.H;
  int grid = grid_per_sm[dev] * sm_count[dev];
  if (grid > units) grid = units;
  kern<<<grid, 32, Lay::bytes, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
}

template <int FORM, int DK, int DV>
static int launch_warp_dims(const DecodeParams& p, cudaStream_t st) {
  const int maxc = p.R + p.W - 1;
  if (maxc <= 8) return launch_warp_t<FORM, DK, DV, 8, 1>(p, st);
  if (maxc <= 16) return launch_warp_t<FORM, DK, DV, 16, 1>(p, st);
  return launch_warp_t<FORM, DK, DV, 32, 1>(p, st);
}

bool decode_warp_supported(const seed_dims& d) { return d.R + d.W - 1 <= 32; }

int launch_decode_warp(const DecodeParams& p, int form, int dk, int dv, cudaStream_t st) {
#define SEED_WARP_DIMS(FORM)                                                     \
  do {                                                                           \
    if (dk == 16 && dv == 16) return launch_warp_dims<FORM, 16, 16>(p, st);      \
    if (dk == 32 && dv == 32) return launch_warp_dims<FORM, 32, 32>(p, st);      \
    if (dk == 64 && dv == 64) return launch_warp_dims<FORM, 64, 64>(p, st);      \
    if (dk == 128 && dv == 128) return launch_warp_dims<FORM, 128, 128>(p, st);  \
    if (dk == 128 && dv == 64) return launch_warp_dims<FORM, 128, 64>(p, st);    \
    if (dk == 64 && dv == 128) return launch_warp_dims<FORM, 64, 128>(p, st);    \
    return SEED_ERR_SHAPE;                                                       \
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
