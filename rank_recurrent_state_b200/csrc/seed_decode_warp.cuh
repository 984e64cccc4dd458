// seed_decode_warp.cuh -- the decode step with one warp per unit, for R + W <= 65.
//
// "Shallow Encoding Emits Deep Memories", SEED summary (picx.dev), "Exact Update
// (Lemma 2)" with the sink recurrence of Lemma 1, and the read-out o = S+^T q;
// the arithmetic is that of seed_decode.cu, organised differently.
//
// With at most 64 stored columns a unit is small enough for one warp, and a warp
// that owns a unit needs no block-level synchronisation at all.  Every warp of a
// persistent grid (one warp per block) owns one shared-memory stage sized for the
// R + W - 1 columns a unit holds at most before a step; lane 0 fills it with two
// TMA bulk copies (cp.async.bulk of the stored U and V columns, completion on the
// stage's mbarrier, no multicast) for the warp's next unit as soon as the warp has
// read the current one, so the copies of one warp overlap the arithmetic of the
// others.  The per-unit vectors (k, q, a, v, vbar, the decay scales, g, beta) go
// straight from HBM into each lane's registers with coalesced loads issued one unit
// ahead, so that they cost neither stage space nor copies:
//   1. U^T q and U^T k by partial dot products over the lane's rows, summed over
//      the warp sixteen columns at a time by a transposed (recursive-halving)
//      reduction that leaves one dot per lane, which that lane scales into the
//      column's coefficient for step 3;
//   2. the scalars k^T a, a^T q, k^T q, v^T vbar, vbar^T vbar the same way;
//   3. y_k = V (g gamma (.) U^T k) and y_q = V (g gamma (.) U^T q), each lane for
//      its own rows, no reduction;
//   4. the sink update, the new column pair and the read-out, written straight
//      from registers.
// With 16-bit factors (fp16, bf16) the stage holds the stored 16-bit columns (half
// the space, so more warps per SM), widened to float32 as they are read; the new
// pair is rounded to nearest as it is stored.
#pragma once

#include "seed_common.cuh"
#include "seed_compress_fast.cuh"
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

// The per-unit vectors one lane needs, in registers: its d_k / 32 rows of k, q, a
// (KDA: alpha, P) and d_v / 32 rows of v, vbar; the decay scales of the columns
// whose coefficients it forms (j = lane & 15 and 16 + (lane & 15); Mamba-2: j =
// lane); and the unit's g (alpha) and beta.
template <int FORM, int DK, int DV>
struct UnitVecs {
  static constexpr int PK = DK >= 32 ? DK / 32 : 1, PV = DV >= 32 ? DV / 32 : 1;
  float k[PK], q[PK], a[PK], al[PK], P[PK], v[PV], vb[PV];
  float gam_lo, gam_hi, g, be;
};

template <int FORM, int DK, int DV>
SEED_DEV void load_vecs(const DecodeParams& p, int u, int c, UnitVecs<FORM, DK, DV>& r) {
  constexpr bool KDA = FORM == SEED_KDA, M2 = FORM == SEED_MAMBA2;
  constexpr int PK = UnitVecs<FORM, DK, DV>::PK, PV = UnitVecs<FORM, DK, DV>::PV;
  const int lane = threadIdx.x & 31;
  const long long unit = unit_index(p, u);
  const int h = u % p.H;
#pragma unroll
  for (int e = 0; e < PK; ++e) r.k[e] = r.q[e] = r.a[e] = 0.f, r.al[e] = r.P[e] = 1.f;
#pragma unroll
  for (int e = 0; e < PV; ++e) r.v[e] = r.vb[e] = 0.f;
  if (DK >= 32 || lane < DK) {
    ldv<PK>(p.k + (long long)u * DK + lane * PK, r.k);
    ldv<PK>(p.q + (long long)u * DK + lane * PK, r.q);
    ldv<PK>(p.a + unit * DK + lane * PK, r.a);
    if constexpr (KDA) {
      ldv<PK>(p.alpha + (long long)u * DK + lane * PK, r.al);
      ldv<PK>(p.scale + unit * DK + lane * PK, r.P);
    }
  }
  if (DV >= 32 || lane < DV) {
    ldv<PV>(p.v + (long long)u * DV + lane * PV, r.v);
    ldv<PV>(p.vbar + ((long long)p.layer * p.H + h) * DV + lane * PV, r.vb);
  }
  r.gam_lo = r.gam_hi = 1.f;
  if constexpr (!KDA) {
    const int j0 = M2 ? lane : (lane & 15), j1 = 16 + (lane & 15);
    if (j0 < c) r.gam_lo = p.scale[unit * p.slen + j0];
    if (!M2 && j1 < c) r.gam_hi = p.scale[unit * p.slen + j1];
  }
  r.g = KDA ? 1.f : p.alpha[u];
  r.be = p.beta[u];
}

// Lane 0: the bulk copies of the c stored columns of U and of V of unit u into the
// stage (U at sU, V at sV, in their stored type TS), completing on bar.  A unit
// with an invalid column count gets no copies (the wait still ends).  A column is
// d_k (d_v) values of at least 2 bytes, d >= 16: every copy is a multiple of 16 bytes.
// withhold: announce the bytes but issue no copy (the injected wait fault).
template <int DK, int DV, typename TS>
SEED_DEV void issue_unit(const DecodeParams& p, TS* sU, TS* sV, uint64_t* bar, int u, int c, int m,
                         bool withhold = false) {
  const bool valid = c > 0 && c < m;
  mbar_arrive_expect_tx(bar, valid ? (uint32_t)(c * (DK + DV) * sizeof(TS)) : 0u);
  if (!valid || withhold) return;
  const long long unit = unit_index(p, u);
  bulk_g2s(sU, static_cast<const TS*>(p.U) + unit * (long long)m * DK, (uint32_t)(c * DK * sizeof(TS)), bar);
  bulk_g2s(sV, static_cast<const TS*>(p.V) + unit * (long long)m * DV, (uint32_t)(c * DV * sizeof(TS)), bar);
}

// Shared memory of one warp: the stage (U columns, then V columns, each sized for
// the R + W - 1 columns a unit can hold before a step), the column coefficients and
// the stage's mbarrier.
__host__ __device__ constexpr size_t warp_stage_bytes(int maxc, int dk, int dv, int elem) {
  return (size_t)maxc * (dk + dv) * elem;
}
constexpr int kCoefFloats = 2 * 32;
// The column coefficients of a stage of up to MAXC columns: a (q, k) pair each.
__host__ __device__ constexpr int coef_floats(int maxc) { return 2 * (maxc > 32 ? maxc : 32); }

// The body of both kernels below.  FUSE: after the step of a unit that brings it to
// R + W columns, the same warp compresses it in place (compress_fast_unit, panel
// tiles of MP columns) before it stages its next unit; its columns were staged a
// moment ago and are read again from L2.  The compression reuses the dynamic
// shared memory (the stage is idle then); the barriers live in static shared memory.
template <int FORM, int DK, int DV, int MAXC, typename TS, bool FUSE, int MP>
SEED_DEV void decode_warp_run(const DecodeParams& p, const FastParams* fp, const CUtensorMap* tmU,
                              const CUtensorMap* tmV) {
  using Vecs = UnitVecs<FORM, DK, DV>;
  constexpr bool KDA = FORM == SEED_KDA;
  constexpr bool M2 = FORM == SEED_MAMBA2;
  constexpr int PK = Vecs::PK, PV = Vecs::PV;
  constexpr int CPS = M2 ? 32 : 16;            // columns per warp reduction
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const int m = p.R + p.W;
  const int maxc = m - 1;
  TS* sU = reinterpret_cast<TS*>(smem_raw);
  TS* sV = sU + (size_t)maxc * DK;
  float* s_f = reinterpret_cast<float*>(smem_raw + warp_stage_bytes(maxc, DK, DV, sizeof(TS)));   // [32][2] (q, k)
  __shared__ __align__(8) uint64_t bars[3];   // the stage's; FUSE: the compression's two chunk barriers
  uint64_t* full = &bars[0];
  uint32_t cuses[2] = {0u, 0u};
  float* sA = reinterpret_cast<float*>(smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023));

  const int lane = threadIdx.x;
  const bool kact = DK >= 32 || lane < DK;
  const bool vact = DV >= 32 || lane < DV;
  const int n_units = p.B * p.H;
  const int stride = gridDim.x;
  const int u0 = blockIdx.x;
  if (lane == 0) {
    mbar_init(full, 1);
    if (FUSE) {
      mbar_init(&bars[1], 1);
      mbar_init(&bars[2], 1);
    }
    fence_mbar_init();
  }
  __syncwarp();

  // the first unit: its columns to the stage, its vectors to registers
  const bool fault = wait_fault_injected(p.status);
  int c = p.ncols[unit_index(p, u0)];
  if (lane == 0) issue_unit<DK, DV, TS>(p, sU, sV, full, u0, c, m, fault);
  // as in the ring kernel: an overlapped launch has read only this layer's stored
  // state so far; the step's inputs wait for the launch before it
  griddep_wait();
  griddep_launch_dependents();
  Vecs cur, nxt;
  load_vecs<FORM, DK, DV>(p, u0, c, cur);
  int c_next = u0 + stride < n_units ? p.ncols[unit_index(p, u0 + stride)] : 0;

  for (int i = 0, u = u0; u < n_units; ++i, u += stride) {
    const long long unit = unit_index(p, u);
    const int u_next = u + stride;
    // the next unit's vectors and the column count after it, while this one waits
    if (u_next < n_units) load_vecs<FORM, DK, DV>(p, u_next, c_next, nxt);
    const int c_after = u_next + stride < n_units ? p.ncols[unit_index(p, u_next + stride)] : 0;
    const float g = cur.g, be = cur.be;

    const uint64_t limit = (fault && i == 0) ? 0ull : kWaitLimitNs;
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(full, (uint32_t)i & 1u, limit))) {
      if (lane == 0) raise_flag(p.status, SEED_FLAG_TIMEOUT);
      mbar_wait_bounded(full, (uint32_t)i & 1u, kWaitLimitNs);   // let the copies land before exit
      return;
    }
    if (c < 0 || c >= m) {
      if (lane == 0) raise_flag(p.status, c == m ? SEED_FLAG_FULL : SEED_FLAG_BADCOLS);
    } else {
      // 1. dots of the stored U columns with q and k (KDA: with P+ (.) q and P+ (.) k,
      //    P+ = P (.) alpha, the dots of the decayed true columns)
      float kk[PK], qq[PK];
#pragma unroll
      for (int e = 0; e < PK; ++e) {
        const float pp = KDA ? cur.P[e] * cur.al[e] : 1.f;
        kk[e] = cur.k[e] * pp;
        qq[e] = cur.q[e] * pp;
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
          if (j < c && kact) fac_ld<TS, PK>(sU + j * DK + lane * PK, ue);
          dv[t] = dotv<PK>(ue, qq);
          if constexpr (!M2) dv[16 + t] = dotv<PK>(ue, kk);
        }
        const float tot = warp_xreduce<32>(dv);
        const int j = c0 + (M2 ? lane : (lane & 15));
        if (j < c) {
          // gamma_j: from registers for j < 32, from HBM (cached) above (stages of more
          // than 32 columns only)
          const float gj = (MAXC > 32 && c0 >= 32) ? p.scale[unit * p.slen + j] : (c0 == 0 ? cur.gam_lo : cur.gam_hi);
          const float f = KDA ? 1.f : g * gj;
          s_f[2 * j + (M2 ? 0 : (lane >> 4))] = f * tot;
        }
      }
      // 2. scalars: k^T a', a'^T q, k^T q (a' = alpha (.) a for KDA), v^T vbar, vbar^T vbar
      float sc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int e = 0; e < PK; ++e) {
        const float ae = KDA ? cur.al[e] * cur.a[e] : cur.a[e];
        sc[0] = fmaf(cur.k[e], ae, sc[0]);
        sc[1] = fmaf(ae, cur.q[e], sc[1]);
        sc[2] = fmaf(cur.k[e], cur.q[e], sc[2]);
      }
#pragma unroll
      for (int e = 0; e < PV; ++e) {
        sc[3] = fmaf(cur.v[e], cur.vb[e], sc[3]);
        sc[4] = fmaf(cur.vb[e], cur.vb[e], sc[4]);
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
          if (vact) fac_ld<TS, PV>(sV + j * DV + lane * PV, ve);
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
            const float eps = cur.v[e] - omega * cur.vb[e];
            ncol[e] = M2 ? be * eps : be * (eps - yk[e]);
            oe[e] = fmaf(cur.vb[e], apq, yq[e]) + ncol[e] * kq;
            bad |= !(isfinite(fac_round<TS>(ncol[e])) && isfinite(oe[e]));
          }
          fac_st<TS, PV>(static_cast<TS*>(p.V) + unit * (long long)m * DV + (long long)c * DV + lane * PV, ncol);
          stv<PV>(p.o + (long long)u * DV + lane * PV, oe);
        }
        if (kact) {
          float anew[PK], unew[PK], pn[PK];
#pragma unroll
          for (int e = 0; e < PK; ++e) {
            if constexpr (KDA) {
              pn[e] = cur.P[e] * cur.al[e];
              anew[e] = fmaf(cur.al[e], cur.a[e], coef * cur.k[e]);
              unew[e] = cur.k[e] / pn[e];
              bad |= !isfinite(fac_round<TS>(unew[e]));
            } else {
              anew[e] = fmaf(g, cur.a[e], coef * cur.k[e]);
              unew[e] = cur.k[e];
              bad |= !isfinite(fac_round<TS>(unew[e]));
            }
            bad |= !isfinite(anew[e]);
          }
          fac_st<TS, PK>(static_cast<TS*>(p.U) + unit * (long long)m * DK + (long long)c * DK + lane * PK, unew);
          stv<PK>(p.a + unit * DK + lane * PK, anew);
          if constexpr (KDA) stv<PK>(p.scale + unit * DK + lane * PK, pn);
        }
        if constexpr (!KDA) {
          // gamma_j of column j = lane: gam_lo for lanes < 16 (and every lane for
          // Mamba-2), gam_hi above; the new column's scale is 1
          const float gl = (M2 || lane < 16) ? cur.gam_lo : cur.gam_hi;
          for (int j = lane; j <= c; j += 32)
            p.scale[unit * p.slen + j] = j < c ? g * ((MAXC > 32 && j >= 32) ? p.scale[unit * p.slen + j] : gl) : 1.f;
        }
        if (lane == 0) p.ncols[unit] = c + 1;
        if (__any_sync(0xffffffffu, bad) && lane == 0) raise_flag(p.status, SEED_FLAG_NONFINITE);
      }
    }
    // every read of the stage (and of s_f) is above and complete (its values were
    // consumed); only bulk copies write the stage, so no proxy fence is needed
    __syncwarp();
    if constexpr (FUSE) {
      if (c + 1 == m) {   // due (compress_fast_unit checks the count the step wrote)
        fence_proxy_async_global();   // the new pair and the scales, before the tensor copies
        __syncwarp();
        if (!compress_fast_unit<FORM, DK, DV, MP, TS>(*fp, *tmU, *tmV, u, sA, &bars[1], cuses)) return;
        fence_proxy_async_smem();     // the compression wrote the stage's memory
        __syncwarp();
      }
    }
    if (lane == 0 && u_next < n_units) issue_unit<DK, DV, TS>(p, sU, sV, full, u_next, c_next, m);
    cur = nxt;
    c = c_next;
    c_next = c_after;
  }
}

}  // namespace seed
