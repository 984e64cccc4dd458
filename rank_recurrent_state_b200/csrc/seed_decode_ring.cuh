// seed_decode_ring.cuh -- the decode step with one warp per unit and a ring of
// column chunks, for R + W <= 65.
//
// "Shallow Encoding Emits Deep Memories", SEED summary (picx.dev), "Exact Update
// (Lemma 2)" with the sink recurrence of Lemma 1, and the read-out o = S+^T q; the
// arithmetic is that of seed_decode_warp.cuh, the data movement different.
//
// The step is HBM-bound: the stored columns of U and V must stream through every SM
// without pause.  A warp owns a ring of NSLOT shared-memory slots of 8 columns each.
// A unit's columns go through it as chunks -- its U chunks, then its V chunks -- and
// lane 0 refills a slot as soon as the warp has read it, with the next chunk of the
// warp's sequence, which after the current unit's last chunk belongs to the warp's
// next unit (one TMA bulk copy per chunk, completion on the slot's mbarrier, no
// multicast).  So up to NSLOT chunks of every warp are in flight whatever the warp is
// computing, and a slot costs a quarter of a whole-unit stage: twice the warps share
// an SM.  Per unit the warp computes:
//   1. per U chunk, U^T q and U^T k for its 8 columns (partial dots over the lane's
//      rows, summed over the warp by a transposed reduction), scaled into the columns'
//      coefficients g gamma_j (U^T q)_j, g gamma_j (U^T k)_j;
//   2. the scalars k^T a, a^T q, k^T q, v^T vbar, vbar^T vbar;
//   3. per V chunk, y_k = V (coefficients of k) and y_q = V (coefficients of q), each
//      lane for its own rows;
//   4. the sink update, the new column pair and the read-out, written from registers.
// The per-unit vectors (k, q, a, v, vbar, the decay scales, g, beta) go from HBM to
// each lane's registers with coalesced loads one unit ahead.  16-bit factors travel
// and sit in the slots as stored and are widened as they are read (the library
// launches this kernel for float32 factors; 16-bit factors decode with the whole-unit
// stage of seed_decode_warp.cu, which costs fewer instructions per byte).
#pragma once

#include "seed_common.cuh"
#include "seed_decode.cuh"
#include "seed_launch.h"
#include "seed_tma.cuh"

namespace seed {

constexpr int kRingChunk = 8;   // columns per chunk

// The per-unit vectors one lane needs, in registers: its d_k / 32 rows of k, q, a
// (KDA: alpha, P) and d_v / 32 rows of v, vbar; the decay scales gamma_j of columns
// j = lane and j = 32 + lane; and the unit's g (alpha) and beta.
template <int FORM, int DK, int DV>
struct RingVecs {
  static constexpr int PK = DK >= 32 ? DK / 32 : 1, PV = DV >= 32 ? DV / 32 : 1;
  float k[PK], q[PK], a[PK], al[PK], P[PK], v[PV], vb[PV];
  float gam_lo, gam_hi, g, be;
};

template <int P>
SEED_DEV void ring_ldv(const float* p, float (&e)[P]) {
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
SEED_DEV void ring_stv(float* p, const float (&e)[P]) {
  if constexpr (P == 4) {
    st4(p, make_float4(e[0], e[1], e[2], e[3]));
  } else if constexpr (P == 2) {
    *reinterpret_cast<float2*>(p) = make_float2(e[0], e[1]);
  } else {
    *p = e[0];
  }
}

template <int P>
SEED_DEV float ring_dot(const float (&a)[P], const float (&b)[P]) {
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < P; ++e) s = fmaf(a[e], b[e], s);
  return s;
}

SEED_DEV long long ring_unit(const DecodeParams& p, int u) {
  const int b = u / p.H, h = u - b * p.H;
  return ((long long)b * p.L + p.layer) * p.H + h;
}

template <int FORM, int DK, int DV, int MAXC>
SEED_DEV void ring_load_vecs(const DecodeParams& p, int u, int c, RingVecs<FORM, DK, DV>& r) {
  constexpr bool KDA = FORM == SEED_KDA;
  constexpr int PK = RingVecs<FORM, DK, DV>::PK, PV = RingVecs<FORM, DK, DV>::PV;
  const int lane = threadIdx.x & 31;
  const long long unit = ring_unit(p, u);
  const int h = u % p.H;
#pragma unroll
  for (int e = 0; e < PK; ++e) r.k[e] = r.q[e] = r.a[e] = 0.f, r.al[e] = r.P[e] = 1.f;
#pragma unroll
  for (int e = 0; e < PV; ++e) r.v[e] = r.vb[e] = 0.f;
  if (DK >= 32 || lane < DK) {
    ring_ldv<PK>(p.k + (long long)u * DK + lane * PK, r.k);
    ring_ldv<PK>(p.q + (long long)u * DK + lane * PK, r.q);
    ring_ldv<PK>(p.a + unit * DK + lane * PK, r.a);
    if constexpr (KDA) {
      ring_ldv<PK>(p.alpha + (long long)u * DK + lane * PK, r.al);
      ring_ldv<PK>(p.scale + unit * DK + lane * PK, r.P);
    }
  }
  if (DV >= 32 || lane < DV) {
    ring_ldv<PV>(p.v + (long long)u * DV + lane * PV, r.v);
    ring_ldv<PV>(p.vbar + ((long long)p.layer * p.H + h) * DV + lane * PV, r.vb);
  }
  r.gam_lo = r.gam_hi = 1.f;
  if constexpr (!KDA) {
    if (lane < c) r.gam_lo = p.scale[unit * p.slen + lane];
    if (MAXC > 32 && 32 + lane < c) r.gam_hi = p.scale[unit * p.slen + 32 + lane];
  }
  r.g = KDA ? 1.f : p.alpha[u];
  r.be = p.beta[u];
}

// Chunks of a unit holding c columns: ceil(c / 8) of U then as many of V; none for a
// count outside [1, m - 1] (an empty, full or invalid unit).
SEED_DEV int ring_chunks(int c, int m) { return (c > 0 && c < m) ? 2 * ((c + kRingChunk - 1) / kRingChunk) : 0; }

// Lane 0: chunk kidx of unit u (c columns) into slot `slot`, completing on bar.
// withhold: announce the bytes but issue no copy (the injected wait fault).
template <int DK, int DV, typename TS, int SLOT>
SEED_DEV void ring_issue(const DecodeParams& p, TS* slots, uint64_t* bars, int slot, int u, int c, int m, int kidx,
                         bool withhold) {
  const int n = (c + kRingChunk - 1) / kRingChunk;
  const bool isV = kidx >= n;
  const int col0 = (isV ? kidx - n : kidx) * kRingChunk;
  const int ncol = c - col0 < kRingChunk ? c - col0 : kRingChunk;
  const int D = isV ? DV : DK;
  const uint32_t bytes = (uint32_t)(ncol * D * sizeof(TS));
  const long long unit = ring_unit(p, u);
  const TS* src = static_cast<const TS*>(isV ? p.V : p.U) + (unit * (long long)m + col0) * D;
  mbar_arrive_expect_tx(&bars[slot], bytes);
  if (!withhold) bulk_g2s(slots + (size_t)slot * SLOT, src, bytes, &bars[slot]);
}

template <int FORM, int DK, int DV, int MAXC, int NSLOT, typename TS>
SEED_DEV void decode_ring_run(const DecodeParams& p) {
  using Vecs = RingVecs<FORM, DK, DV>;
  constexpr bool KDA = FORM == SEED_KDA;
  constexpr bool M2 = FORM == SEED_MAMBA2;
  constexpr int PK = Vecs::PK, PV = Vecs::PV;
  constexpr int CH = kRingChunk;
  constexpr int SLOT = CH * (DK > DV ? DK : DV);   // elements of one slot
  extern __shared__ __align__(128) unsigned char smem_raw[];
  TS* slots = reinterpret_cast<TS*>(smem_raw);
  float* s_f = reinterpret_cast<float*>(smem_raw + (size_t)NSLOT * SLOT * sizeof(TS));   // [MAXC][2] (q, k)
  __shared__ __align__(8) uint64_t bars[NSLOT];
  const int m = p.R + p.W;
  const int lane = threadIdx.x;
  const bool kact = DK >= 32 || lane < DK;
  const bool vact = DV >= 32 || lane < DV;
  const int n_units = p.B * p.H;
  const int stride = gridDim.x;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < NSLOT; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const bool fault = wait_fault_injected(p.status);

  // unit i of this warp is u0 + i stride; chunk sequence numbers run over the warp's
  // units in order: the current unit's chunks are [base, base + n_cur), the next
  // unit's follow.  Slot of chunk s: s % NSLOT, phase (s / NSLOT) & 1.
  int u = blockIdx.x;
  int c_cur = u < n_units ? p.ncols[ring_unit(p, u)] : 0;
  int c_nxt = u + stride < n_units ? p.ncols[ring_unit(p, u + stride)] : 0;
  int n_cur = ring_chunks(c_cur, m), n_nxt = u + stride < n_units ? ring_chunks(c_nxt, m) : 0;
  int base = 0, issued = 0, consumed = 0;
  auto fill = [&]() {
    while (issued < consumed + NSLOT) {
      int uu, cc, kk;
      if (issued < base + n_cur) {
        uu = u, cc = c_cur, kk = issued - base;
      } else if (issued < base + n_cur + n_nxt) {
        uu = u + stride, cc = c_nxt, kk = issued - base - n_cur;
      } else {
        break;
      }
      if (lane == 0)
        ring_issue<DK, DV, TS, SLOT>(p, slots, bars, issued % NSLOT, uu, cc, m, kk, fault && issued == 0);
      ++issued;
    }
  };
  // the bounded wait for chunk `consumed`; on a timeout, waits (bounded) for the
  // chunks still in flight and reports false
  auto wait_chunk = [&]() -> bool {
    const uint64_t limit = (fault && consumed == 0) ? 0ull : kWaitLimitNs;
    if (__all_sync(0xffffffffu, mbar_wait_bounded(&bars[consumed % NSLOT], (uint32_t)(consumed / NSLOT) & 1u, limit)))
      return true;
    if (lane == 0) raise_flag(p.status, SEED_FLAG_TIMEOUT);
    for (int s = consumed; s < issued; ++s)
      mbar_wait_bounded(&bars[s % NSLOT], (uint32_t)(s / NSLOT) & 1u, kWaitLimitNs);
    return false;
  };
  fill();
  // Up to here the launch has read only this layer's stored state (column counts, and
  // the first chunks now in flight).  An overlapped launch (seed_decode_step_overlapped)
  // may have begun while the launch before it on the stream was still running, which
  // by the caller's guarantee writes none of that state but may write this step's
  // inputs: everything else waits for it.  Then the next launch may begin.
  griddep_wait();
  griddep_launch_dependents();

  Vecs cur, nxt;
  if (u < n_units) ring_load_vecs<FORM, DK, DV, MAXC>(p, u, c_cur, cur);

  while (u < n_units) {
    const long long unit = ring_unit(p, u);
    const int u_next = u + stride;
    // the next unit's vectors and the column count two units ahead, while this one runs
    if (u_next < n_units) ring_load_vecs<FORM, DK, DV, MAXC>(p, u_next, c_nxt, nxt);
    const int c_aft = u_next + stride < n_units ? p.ncols[ring_unit(p, u_next + stride)] : 0;
    const int c = c_cur;
    const float g = cur.g, be = cur.be;
    const int nch = n_cur / 2;

    if (c < 0 || c >= m) {
      if (lane == 0) raise_flag(p.status, c == m ? SEED_FLAG_FULL : SEED_FLAG_BADCOLS);
    } else {
      // 1. U^T q and U^T k, chunk by chunk (KDA: with P+ (.) q and P+ (.) k, the dots of
      //    the decayed true columns), into the columns' (q, k) coefficients
      float kk[PK], qq[PK];
#pragma unroll
      for (int e = 0; e < PK; ++e) {
        const float pp = KDA ? cur.P[e] * cur.al[e] : 1.f;
        kk[e] = cur.k[e] * pp;
        qq[e] = cur.q[e] * pp;
      }
      for (int ch = 0; ch < nch; ++ch) {
        if (!wait_chunk()) return;
        const TS* sU = slots + (size_t)(consumed % NSLOT) * SLOT;
        const int j0 = ch * CH;
        constexpr int NV = M2 ? CH : 2 * CH;
        float dv[NV];
#pragma unroll
        for (int t = 0; t < CH; ++t) {
          float ue[PK];
#pragma unroll
          for (int e = 0; e < PK; ++e) ue[e] = 0.f;
          if (j0 + t < c && kact) fac_ld<TS, PK>(sU + t * DK + lane * PK, ue);
          dv[t] = ring_dot<PK>(ue, qq);
          if constexpr (!M2) dv[CH + t] = ring_dot<PK>(ue, kk);
        }
        const float tot = warp_xreduce<NV>(dv);
        // lane l holds value (l >> (5 - log2 NV)): column j0 + (that & 7), q or k
        const int vi = lane >> (5 - log2c<NV>());
        const int j = j0 + (vi & (CH - 1));
        const float gj = __shfl_sync(0xffffffffu, j0 < 32 ? cur.gam_lo : cur.gam_hi, j & 31);
        if (j < c && (lane & ((1 << (5 - log2c<NV>())) - 1)) == 0)
          s_f[2 * j + (M2 ? 0 : vi / CH)] = (KDA ? 1.f : g * gj) * tot;
        __syncwarp();   // every lane has read the slot
        ++consumed;
        fill();
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
      // 3. y_k = V (g gamma (.) U^T k) for the erase, y_q = V (g gamma (.) U^T q) for
      //    the read-out (decayed true columns); each lane its own rows
      float yk[PV], yq[PV];
#pragma unroll
      for (int e = 0; e < PV; ++e) yk[e] = yq[e] = 0.f;
      for (int ch = 0; ch < nch; ++ch) {
        if (!wait_chunk()) return;
        const TS* sV = slots + (size_t)(consumed % NSLOT) * SLOT;
        const int j0 = ch * CH;
#pragma unroll
        for (int t = 0; t < CH; ++t) {
          const int j = j0 + t;
          if (j < c) {
            float ve[PV];
#pragma unroll
            for (int e = 0; e < PV; ++e) ve[e] = 0.f;
            if (vact) fac_ld<TS, PV>(sV + t * DV + lane * PV, ve);
            const float2 f2 = *reinterpret_cast<const float2*>(s_f + 2 * j);   // (q, k) coefficients
#pragma unroll
            for (int e = 0; e < PV; ++e) {
              if constexpr (!M2) yk[e] = fmaf(f2.y, ve[e], yk[e]);
              yq[e] = fmaf(f2.x, ve[e], yq[e]);
            }
          }
        }
        __syncwarp();   // every lane has read the slot
        ++consumed;
        fill();
      }
      if (!(vbvb > 0.f)) {
        if (lane == 0) raise_flag(p.status, SEED_FLAG_ZERO_VBAR);
      } else {
        const float omega = vvb / vbvb;
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
          ring_stv<PV>(p.o + (long long)u * DV + lane * PV, oe);
        }
        if (kact) {
          float anew[PK], unew[PK], pn[PK];
#pragma unroll
          for (int e = 0; e < PK; ++e) {
            if constexpr (KDA) {
              pn[e] = cur.P[e] * cur.al[e];
              anew[e] = fmaf(cur.al[e], cur.a[e], coef * cur.k[e]);
              unew[e] = cur.k[e] / pn[e];
            } else {
              anew[e] = fmaf(g, cur.a[e], coef * cur.k[e]);
              unew[e] = cur.k[e];
            }
            bad |= !isfinite(fac_round<TS>(unew[e]));
            bad |= !isfinite(anew[e]);
          }
          fac_st<TS, PK>(static_cast<TS*>(p.U) + unit * (long long)m * DK + (long long)c * DK + lane * PK, unew);
          ring_stv<PK>(p.a + unit * DK + lane * PK, anew);
          if constexpr (KDA) ring_stv<PK>(p.scale + unit * DK + lane * PK, pn);
        }
        if constexpr (!KDA) {
          // column j (lane, 32 + lane, ...): decayed by g; the new column's scale is 1
          for (int j = lane; j <= c; j += 32)
            p.scale[unit * p.slen + j] = j < c ? g * (j < 32 ? cur.gam_lo : cur.gam_hi) : 1.f;
        }
        if (lane == 0) p.ncols[unit] = c + 1;
        if (__any_sync(0xffffffffu, bad) && lane == 0) raise_flag(p.status, SEED_FLAG_NONFINITE);
      }
    }
    // the next unit: its chunks follow this unit's in the sequence.  u moves on before
    // the ring is refilled: fill() names the current unit u and the next u + stride
    base += n_cur;
    n_cur = n_nxt;
    c_cur = c_nxt;
    c_nxt = c_aft;
    n_nxt = u_next + stride < n_units ? ring_chunks(c_aft, m) : 0;
    cur = nxt;
    u = u_next;
    fill();
  }
}

}  // namespace seed
