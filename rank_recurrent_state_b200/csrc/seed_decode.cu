// seed_decode.cu -- the fused decode step of the sink-plus-low-rank state.
//
// "Shallow Encoding Emits Deep Memories", SEED summary (picx.dev), "Exact Update
// (Lemma 2)" with the sink recurrence of Lemma 1, and the read-out o = S+^T q.
//
// The step is HBM-bound: each (request, head) unit reads its c stored columns of
// U and V once and writes back only the touched bytes (the sink a, one new column
// of U and of V, the decay scales, the column count).  The kernel is persistent
// and warp-specialised: in each CTA one producer warp streams units through a
// ring of shared-memory stages with TMA bulk copies (cp.async.bulk, completion on
// an mbarrier, no multicast), and four consumer warps compute each unit from
// shared memory and hand the stage back through a second mbarrier.  The producer
// runs NS units ahead, so every SM keeps several units' panels in flight.
//
// Lazy decay.  Gated DeltaNet and Mamba-2 scale every old U column by the same
// scalar per step; instead of rewriting U the kernel keeps per-column scales
// gamma_j (true column = gamma_j * stored column) and updates only those.  KDA's
// decay is per channel (a row scaling of U), kept as a per-unit running product
// P (true U = Diag(P) * stored U); the new column is stored as k / P so that its
// true value is k.  Both are folded back into U by the compression.
#include "seed_common.cuh"
#include "seed_decode.cuh"
#include "seed_launch.h"
#include "seed_tma.cuh"

namespace seed {

constexpr int kConsumerWarps = 4;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;

SEED_DEV void consumer_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Barrier over the consumer warps that also ANDs a predicate across them.
SEED_DEV bool consumer_and(bool v) {
  uint32_t out;
  asm volatile(
      "{\n .reg .pred pi, po;\n setp.ne.u32 pi, %1, 0;\n bar.red.and.pred po, 1, 128, pi;\n"
      " selp.u32 %0, 1, 0, po;\n}"
      : "=r"(out)
      : "r"((uint32_t)v)
      : "memory");
  return out != 0;
}

template <int FORM, int DK, int DV, int MAXC, int NS, typename TS>
__global__ void __launch_bounds__(kDecodeThreads) decode_step_kernel(const DecodeParams p) {
  using Stage = DecodeStage<FORM, DK, DV, MAXC, TS>;
  constexpr int NW = kConsumerWarps;
  constexpr int NT = NW * 32;
  constexpr int LK = DK / 4;            // lanes per U column (float4 each)
  constexpr int CPK = 32 / LK;          // U columns per warp pass
  constexpr int GK = NW * CPK;          // U column groups
  constexpr int CU = (MAXC + GK - 1) / GK;
  constexpr int LV = DV / 4;
  constexpr int CPV = 32 / LV;
  constexpr int GV = NW * CPV;
  constexpr int CV = (MAXC + GV - 1) / GV;
  constexpr bool KDA = FORM == SEED_KDA;
  constexpr bool M2 = FORM == SEED_MAMBA2;
  constexpr int NDOT = M2 ? 1 : 2;      // dots per U column: with q, and with k for the erase

  extern __shared__ __align__(128) unsigned char smem_raw[];
  Stage* stages = reinterpret_cast<Stage*>(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw + NS * sizeof(Stage));
  uint64_t* empty = full + NS;
  __shared__ float s_dk[MAXC];
  __shared__ float s_dq[MAXC];
  __shared__ __align__(16) float s_yk[NW][DV];
  __shared__ __align__(16) float s_yq[NW][DV];
  __shared__ float s_red[NW][8];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n_units = p.B * p.H;
  const int m = p.R + p.W;
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  // ------------------------------------------------------------------ producer warp
  if (warp == NW) {
    if (lane != 0) return;
    int u = blockIdx.x;
    int c_next = 0;
    float g_next = 0.f, b_next = 0.f;
    if (u < n_units) {
      const long long un = ((long long)(u / p.H) * p.L + p.layer) * p.H + (u % p.H);
      c_next = p.ncols[un];
      g_next = KDA ? 1.f : p.alpha[u];
      b_next = p.beta[u];
    }
    for (int i = 0; u < n_units; u += gridDim.x, ++i) {
      const int s = i % NS;
      const uint32_t ph = (uint32_t)(i / NS) & 1u;
      const int b = u / p.H, h = u - (u / p.H) * p.H;
      const long long unit = ((long long)b * p.L + p.layer) * p.H + h;
      const int c = c_next;
      const float g = g_next, be = b_next;
      const int u2 = u + gridDim.x;
      if (u2 < n_units) {   // prefetch the next unit's scalars while this one is issued
        const long long un = ((long long)(u2 / p.H) * p.L + p.layer) * p.H + (u2 % p.H);
        c_next = p.ncols[un];
        g_next = KDA ? 1.f : p.alpha[u2];
        b_next = p.beta[u2];
      }
      if (i >= NS && !mbar_wait_bounded(&empty[s], ph ^ 1u, kWaitLimitNs)) {
        raise_flag(p.status, SEED_FLAG_TIMEOUT);
        return;
      }
      Stage& S = stages[s];
      S.c = c;
      S.g = g;
      S.beta = be;
      const bool valid = c >= 0 && c < m;
      uint32_t bytes = 0;
      if (valid) {
        bytes = (uint32_t)(c * (DK + DV) * sizeof(TS)) + (uint32_t)(3 * DK + 2 * DV) * 4u;
        bytes += KDA ? 2u * DK * 4u : (uint32_t)((c + 3) & ~3) * 4u;
      }
      mbar_arrive_expect_tx(&full[s], bytes);
      if (valid) {
        if (c > 0) {
          bulk_g2s(S.U, static_cast<const TS*>(p.U) + unit * (long long)m * DK, (uint32_t)(c * DK * sizeof(TS)),
                   &full[s]);
          bulk_g2s(S.V, static_cast<const TS*>(p.V) + unit * (long long)m * DV, (uint32_t)(c * DV * sizeof(TS)),
                   &full[s]);
        }
        bulk_g2s(S.a, p.a + unit * DK, DK * 4, &full[s]);
        bulk_g2s(S.k, p.k + (long long)u * DK, DK * 4, &full[s]);
        bulk_g2s(S.q, p.q + (long long)u * DK, DK * 4, &full[s]);
        bulk_g2s(S.v, p.v + (long long)u * DV, DV * 4, &full[s]);
        bulk_g2s(S.vb, p.vbar + ((long long)p.layer * p.H + h) * DV, DV * 4, &full[s]);
        if constexpr (KDA) {
          bulk_g2s(S.al, p.alpha + (long long)u * DK, DK * 4, &full[s]);
          bulk_g2s(S.P, p.scale + unit * DK, DK * 4, &full[s]);
        } else if (c > 0) {
          bulk_g2s(S.gam, p.scale + unit * p.slen, (uint32_t)((c + 3) & ~3) * 4u, &full[s]);
        }
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumer warps
  const int gk = warp * CPK + lane / LK, lk = lane % LK;
  const int gv = warp * CPV + lane / LV, lv = lane % LV;
  for (int i = 0, u = blockIdx.x; u < n_units; u += gridDim.x, ++i) {
    const int s = i % NS;
    const uint32_t ph = (uint32_t)(i / NS) & 1u;
    if (!consumer_and(mbar_wait_bounded(&full[s], ph, kWaitLimitNs))) {
      if (tid == 0) raise_flag(p.status, SEED_FLAG_TIMEOUT);
      mbar_wait_bounded(&full[s], ph, kWaitLimitNs);   // let copies in flight land
      return;
    }
    const Stage& S = stages[s];
    const int b = u / p.H, h = u - (u / p.H) * p.H;
    const long long unit = ((long long)b * p.L + p.layer) * p.H + h;
    const int c = S.c;
    const float g = S.g, be = S.beta;
    bool skip = false;
    if (c < 0 || c >= m) {
      if (tid == 0) raise_flag(p.status, c == m ? SEED_FLAG_FULL : SEED_FLAG_BADCOLS);
      skip = true;
    }
    if (!skip) {
      // 1. dots of the stored U columns with k and q (KDA: with P+ (.) k, P+ (.) q,
      //    P+ = P (.) alpha, the dots of the decayed true columns)
      float4 kk = ld4(S.k + 4 * lk), qq = ld4(S.q + 4 * lk);
      if constexpr (KDA) {
        const float4 pp = mul4(ld4(S.P + 4 * lk), ld4(S.al + 4 * lk));
        kk = mul4(kk, pp);
        qq = mul4(qq, pp);
      }
      float dv[NDOT * CU];
#pragma unroll
      for (int r = 0; r < CU; ++r) {
        const int j = gk + GK * r;
        const float4 uc = j < c ? fac_ld4(S.U + j * DK + 4 * lk) : zero4();
        dv[r] = dot4(uc, qq);
        if constexpr (!M2) dv[CU + r] = dot4(uc, kk);
      }
      if constexpr (LK == 32 && ((NDOT * CU) & (NDOT * CU - 1)) == 0) {
        constexpr int NV = NDOT * CU;
        const float tot = warp_xreduce<NV>(dv);
        constexpr int SH = 5 - log2c<NV>();
        if ((lane & ((1 << SH) - 1)) == 0) {
          const int idx = (lane >> SH) & (NV - 1);
          const int r = idx % CU;
          const int j = gk + GK * r;
          if (j < c) {
            if (idx < CU) s_dq[j] = tot;
            else s_dk[j] = tot;
          }
        }
      } else {
#pragma unroll
        for (int r = 0; r < NDOT * CU; ++r) dv[r] = group_sum<LK>(dv[r]);
        if (lk == 0) {
#pragma unroll
          for (int r = 0; r < CU; ++r) {
            const int j = gk + GK * r;
            if (j < c) {
              s_dq[j] = dv[r];
              if constexpr (!M2) s_dk[j] = dv[CU + r];
            }
          }
        }
      }
      // scalars: k^T a', a'^T q, k^T q (a' = alpha (.) a for KDA), v^T vbar, vbar^T vbar
      float sc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int e = tid; e < DK; e += NT) {
        const float ae = KDA ? S.al[e] * S.a[e] : S.a[e];
        sc[0] = fmaf(S.k[e], ae, sc[0]);
        sc[1] = fmaf(ae, S.q[e], sc[1]);
        sc[2] = fmaf(S.k[e], S.q[e], sc[2]);
      }
      for (int e = tid; e < DV; e += NT) {
        sc[3] = fmaf(S.v[e], S.vb[e], sc[3]);
        sc[4] = fmaf(S.vb[e], S.vb[e], sc[4]);
      }
      {
        const float tot = warp_xreduce<8>(sc);
        if ((lane & 3) == 0) s_red[warp][(lane >> 2) & 7] = tot;
      }
      consumer_sync();
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
        skip = true;
      }
      if (!skip) {
        const float omega = vvb / vbvb;
        // 2. V times the column coefficients: y_k = V (g gamma (.) U^T k) for the
        //    erase, y_q = V (g gamma (.) U^T q) for the read-out (decayed true columns)
        float4 yk = zero4(), yq = zero4();
#pragma unroll
        for (int r = 0; r < CV; ++r) {
          const int j = gv + GV * r;
          if (j < c) {
            const float4 vc = fac_ld4(S.V + j * DV + 4 * lv);
            const float f = KDA ? 1.f : g * S.gam[j];
            if constexpr (!M2) yk = fma4(f * s_dk[j], vc, yk);
            yq = fma4(f * s_dq[j], vc, yq);
          }
        }
#pragma unroll
        for (int off = LV; off < 32; off <<= 1) {
          if constexpr (!M2) {
            yk.x += __shfl_xor_sync(0xffffffffu, yk.x, off);
            yk.y += __shfl_xor_sync(0xffffffffu, yk.y, off);
            yk.z += __shfl_xor_sync(0xffffffffu, yk.z, off);
            yk.w += __shfl_xor_sync(0xffffffffu, yk.w, off);
          }
          yq.x += __shfl_xor_sync(0xffffffffu, yq.x, off);
          yq.y += __shfl_xor_sync(0xffffffffu, yq.y, off);
          yq.z += __shfl_xor_sync(0xffffffffu, yq.z, off);
          yq.w += __shfl_xor_sync(0xffffffffu, yq.w, off);
        }
        if (lane < LV) {
          if constexpr (!M2) st4(&s_yk[warp][4 * lane], yk);
          st4(&s_yq[warp][4 * lane], yq);
        }
        consumer_sync();

        // 3. sink update, new column pair, read-out
        float coef;   // a+ = a' + coef * k   (a' = g a, alpha (.) a, alpha a)
        if constexpr (FORM == SEED_GDN) coef = be * (omega - g * ka);
        else if constexpr (KDA) coef = be * (omega - ka);
        else coef = be * omega;
        const float apq = (KDA ? aq : g * aq) + coef * kq;   // a+^T q
        bool bad = false;
        TS* Vnew = static_cast<TS*>(p.V) + unit * (long long)m * DV + (long long)c * DV;
        TS* Unew = static_cast<TS*>(p.U) + unit * (long long)m * DK + (long long)c * DK;
        for (int e = tid; e < DV; e += NT) {
          float yke = 0.f, yqe = 0.f;
#pragma unroll
          for (int w = 0; w < NW; ++w) {
            if constexpr (!M2) yke += s_yk[w][e];
            yqe += s_yq[w][e];
          }
          const float eps = S.v[e] - omega * S.vb[e];
          const float ncol = M2 ? be * eps : be * (eps - yke);
          const float oe = fmaf(S.vb[e], apq, yqe) + ncol * kq;
          bad |= !(isfinite(fac_round<TS>(ncol)) && isfinite(oe));
          Vnew[e] = fac_from_f<TS>(ncol);
          p.o[(long long)u * DV + e] = oe;
        }
        for (int e = tid; e < DK; e += NT) {
          const float ae = S.a[e];
          const float ke = S.k[e];
          float anew;
          if constexpr (KDA) {
            const float pn = S.P[e] * S.al[e];
            anew = fmaf(S.al[e], ae, coef * ke);
            const float us = ke / pn;
            bad |= !isfinite(fac_round<TS>(us));
            Unew[e] = fac_from_f<TS>(us);
            p.scale[unit * DK + e] = pn;
          } else {
            anew = fmaf(g, ae, coef * ke);
            bad |= !isfinite(fac_round<TS>(ke));
            Unew[e] = fac_from_f<TS>(ke);
          }
          bad |= !isfinite(anew);
          p.a[unit * DK + e] = anew;
        }
        if constexpr (!KDA) {
          for (int j = tid; j <= c; j += NT) p.scale[unit * p.slen + j] = j < c ? g * S.gam[j] : 1.f;
        }
        if (tid == 0) p.ncols[unit] = c + 1;
        if (bad) raise_flag(p.status, SEED_FLAG_NONFINITE);
      }
    }
    // hand the stage back to the producer (every consumer read of S is above)
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

template <int FORM, int DK, int DV, int MAXC, typename TS>
static int launch_one(const DecodeParams& p, cudaStream_t st) {
  using Stage = DecodeStage<FORM, DK, DV, MAXC, TS>;
  // stages: as many as fit in ~108 KB so that two CTAs share an SM, at least two
  constexpr int NS0 = (int)((108 * 1024) / sizeof(Stage));
  constexpr int NS = NS0 < 2 ? 2 : (NS0 > 6 ? 6 : NS0);
  const size_t smem = NS * sizeof(Stage) + 2 * NS * sizeof(uint64_t);
  auto kern = decode_step_kernel<FORM, DK, DV, MAXC, NS, TS>;
  // per device: the shared-memory opt-in and the resident CTAs per SM
  static LaunchCache cache;
  static std::atomic<int> grid_per_sm[kMaxDev];
  int dev = 0;
  if (const int rc = cache.prepare(reinterpret_cast<const void*>(kern), smem, &dev)) return rc;
  int per_sm = grid_per_sm[dev].load(std::memory_order_relaxed);
  if (per_sm == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kDecodeThreads, smem) != cudaSuccess)
      return SEED_ERR_CUDA;
    per_sm = n > 0 ? n : 1;
    grid_per_sm[dev].store(per_sm, std::memory_order_relaxed);
  }
  const int units = p.B * p.H;
  int grid = per_sm * cache.sm_count[dev].load(std::memory_order_relaxed);
  if (grid > units) grid = units;
  kern<<<grid, kDecodeThreads, smem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
}

// Up to 64 stored columns: one warp per unit (float32 factors through a ring of
// column chunks, seed_decode_ring.cu; 16-bit factors with a whole-unit stage,
// seed_decode_warp.cu); above (up to SEED_MAX_COLS - 1), this kernel with four
// consumer warps per unit.
template <int FORM, int DK, int DV, typename TS>
static int launch_cols_t(const DecodeParams& p, cudaStream_t st) {
  return launch_one<FORM, DK, DV, 96, TS>(p, st);
}

template <int FORM, int DK, int DV>
static int launch_cols(const DecodeParams& p, int factors, cudaStream_t st) {
  if (p.R + p.W - 1 <= 64)
    return factors == SEED_FACTORS_F32 ? launch_decode_ring(p, FORM, DK, DV, factors, st)
                                       : launch_decode_warp16(p, FORM, DK, DV, factors, st);
  switch (factors) {
    case SEED_FACTORS_F32: return launch_cols_t<FORM, DK, DV, float>(p, st);
    case SEED_FACTORS_F16: return launch_cols_t<FORM, DK, DV, __half>(p, st);
    case SEED_FACTORS_BF16: return launch_cols_t<FORM, DK, DV, __nv_bfloat16>(p, st);
  }
  return SEED_ERR_INVALID_ARG;
}

template <int FORM>
static int launch_dims(const DecodeParams& p, int dk, int dv, int factors, cudaStream_t st) {
#define SEED_DIMS_CASE(K, V) \
  if (dk == K && dv == V) return launch_cols<FORM, K, V>(p, factors, st);
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
                       float* o, uint32_t* status, cudaStream_t st, bool overlap) {
  DecodeParams p{q, k, v, alpha, beta, o, s.a, s.U, s.V, s.scale, s.ncols, s.vbar, status,
                 d.batch, d.layers, d.heads, layer, d.R, d.W, scale_len(d), overlap ? 1 : 0};
  switch (d.form) {
    case SEED_GDN: return launch_dims<SEED_GDN>(p, d.d_k, d.d_v, d.factors, st);
    case SEED_KDA: return launch_dims<SEED_KDA>(p, d.d_k, d.d_v, d.factors, st);
    case SEED_MAMBA2: return launch_dims<SEED_MAMBA2>(p, d.d_k, d.d_v, d.factors, st);
  }
  return SEED_ERR_INVALID_ARG;
}

bool decode_dims_supported(int dk, int dv) {
  return (dk == dv && (dk == 16 || dk == 32 || dk == 64 || dk == 128)) ||
         (dk == 128 && dv == 64) || (dk == 64 && dv == 128);
}

}  // namespace seed
