// seed_compress_fast.cu -- the compression of units with R + W <= 32 columns.
//
// "Shallow Encoding Emits Deep Memories", SEED figures & tables (thelatestinai.com),
// Figure 1(b): every W steps the factors are compressed back to rank R.  Two warps
// per unit, everything in shared memory or registers, no Householder sweeps:
//
//   1. TMA copies of both panels (one 512-byte bulk copy per column, into rows
//      padded by 4 floats so that the Gram loops read without bank conflicts);
//   2. Gram matrices of the column-equilibrated panels, G = Uhat^T Uhat and
//      Vhat^T Vhat (warp 0 and warp 1 in parallel), and their Cholesky factors
//      L_u, L_v, so that U = Q_u R_u, V = Q_v R_v with R = L^T D (D the column
//      norms, and the lazy decay scales for GDN / Mamba-2);
//   3. the core M = R_u R_v^T = L_u^T D_u D_v L_v (m x m);
//   4. one-sided Jacobi on M (Hestenes; round-robin pairs split over both warps,
//      four lanes per pair; column norms carried by the exact update
//      a' = a - t g, b' = b + t g and recomputed every sweep), M Z = X Sigma;
//   5. with X_R the R leading left singular vectors:
//        U' = Q_u X_R Sigma^{1/2} = Uhat (L_u^{-T} X_R Sigma^{1/2})
//        V' = A^T U' Sigma^{-1}   = V (D_u L_u X_R Sigma^{-1/2})
//      so that U' V'^T = Q_u X_R X_R^T Q_u^T U V^T, the projection of U V^T on the
//      computed rank-R left subspace.
//
// Cholesky QR is exact when the equilibrated Gram is well conditioned.  A unit
// whose Cholesky meets a pivot below 1e-2 (condition number above about 10: two
// nearly parallel keys or values inside one window) is left untouched here; the
// Householder kernel (seed_compress.cu) then compresses it.  Exactly zero columns
// (a rank-deficient start, or a decay scale that underflowed) are dropped, which
// is exact.
#include "seed_common.cuh"
#include "seed_launch.h"
#include "seed_tma.cuh"

namespace seed {

struct FastParams {
  float* U;
  float* V;
  float* scale;
  int32_t* ncols;
  float* sigma_out;
  uint32_t* status;
  int B, L, H, layer, R, W, slen;
};

constexpr float kCholPivotMin = 1e-2f;

SEED_DEV void pair_sync() { asm volatile("bar.sync 1, 64;" ::: "memory"); }

template <int PER>
struct VecT;
template <>
struct VecT<4> {
  using T = float4;
  static SEED_DEV float4 load(const float* p) { return *reinterpret_cast<const float4*>(p); }
  static SEED_DEV float get(const float4& v, int e) { return e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w; }
};
template <>
struct VecT<2> {
  using T = float2;
  static SEED_DEV float2 load(const float* p) { return *reinterpret_cast<const float2*>(p); }
  static SEED_DEV float get(const float2& v, int e) { return e == 0 ? v.x : v.y; }
};

// Row `lane` of the Gram matrix P^T P of a panel with MP columns (column j at
// P + j * LD, D rows), i.e. the dot products of column `lane` with every column.
template <int MP, int D, int LD>
SEED_DEV void gram_row(const float* P, float (&acc)[MP]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < MP; ++i) acc[i] = 0.f;
  const float* own = P + (lane < MP ? lane : 0) * LD;
#pragma unroll 2
  for (int r = 0; r < D; r += 4) {
    const float4 o = ld4(own + r);
#pragma unroll
    for (int i = 0; i < MP; ++i) acc[i] += dot4(ld4(P + i * LD + r), o);
  }
}

// Equilibrate the Gram row of lane i (divide by the column norms), store it as row i
// of G (ld MP+1), and store the norm of column i in nrm[i].
template <int MP>
SEED_DEV void equilibrate_store(float (&acc)[MP], float* G, float* nrm) {
  const int lane = threadIdx.x & 31;
  float d = 0.f;
#pragma unroll
  for (int i = 0; i < MP; ++i)
    if (i == lane) d = acc[i];
  const float n = sqrtf(fmaxf(d, 0.f));
  const float ninv = n > 0.f ? 1.f / n : 0.f;
#pragma unroll
  for (int i = 0; i < MP; ++i) {
    const float ni = __shfl_sync(0xffffffffu, ninv, i);
    if (lane < MP) G[lane * (MP + 1) + i] = acc[i] * ni * ninv;
  }
  if (lane < MP) nrm[lane] = n;
}

// Right-looking Cholesky of the equilibrated Gram in place (lower triangle, ld
// MP+1), one warp, lane i owns row i.  Zero columns (norm 0) are dropped; a pivot
// below kCholPivotMin on a nonzero column sets *bad and is dropped as well.
template <int MP>
SEED_DEV void cholesky_warp(float* G, const float* nrm, int* bad) {
  const int i = threadIdx.x & 31;
  constexpr int LG = MP + 1;
  for (int j = 0; j < MP; ++j) {
    const float d = G[j * LG + j];
    const bool zero = !(nrm[j] > 0.f);
    bool drop = zero || !(d > 0.f);
    if (!zero && d < kCholPivotMin) {
      drop = true;
      if (i == 0) *bad = 1;
    }
    const float ljj = drop ? 0.f : sqrtf(d);
    const float inv = drop ? 0.f : 1.f / ljj;
    float lij = 0.f;
    if (i > j && i < MP) {
      lij = G[i * LG + j] * inv;
      G[i * LG + j] = lij;
    }
    __syncwarp();
    if (i == j) G[j * LG + j] = ljj;
    if (i > j && i < MP && lij != 0.f) {
      for (int k = j + 1; k <= i; ++k) G[i * LG + k] = fmaf(-lij, G[k * LG + j], G[i * LG + k]);
    }
    __syncwarp();
  }
  // zero the strict upper triangle so that later loops may read it unconditionally
  for (int k = i + 1; k < MP; ++k) G[i * LG + k] = 0.f;
  __syncwarp();
}

template <int FORM, int DK, int DV, int MP>
struct FastLayout {
  static constexpr int LDK = DK + 4, LDV = DV + 4, LG = MP + 1, LM = MP + 4;
  static constexpr int SL = (FORM == SEED_KDA ? DK : MP);
  static constexpr int floats = MP * LDK + MP * LDV + 2 * MP * LG + MP * LM + 2 * MP * MP + 4 * MP + SL;
  static constexpr size_t bytes = floats * sizeof(float) + (MP + 4) * sizeof(int);
};

template <int FORM, int DK, int DV, int MP>
__global__ void __launch_bounds__(64) compress_fast_kernel(const FastParams p) {
  using Lay = FastLayout<FORM, DK, DV, MP>;
  constexpr bool KDA = FORM == SEED_KDA;
  constexpr int LDK = Lay::LDK, LDV = Lay::LDV, LG = Lay::LG, LM = Lay::LM;
  constexpr int PK = DK / 32, PV = DV / 32;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  float* sU = reinterpret_cast<float*>(smem_raw);
  float* sV = sU + MP * LDK;
  float* sGu = sV + MP * LDV;
  float* sGv = sGu + MP * LG;
  float* sM = sGv + MP * LG;
  float* sTu = sM + MP * LM;
  float* sTv = sTu + MP * MP;
  float* nu = sTv + MP * MP;
  float* nv = nu + MP;
  float* nrm = nv + MP;
  float* sig = nrm + MP;
  float* scl = sig + MP;
  int* sel = reinterpret_cast<int*>(scl + Lay::SL);
  int* flags = sel + MP;   // [0] ill-conditioned, [1] rotated this sweep
  __shared__ __align__(8) uint64_t bar;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int m = p.R + p.W;
  const int per = p.layer < 0 ? p.L * p.H : p.H;
  const int idx = blockIdx.x;
  const int b = idx / per, rest = idx - b * per;
  const long long unit =
      p.layer < 0 ? (long long)idx : ((long long)b * p.L + p.layer) * p.H + rest;
  if (p.ncols[unit] != m) return;   // not due (the fallback kernel flags invalid counts)

  // 1. panels -> shared memory
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&bar, (uint32_t)(m * (DK + DV) * 4));
    flags[0] = 0;
  }
  __syncthreads();
  if (warp == 0 && lane < m) {
    bulk_g2s(sU + lane * LDK, p.U + unit * (long long)m * DK + (long long)lane * DK, DK * 4, &bar);
    bulk_g2s(sV + lane * LDV, p.V + unit * (long long)m * DV + (long long)lane * DV, DV * 4, &bar);
  }
  for (int e = m * LDK + tid; e < MP * LDK; e += 64) sU[e] = 0.f;
  for (int e = m * LDV + tid; e < MP * LDV; e += 64) sV[e] = 0.f;
  for (int e = tid; e < p.slen; e += 64) scl[e] = p.scale[unit * p.slen + e];
  if (!__syncthreads_and(mbar_wait_bounded(&bar, 0, kWaitLimitNs))) {
    if (tid == 0) raise_flag(p.status, SEED_FLAG_TIMEOUT);
    mbar_wait_bounded(&bar, 0, kWaitLimitNs);
    return;
  }
  if constexpr (KDA) {   // true U = Diag(P) U
    for (int e = tid; e < m * DK; e += 64) {
      const int j = e / DK, r = e - j * DK;
      sU[j * LDK + r] *= scl[r];
    }
    __syncthreads();
  }

  // 2. equilibrated Grams and their Cholesky factors (warp 0: U, warp 1: V)
  {
    float acc[MP];
    if (warp == 0) {
      gram_row<MP, DK, LDK>(sU, acc);
      equilibrate_store<MP>(acc, sGu, nu);
    } else {
      gram_row<MP, DV, LDV>(sV, acc);
      equilibrate_store<MP>(acc, sGv, nv);
    }
    __syncwarp();
    cholesky_warp<MP>(warp == 0 ? sGu : sGv, warp == 0 ? nu : nv, flags);
  }
  __syncthreads();
  if (flags[0]) return;   // ill-conditioned: left for the Householder kernel

  // D_u: true column norms of U (GDN / Mamba-2 include the lazy scale gamma_j)
  if (tid < MP) {
    const float gj = (KDA || tid >= m) ? 1.f : scl[tid];
    nrm[tid] = nu[tid] * gj;   // nrm temporarily holds D_u
  }
  __syncthreads();

  // 3. core M = L_u^T diag(D_u D_v) L_v, column-major (ld LM)
  for (int e = tid; e < MP * MP; e += 64) {
    const int j = e / MP, i = e - j * MP;
    float acc = 0.f;
    for (int k = max(i, j); k < MP; ++k)
      acc = fmaf(sGu[k * LG + i] * (nrm[k] * nv[k]), sGv[k * LG + j], acc);
    sM[j * LM + i] = acc;
  }
  __syncthreads();
  if (tid < MP) sig[tid] = nrm[tid];   // keep D_u in sig until the Jacobi is done
  __syncthreads();

  // 4. one-sided Jacobi on M: 16 pairs per round, pair pr = warp * 8 + lane / 4,
  //    lane quarter q holds rows 8q .. 8q+7 of both columns
  const int pr = warp * 8 + (lane >> 2), qt = lane & 3;
  const float tol = 8.f * sqrtf((float)MP) * 5.9604645e-8f;
  float tiny = 0.f;
  int sweeps = 0;
  bool converged = false;
  for (int sweep = 0; sweep < 30; ++sweep) {
    if (tid < MP) {
      float s2 = 0.f;
#pragma unroll
      for (int r = 0; r < MP; r += 4) {
        const float4 x = ld4(sM + tid * LM + r);
        s2 += dot4(x, x);
      }
      nrm[tid] = s2;
    }
    if (tid == 0) flags[1] = 0;
    pair_sync();
    if (sweep == 0) {
      float f2 = 0.f;
      for (int j = 0; j < MP; ++j) f2 += nrm[j];
      tiny = 1e-10f * f2;
    }
    for (int round = 0; round < MP - 1; ++round) {
      int P, Q;
      if (pr == 0) {
        P = MP - 1;
        Q = round;
      } else {
        P = round + pr;
        if (P >= MP - 1) P -= MP - 1;
        Q = round - pr;
        if (Q < 0) Q += MP - 1;
      }
      constexpr int NF = MP / 16;    // float4 per lane per column (rows 4*NF*qt ..)
      const bool active = pr < MP / 2;
      float* xp = sM + P * LM + 4 * NF * qt;
      float* yp = sM + Q * LM + 4 * NF * qt;
      float4 xv[NF], yv[NF];
      float g = 0.f;
#pragma unroll
      for (int f = 0; f < NF; ++f) {
        xv[f] = active ? ld4(xp + 4 * f) : zero4();
        yv[f] = active ? ld4(yp + 4 * f) : zero4();
        g += dot4(xv[f], yv[f]);
      }
      g += __shfl_xor_sync(0xffffffffu, g, 1);
      g += __shfl_xor_sync(0xffffffffu, g, 2);
      const float al = active ? nrm[P] : 0.f, be = active ? nrm[Q] : 0.f;
      if (active && al > tiny && be > tiny && fabsf(g) > tol * sqrtf(al) * sqrtf(be)) {
        const float zeta = (be - al) / (2.f * g);
        float t;
        if (fabsf(zeta) > 1e18f) t = 0.5f / zeta;
        else t = copysignf(1.f, zeta) / (fabsf(zeta) + sqrtf(fmaf(zeta, zeta, 1.f)));
        const float cs = rsqrtf(fmaf(t, t, 1.f));
        const float sn = cs * t;
#pragma unroll
        for (int f = 0; f < NF; ++f) {
          const float4 x = xv[f], y = yv[f];
          float4 a, bb;
          a.x = cs * x.x - sn * y.x; bb.x = fmaf(sn, x.x, cs * y.x);
          a.y = cs * x.y - sn * y.y; bb.y = fmaf(sn, x.y, cs * y.y);
          a.z = cs * x.z - sn * y.z; bb.z = fmaf(sn, x.z, cs * y.z);
          a.w = cs * x.w - sn * y.w; bb.w = fmaf(sn, x.w, cs * y.w);
          st4(xp + 4 * f, a);
          st4(yp + 4 * f, bb);
        }
        if (qt == 0) {
          nrm[P] = al - t * g;
          nrm[Q] = be + t * g;
          flags[1] = 1;
        }
      }
      pair_sync();
    }
    sweeps = sweep + 1;
    const int any = flags[1];
    pair_sync();
    if (!any) {
      converged = true;
      break;
    }
  }
  if (tid == 0) {
    atomicAdd(p.status + 1, (uint32_t)sweeps);
    atomicAdd(p.status + 2, 1u);
    if (!converged) raise_flag(p.status, SEED_FLAG_NOCONVERGE);
  }

  // 5. singular values = column norms of M Z; the R largest
  if (tid < MP) {
    float s2 = 0.f;
#pragma unroll
    for (int r = 0; r < MP; r += 4) {
      const float4 x = ld4(sM + tid * LM + r);
      s2 += dot4(x, x);
    }
    nrm[tid] = sqrtf(s2);
  }
  __syncthreads();
  if (tid < MP) {
    const float s = nrm[tid];
    int rank = 0;
    for (int k = 0; k < MP; ++k) {
      const float t = nrm[k];
      rank += (t > s) || (t == s && k < tid);
    }
    if (rank < p.R) sel[rank] = tid;
  }
  __syncthreads();
  float smax = 0.f;
  for (int j = 0; j < MP; ++j) smax = fmaxf(smax, nrm[j]);
  const float szero = (float)(DK > DV ? DK : DV) * 1.1920929e-7f * smax;

  // 6. small right factors: T_u = diag(1/n_u) L_u^{-T} X_R Sigma^{1/2} (warp 0),
  //    T_v = D_u L_u X_R Sigma^{-1/2} (warp 1); column r in lane r, stored [k][r]
  if (lane < p.R) {
    const int r = lane;
    const int j = sel[r];
    const float s = nrm[j];
    const bool zero = !(s > szero);
    if (warp == 0) {
      // back substitution with L_u^T (upper): t_k = (x_k - sum_{i>k} L_u[i][k] t_i) / L_u[k][k]
      const float f = zero ? 0.f : rsqrtf(s);   // x = (M Z)_j / s * sqrt(s)
      for (int k = MP - 1; k >= 0; --k) {
        float acc = sM[j * LM + k] * f;
        for (int i = k + 1; i < MP; ++i) acc = fmaf(-sGu[i * LG + k], sTu[i * MP + r], acc);
        const float lkk = sGu[k * LG + k];
        sTu[k * MP + r] = lkk != 0.f ? acc / lkk : 0.f;
      }
      for (int k = 0; k < MP; ++k) {
        const float n = nu[k];
        sTu[k * MP + r] = n > 0.f ? sTu[k * MP + r] / n : 0.f;
      }
    } else {
      const float f = zero ? 0.f : 1.f / (s * sqrtf(s));   // x = (M Z)_j / s, times s^{-1/2}
      for (int k = 0; k < MP; ++k) {
        float acc = 0.f;
        for (int i = 0; i <= k; ++i) acc = fmaf(sGu[k * LG + i], sM[j * LM + i], acc);
        sTv[k * MP + r] = sig[k] * acc * f;   // sig holds D_u here
      }
    }
  }
  __syncthreads();

  // 7. U' = Uhat T_u (warp 0), V' = V T_v (warp 1), written to slots 0..R-1
  bool bad = false;
  float* Ug = p.U + unit * (long long)m * DK;
  float* Vg = p.V + unit * (long long)m * DV;
  if (warp == 0) {
    for (int r0 = 0; r0 < p.R; r0 += 8) {
      float acc[8][PK];
#pragma unroll
      for (int q = 0; q < 8; ++q)
#pragma unroll
        for (int e = 0; e < PK; ++e) acc[q][e] = 0.f;
      for (int k = 0; k < m; ++k) {
        const auto u = VecT<PK>::load(sU + k * LDK + PK * lane);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float tk = (r0 + q < p.R) ? sTu[k * MP + r0 + q] : 0.f;
#pragma unroll
          for (int e = 0; e < PK; ++e) acc[q][e] = fmaf(VecT<PK>::get(u, e), tk, acc[q][e]);
        }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (r0 + q < p.R) {
#pragma unroll
          for (int e = 0; e < PK; ++e) {
            bad |= !isfinite(acc[q][e]);
            Ug[(long long)(r0 + q) * DK + PK * lane + e] = acc[q][e];
          }
        }
      }
    }
  } else {
    for (int r0 = 0; r0 < p.R; r0 += 8) {
      float acc[8][PV];
#pragma unroll
      for (int q = 0; q < 8; ++q)
#pragma unroll
        for (int e = 0; e < PV; ++e) acc[q][e] = 0.f;
      for (int k = 0; k < m; ++k) {
        const auto v = VecT<PV>::load(sV + k * LDV + PV * lane);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float tk = (r0 + q < p.R) ? sTv[k * MP + r0 + q] : 0.f;
#pragma unroll
          for (int e = 0; e < PV; ++e) acc[q][e] = fmaf(VecT<PV>::get(v, e), tk, acc[q][e]);
        }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (r0 + q < p.R) {
#pragma unroll
          for (int e = 0; e < PV; ++e) {
            bad |= !isfinite(acc[q][e]);
            Vg[(long long)(r0 + q) * DV + PV * lane + e] = acc[q][e];
          }
        }
      }
    }
  }
  if (p.sigma_out && tid < p.R) p.sigma_out[(long long)idx * p.R + tid] = nrm[sel[tid]];
  for (int e = tid; e < p.slen; e += 64) p.scale[unit * p.slen + e] = 1.f;
  __syncthreads();
  if (tid == 0) p.ncols[unit] = p.R;
  if (bad) raise_flag(p.status, SEED_FLAG_NONFINITE);
}

template <int FORM, int DK, int DV, int MP>
static int launch_fast_t(const FastParams& p, int blocks, cudaStream_t st) {
  using Lay = FastLayout<FORM, DK, DV, MP>;
  auto kern = compress_fast_kernel<FORM, DK, DV, MP>;
  constexpr int kMaxDev = 64;
  static bool attr_set[kMaxDev] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return SEED_ERR_CUDA;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lay::bytes) !=
        cudaSuccess)
      return SEED_ERR_CUDA;
    attr_set[dev] = true;
  }
  kern<<<blocks, 64, Lay::bytes, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
}

template <int FORM, int DK, int DV>
static int launch_fast_m(const FastParams& p, int blocks, cudaStream_t st) {
  const int m = p.R + p.W;
  if (m <= 16) return launch_fast_t<FORM, DK, DV, 16>(p, blocks, st);
  return launch_fast_t<FORM, DK, DV, 32>(p, blocks, st);
}

bool compress_fast_supported(const seed_dims& d) {
  const int m = d.R + d.W;
  return m <= 32 && (d.d_k == 64 || d.d_k == 128) && (d.d_v == 64 || d.d_v == 128);
}

int launch_compress_fast(const seed_dims& d, const seed_state& s, int layer, float* sigma_out,
                         uint32_t* status, cudaStream_t st) {
  FastParams p{s.U, s.V, s.scale, s.ncols, sigma_out, status,
               d.batch, d.layers, d.heads, layer, d.R, d.W, scale_len(d)};
  const int blocks = d.batch * d.heads * (layer < 0 ? d.layers : 1);
#define SEED_FAST_DIMS(FORM)                                                                       \
  do {                                                                                             \
    if (d.d_k == 128 && d.d_v == 128) return launch_fast_m<FORM, 128, 128>(p, blocks, st);          \
    if (d.d_k == 128 && d.d_v == 64) return launch_fast_m<FORM, 128, 64>(p, blocks, st);            \
    if (d.d_k == 64 && d.d_v == 128) return launch_fast_m<FORM, 64, 128>(p, blocks, st);            \
    if (d.d_k == 64 && d.d_v == 64) return launch_fast_m<FORM, 64, 64>(p, blocks, st);              \
    return SEED_ERR_SHAPE;                                                                         \
  } while (0)
  switch (d.form) {
    case SEED_GDN: SEED_FAST_DIMS(SEED_GDN);
    case SEED_KDA: SEED_FAST_DIMS(SEED_KDA);
    case SEED_MAMBA2: SEED_FAST_DIMS(SEED_MAMBA2);
  }
#undef SEED_FAST_DIMS
  return SEED_ERR_INVALID_ARG;
}

}  // namespace seed
