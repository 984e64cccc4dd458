// seed_compress_fast.cu -- the compression of units with R + W <= 32, R <= 16.
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
//   5. with X_R the R leading left singular vectors of M (orthonormalised once
//      more, in descending order, by two passes of Gram-Schmidt):
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

// Equilibrate the Gram row held by lane i (divide by the column norms) and return
// the norm of column i.  Row i of the result is Uhat^T Uhat restricted to row i.
template <int MP>
SEED_DEV float equilibrate_row(float (&g)[MP]) {
  const int lane = threadIdx.x & 31;
  float d = 0.f;
#pragma unroll
  for (int i = 0; i < MP; ++i)
    if (i == lane) d = g[i];
  const float n = sqrtf(fmaxf(d, 0.f));
  const float ninv = n > 0.f ? 1.f / n : 0.f;
#pragma unroll
  for (int i = 0; i < MP; ++i) g[i] *= __shfl_sync(0xffffffffu, ninv, i) * ninv;
  return lane < MP ? n : 0.f;
}

// Right-looking Cholesky in registers, one warp, lane i holding row i of the
// equilibrated Gram; on return row i of L (lower; the upper part zero).  Column j
// is dropped (zero) when column j of the panel is zero (norm_j == 0) or the pivot
// is not positive; a pivot below kCholPivotMin on a nonzero column also sets *bad.
template <int MP>
SEED_DEV void cholesky_regs(float (&g)[MP], float norm_self, int* bad) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < MP; ++j) {
    const float d = __shfl_sync(0xffffffffu, g[j], j);
    const bool zero = !(__shfl_sync(0xffffffffu, norm_self, j) > 0.f);
    bool drop = zero || !(d > 0.f);
    if (!zero && d < kCholPivotMin) {
      drop = true;
      if (lane == 0) *bad = 1;
    }
    const float rs = drop ? 0.f : rsqrtf(d);
    const float lij = lane > j ? g[j] * rs : 0.f;
    g[j] = lane == j ? d * rs : lij;
#pragma unroll
    for (int k = j + 1; k < MP; ++k) {
      const float lkj = __shfl_sync(0xffffffffu, lij, k);
      if (k <= lane) g[k] = fmaf(-lij, lkj, g[k]);
    }
  }
}

// Shared memory: the two panels (region A) are only read by the Gram phase; every
// later buffer aliases region A.  The small per-column arrays live after it.
template <int FORM, int DK, int DV, int MP>
struct FastLayout {
  static constexpr int LDK = DK + 4, LDV = DV + 4, LG = MP + 1, LM = MP + 4;
  static constexpr int SL = (FORM == SEED_KDA ? DK : MP);
  static constexpr int A = MP * LDK + MP * LDV;                 // panels
  static constexpr int B = 2 * MP * LG + MP * LM + MP * MP;     // L_u, L_v / X, M / T_u, T_v
  static_assert(B <= A, "aliased buffers must fit in the panel region");
  static constexpr int SMALL = 6 * MP + SL;                     // nu nv nrm sig csu csv scl
  static constexpr size_t bytes = (A + SMALL) * sizeof(float) + (MP + 4) * sizeof(int);
};

template <int FORM, int DK, int DV, int MP>
__global__ void __launch_bounds__(64) compress_fast_kernel(const FastParams p) {
  using Lay = FastLayout<FORM, DK, DV, MP>;
  constexpr bool KDA = FORM == SEED_KDA;
  constexpr int LDK = Lay::LDK, LDV = Lay::LDV, LG = Lay::LG, LM = Lay::LM;
  constexpr int PK = DK / 32, PV = DV / 32;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  float* sU = reinterpret_cast<float*>(smem_raw);   // region A
  float* sV = sU + MP * LDK;
  float* sGu = sU;                                   // region B, after the Grams
  float* sGv = sGu + MP * LG;                        // L_v, then the selected vectors X
  float* sM = sGv + MP * LG;                         // the core, then T_u
  float* sTv = sM + MP * LM;                         // Gram-Schmidt scratch, then T_v
  float* nu = sU + Lay::A;                           // small arrays
  float* nv = nu + MP;
  float* nrm = nv + MP;
  float* sig = nrm + MP;
  float* csu = sig + MP;
  float* csv = csu + MP;
  float* scl = csv + MP;
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
  const float* Ug = p.U + unit * (long long)m * DK;
  const float* Vg = p.V + unit * (long long)m * DV;

  // 1. panels -> shared memory
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&bar, (uint32_t)(m * (DK + DV) * 4));
    flags[0] = 0;
  }
  __syncthreads();
  if (warp == 0 && lane < m) {
    bulk_g2s(sU + lane * LDK, Ug + (long long)lane * DK, DK * 4, &bar);
    bulk_g2s(sV + lane * LDV, Vg + (long long)lane * DV, DV * 4, &bar);
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

  // column scaling by the largest magnitude (warp 0: U, warp 1: V) so that no
  // Gram entry is formed from values near the float32 underflow
  {
    float* Pn = warp == 0 ? sU : sV;
    const int LD = warp == 0 ? LDK : LDV;
    const int D = warp == 0 ? DK : DV;
    float mx = 0.f;
    if (lane < m) {
      for (int r = 0; r < D; r += 4) {
        const float4 x = ld4(Pn + lane * LD + r);
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
      }
      const float inv = mx > 0.f ? 1.f / mx : 0.f;
      for (int r = 0; r < D; r += 4) {
        float4 x = ld4(Pn + lane * LD + r);
        x.x *= inv; x.y *= inv; x.z *= inv; x.w *= inv;
        st4(Pn + lane * LD + r, x);
      }
    }
    if (lane < MP) (warp == 0 ? csu : csv)[lane] = mx;
  }
  __syncthreads();

  // 2. equilibrated Grams and their Cholesky factors, in registers (warp 0: U,
  //    warp 1: V); L then stored row-major (ld MP+1) over the panel region
  {
    float g[MP];
    if (warp == 0) gram_row<MP, DK, LDK>(sU, g);
    else gram_row<MP, DV, LDV>(sV, g);
    const float n = equilibrate_row<MP>(g);
    if (lane < MP) (warp == 0 ? nu : nv)[lane] = n;
    cholesky_regs<MP>(g, n, flags);
    __syncthreads();   // both Grams are read before L overwrites the panels
    float* G = warp == 0 ? sGu : sGv;
    if (lane < MP) {
#pragma unroll
      for (int k = 0; k < MP; ++k) G[lane * LG + k] = g[k];
    }
  }
  __syncthreads();
  if (flags[0]) {   // ill-conditioned: left for the Householder kernel
    if (tid == 0) atomicAdd(p.status + 6, 1u);
    return;
  }

  // D_u, D_v: true column norms (panel scale times the scaled-column norm, and for
  // GDN / Mamba-2 the lazy scale gamma_j)
  if (tid < MP) {
    const float gj = (KDA || tid >= m) ? 1.f : scl[tid];
    nrm[tid] = nu[tid] * csu[tid] * gj;   // D_u
    csv[tid] = nv[tid] * csv[tid];        // D_v
  }
  __syncthreads();

  // 3. core M = L_u^T diag(D_u D_v) L_v, column-major (ld LM)
  for (int e = tid; e < MP * MP; e += 64) {
    const int j = e / MP, i = e - j * MP;
    float acc = 0.f;
    for (int k = max(i, j); k < MP; ++k)
      acc = fmaf(sGu[k * LG + i] * (nrm[k] * csv[k]), sGv[k * LG + j], acc);
    sM[j * LM + i] = acc;
  }
  __syncthreads();
  if (tid < MP) sig[tid] = nrm[tid];   // keep D_u in sig until the end
  __syncthreads();

  // 4. one-sided Jacobi on M: 16 pairs per round, pair pr = warp * 8 + lane / 4,
  //    lane quarter q holds rows 4 NF q .. of both columns
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
      constexpr int NF = MP / 16;    // float4 per lane per column
      const bool active = (MP == 32) || pr < MP / 2;   // with MP = 32 every lane has a pair
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
      // rotation test and parameters with the fast intrinsics: t need not be the
      // exact tangent, the rotation stays orthogonal because c = 1 / sqrt(1 + t^2)
      if (active && al > tiny && be > tiny && fabsf(g) > tol * sqrtf(al) * sqrtf(be)) {
        const float zeta = __fdividef(be - al, 2.f * g);
        float t;
        if (fabsf(zeta) > 1e18f) t = __fdividef(0.5f, zeta);
        else {
          const float z1 = fmaf(zeta, zeta, 1.f);
          t = copysignf(__fdividef(1.f, fabsf(zeta) + z1 * rsqrtf(z1)), zeta);
        }
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
    atomicAdd(p.status + 5, 1u);
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

  // 5b. orthonormalise the selected left vectors x_r = (M Z)_{sel r} / sigma_r in
  //     descending order (classical Gram-Schmidt, two passes; warp 0, lane = row).
  //     The Jacobi leaves columns it judged negligible unrotated, so the raw x_r
  //     need not be orthogonal; with orthonormal x_r the result below is exactly
  //     the projection of U V^T on their span.  A vector that loses more than half
  //     its norm to the earlier ones adds no new direction and is dropped.
  float* sX = sGv;   // R x MP (L_v is no longer needed)
  float* sP = sTv;   // scratch, R x (MP+1)
  float* sgk = csu;  // sigma kept for each output column (0: dropped)
  if (warp == 0) {
    for (int r = 0; r < p.R; ++r) {
      const int j = sel[r];
      const float sj = nrm[j];
      float x = (lane < MP && sj > szero) ? sM[j * LM + lane] / sj : 0.f;
      for (int pass = 0; pass < 2; ++pass) {
        for (int k = 0; k < r; ++k)
          if (lane < MP) sP[k * (MP + 1) + lane] = x * sX[k * MP + lane];
        __syncwarp();
        float dk = 0.f;
        if (lane < r)
          for (int i = 0; i < MP; ++i) dk += sP[lane * (MP + 1) + i];
        __syncwarp();
        for (int k = 0; k < r; ++k) {
          const float d = __shfl_sync(0xffffffffu, dk, k);
          if (lane < MP) x = fmaf(-d, sX[k * MP + lane], x);
        }
      }
      const float nx = sqrtf(group_sum<32>(x * x));
      const bool keep = nx > 0.5f;
      x = keep ? x / nx : 0.f;
      if (lane < MP) sX[r * MP + lane] = x;
      if (lane == 0) sgk[r] = keep ? sj : 0.f;
      __syncwarp();
    }
  }
  __syncthreads();

  // 6. small right factors on the raw panels (column r in lane r, stored [k][r]):
  //    U' = U_raw T_u with T_u = diag(gamma / D_u) L_u^{-T} X_R Sigma^{1/2}
  //         (KDA: the row decay P is applied to the product instead of gamma)
  //    V' = V_raw T_v with T_v = D_u L_u X_R Sigma^{-1/2}
  float* sTu = sM;
  if (lane < p.R) {
    const int r = lane;
    const float s = sgk[r];
    const bool zero = !(s > 0.f);
    if (warp == 0) {
      // back substitution with L_u^T (upper): t_k = (x_k - sum_{i>k} L_u[i][k] t_i) / L_u[k][k]
      const float f = zero ? 0.f : sqrtf(s);
      for (int k = MP - 1; k >= 0; --k) {
        float acc = sX[r * MP + k] * f;
        for (int i = k + 1; i < MP; ++i) acc = fmaf(-sGu[i * LG + k], sTu[i * MP + r], acc);
        const float lkk = sGu[k * LG + k];
        sTu[k * MP + r] = lkk != 0.f ? acc / lkk : 0.f;
      }
      for (int k = 0; k < MP; ++k) {
        const float du = sig[k];
        const float gk = (KDA || k >= m) ? 1.f : scl[k];
        sTu[k * MP + r] = du > 0.f ? sTu[k * MP + r] * (gk / du) : 0.f;
      }
    } else {
      const float f = zero ? 0.f : rsqrtf(s);
      for (int k = 0; k < MP; ++k) {
        float acc = 0.f;
        for (int i = 0; i <= k; ++i) acc = fmaf(sGu[k * LG + i], sX[r * MP + i], acc);
        sTv[k * MP + r] = sig[k] * acc * f;   // sig holds D_u
      }
    }
  }
  __syncthreads();

  // 7. U' = U_raw T_u (warp 0), V' = V_raw T_v (warp 1), the panels streamed again
  //    from global memory (read a moment ago, normally still in L2); written to
  //    slots 0..R-1 after the block has read every stored column
  constexpr int CH = 16;
  float accU[CH][PK], accV[CH][PV];
  bool bad = false;
  for (int r0 = 0; r0 < p.R; r0 += CH) {
    if (warp == 0) {
#pragma unroll
      for (int q = 0; q < CH; ++q)
#pragma unroll
        for (int e = 0; e < PK; ++e) accU[q][e] = 0.f;
      for (int k = 0; k < m; ++k) {
        const auto u = VecT<PK>::load(Ug + (long long)k * DK + PK * lane);
#pragma unroll
        for (int q = 0; q < CH; ++q) {
          const float tk = (r0 + q < p.R) ? sTu[k * MP + r0 + q] : 0.f;
#pragma unroll
          for (int e = 0; e < PK; ++e) accU[q][e] = fmaf(VecT<PK>::get(u, e), tk, accU[q][e]);
        }
      }
      if constexpr (KDA) {
#pragma unroll
        for (int e = 0; e < PK; ++e) {
          const float pe = scl[PK * lane + e];
#pragma unroll
          for (int q = 0; q < CH; ++q) accU[q][e] *= pe;
        }
      }
    } else {
#pragma unroll
      for (int q = 0; q < CH; ++q)
#pragma unroll
        for (int e = 0; e < PV; ++e) accV[q][e] = 0.f;
      for (int k = 0; k < m; ++k) {
        const auto v = VecT<PV>::load(Vg + (long long)k * DV + PV * lane);
#pragma unroll
        for (int q = 0; q < CH; ++q) {
          const float tk = (r0 + q < p.R) ? sTv[k * MP + r0 + q] : 0.f;
#pragma unroll
          for (int e = 0; e < PV; ++e) accV[q][e] = fmaf(VecT<PV>::get(v, e), tk, accV[q][e]);
        }
      }
    }
    __syncthreads();   // every stored column of this chunk's range is read
    float* Uo = p.U + unit * (long long)m * DK;
    float* Vo = p.V + unit * (long long)m * DV;
#pragma unroll
    for (int q = 0; q < CH; ++q) {
      if (r0 + q < p.R) {
        if (warp == 0) {
#pragma unroll
          for (int e = 0; e < PK; ++e) {
            bad |= !isfinite(accU[q][e]);
            Uo[(long long)(r0 + q) * DK + PK * lane + e] = accU[q][e];
          }
        } else {
#pragma unroll
          for (int e = 0; e < PV; ++e) {
            bad |= !isfinite(accV[q][e]);
            Vo[(long long)(r0 + q) * DV + PV * lane + e] = accV[q][e];
          }
        }
      }
    }
    __syncthreads();
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

// R <= 16: the R new columns are accumulated in registers in one pass over the
// old ones, so that no output overwrites a column before every column was read.
bool compress_fast_supported(const seed_dims& d) {
  const int m = d.R + d.W;
  return m <= 32 && d.R <= 16 && (d.d_k == 64 || d.d_k == 128) && (d.d_v == 64 || d.d_v == 128);
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
