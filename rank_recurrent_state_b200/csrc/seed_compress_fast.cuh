// seed_compress_fast.cuh -- the compression of units with R + W <= 32, R <= 16.
//
// "Shallow Encoding Emits Deep Memories", SEED figures & tables (thelatestinai.com),
// Figure 1(b): every W steps the factors are compressed back to rank R.  One warp
// per unit, no Householder sweeps:
//
//   1. the U panel streams through two shared-memory chunk buffers, 32 rows of
//      every column per chunk (one 3-D tensor-map copy with a 128-byte swizzle;
//      16-bit factors: cp.async into staging buffers, widened to float32 in the
//      same layout); the Gram matrix G = U^T U accumulates on the tensor cores
//      (mma.sync TF32 with a three-term hi/lo split, float32 accuracy), is
//      equilibrated by the column norms and factored by Cholesky in shared memory
//      (L_u; right-looking, lane = row, each step's column broadcast from shared
//      memory); then the V panel the same way (L_v).  So U = Q_u R_u, V = Q_v R_v
//      with R = L^T D (D the column norms, and the lazy decay scales for GDN /
//      Mamba-2);
//   2. the core M = R_u R_v^T = L_u^T D_u D_v L_v (m x m);
//   3. one-sided Jacobi on M (Hestenes), M Z = X Sigma, with the columns held in
//      registers: a column pair per two lanes (four when m <= 16), rotations of
//      Rutishauser applied to scaled columns (true column = s * stored column,
//      two FMAs per element pair), column norms carried by the exact update and
//      recomputed every sweep.  Pair order: recursive halving -- all pairs between
//      the two halves of the columns (a cyclic shift of one half against the
//      other), then the same within each half, so that each round moves one
//      column of each pair between lanes instead of two;
//   4. with X_R the R leading left singular vectors of M (orthonormalised once
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
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "seed_common.cuh"
#include "seed_launch.h"
#include "seed_tma.cuh"

namespace seed {

struct FastParams {
  void* U;   // element type: the kernel's factor type
  void* V;
  float* scale;
  int32_t* ncols;
  float* sigma_out;
  uint32_t* status;
  int B, L, H, layer, R, W, slen;
};

constexpr float kCholPivotMin = 1e-2f;
constexpr int kFastMaxR = 16;
constexpr int kJacobiMaxSweeps = 30;
constexpr unsigned kFull = 0xffffffffu;
// Stored columns whose largest magnitude lies outside [2^-50, 2^50] (zero allowed)
// could under- or overflow the float32 Gram; such units go to the Householder path.
constexpr float kColMin = 8.8817842e-16f;   // 2^-50
constexpr float kColMax = 1.1258999e15f;    // 2^50

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

// Equilibrate the Gram G (MP x MP, row-major, stride LG; columns at or beyond m are
// zero) by its column norms and factor it by Cholesky in place, one warp, lane i
// owning rows i and i + 32 (MP <= 64).  Right-looking in panels of four columns: the
// lanes hold their rows' four panel entries in registers and factor the panel column
// by column (the pivot and the column below it travel by warp shuffles), store it,
// and then every row below the panel takes the panel's rank-4 update of its columns
// to the right, four at a time, the panel rows of L read back from G (128-bit
// accesses; the part above the diagonal is not read and is zeroed at the end).  Every
// entry receives the same fused multiply-adds in the same order as a column-by-column
// factorisation, with two warp barriers per panel instead of per column.  On return
// G[i * LG + j] = L[i][j] for j <= i, 0 above, and nrm holds the column norms.  A
// zero column, or a non-positive pivot, gives a zero column of L; a pivot below
// kCholPivotMin on a nonzero column also sets bad.  ninv: MP floats of scratch.
// Not inlined: each compression factors two Grams with it, and one copy of the code
// keeps the kernel within the instruction cache.
template <int MP, int LG>
__device__ __noinline__ void cholesky_wide(float* G, int m, float* nrm, float* ninv, bool& bad) {
  static_assert(MP % 4 == 0, "whole panels");
  const int lane = threadIdx.x & 31;
  constexpr int RPL = (MP + 31) / 32;
#pragma unroll
  for (int h = 0; h < RPL; ++h) {
    const int i = lane + 32 * h;
    if (i >= MP) continue;
    const float n = i < m ? sqrtf(fmaxf(G[i * LG + i], 0.f)) : 0.f;
    nrm[i] = n;
    ninv[i] = n > 0.f ? 1.f / n : 0.f;
  }
  __syncwarp();
#pragma unroll
  for (int h = 0; h < RPL; ++h) {
    const int i = lane + 32 * h;
    if (i >= MP) continue;
    const float fi = ninv[i];
#pragma unroll
    for (int j4 = 0; j4 < MP; j4 += 4) {
      float4 g = ld4(G + i * LG + j4);
      const float4 n4 = ld4(ninv + j4);
      g.x *= fi * n4.x; g.y *= fi * n4.y; g.z *= fi * n4.z; g.w *= fi * n4.w;
      st4(G + i * LG + j4, g);
    }
  }
  __syncwarp();
#pragma unroll 1
  for (int jb = 0; jb < m; jb += 4) {
    // the panel: columns jb .. jb + 3 of the lane's rows
    float p[RPL][4];
#pragma unroll
    for (int h = 0; h < RPL; ++h) {
      const int i = lane + 32 * h;
      const float4 t = i < MP ? ld4(G + i * LG + jb) : zero4();
      p[h][0] = t.x; p[h][1] = t.y; p[h][2] = t.z; p[h][3] = t.w;
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int j = jb + t;
      if (j >= m) break;
      const float pj = (RPL > 1 && (j >> 5) == 1) ? p[RPL - 1][t] : p[0][t];
      const float d = __shfl_sync(kFull, pj, j & 31);
      const bool zero = !(nrm[j] > 0.f);
      bool drop = zero || !(d > 0.f);
      if (!zero && d < kCholPivotMin) {
        drop = true;
        bad = true;
      }
      const float rs = drop ? 0.f : rsqrtf(d);
      float l[RPL];
#pragma unroll
      for (int h = 0; h < RPL; ++h) {
        const int i = lane + 32 * h;
        l[h] = 0.f;
        if (i >= MP) continue;
        if (i > j) {
          l[h] = p[h][t] * rs;
          p[h][t] = l[h];
        } else if (i == j) {
          p[h][t] = drop ? 0.f : d * rs;
        }
      }
      // the panel's columns after j: L[c][j] comes from the lane owning row c
#pragma unroll
      for (int t2 = t + 1; t2 < 4; ++t2) {
        const int c = jb + t2;
        const float lsrc = (RPL > 1 && (c >> 5) == 1) ? l[RPL - 1] : l[0];
        const float lc = __shfl_sync(kFull, lsrc, c & 31);
#pragma unroll
        for (int h = 0; h < RPL; ++h) {
          const int i = lane + 32 * h;
          if (i > j && i < m && l[h] != 0.f) p[h][t2] = fmaf(-l[h], lc, p[h][t2]);
        }
      }
    }
#pragma unroll
    for (int h = 0; h < RPL; ++h) {
      const int i = lane + 32 * h;
      if (i < MP) st4(G + i * LG + jb, make_float4(p[h][0], p[h][1], p[h][2], p[h][3]));
    }
    __syncwarp();   // the panel's rows of L are in G
    // rows below the panel: columns jb + 4 .. m - 1 against the panel (the rows of the
    // panel itself have nothing left below the diagonal to the right of it)
    const int c0 = jb + 4;
#pragma unroll
    for (int h = 0; h < RPL; ++h) {
      const int i = lane + 32 * h;
      if (i >= c0 && i < m) {
        const float a0 = p[h][0], a1 = p[h][1], a2 = p[h][2], a3 = p[h][3];
#pragma unroll 2
        for (int c4 = c0; c4 < m; c4 += 4) {
          float4 g = ld4(G + i * LG + c4);
          const float4 r0 = ld4(G + c4 * LG + jb);          // L[c4][jb .. jb + 3]
          const float4 r1 = ld4(G + (c4 + 1) * LG + jb);
          const float4 r2 = ld4(G + (c4 + 2) * LG + jb);
          const float4 r3 = ld4(G + (c4 + 3) * LG + jb);
          g.x = fmaf(-a0, r0.x, g.x); g.x = fmaf(-a1, r0.y, g.x); g.x = fmaf(-a2, r0.z, g.x); g.x = fmaf(-a3, r0.w, g.x);
          g.y = fmaf(-a0, r1.x, g.y); g.y = fmaf(-a1, r1.y, g.y); g.y = fmaf(-a2, r1.z, g.y); g.y = fmaf(-a3, r1.w, g.y);
          g.z = fmaf(-a0, r2.x, g.z); g.z = fmaf(-a1, r2.y, g.z); g.z = fmaf(-a2, r2.z, g.z); g.z = fmaf(-a3, r2.w, g.z);
          g.w = fmaf(-a0, r3.x, g.w); g.w = fmaf(-a1, r3.y, g.w); g.w = fmaf(-a2, r3.z, g.w); g.w = fmaf(-a3, r3.w, g.w);
          st4(G + i * LG + c4, g);
        }
      }
    }
    __syncwarp();   // the updated rows, before the next panel reads them
  }
#pragma unroll
  for (int h = 0; h < RPL; ++h) {
    const int i = lane + 32 * h;
    if (i >= MP) continue;
#pragma unroll
    for (int j4 = 0; j4 < MP; j4 += 4) {
      float4 g = ld4(G + i * LG + j4);
      if (j4 > i || i >= m) g = zero4();
      else {
        if (j4 + 1 > i) g.y = 0.f;
        if (j4 + 2 > i) g.z = 0.f;
        if (j4 + 3 > i) g.w = 0.f;
      }
      st4(G + i * LG + j4, g);
    }
  }
  __syncwarp();
}

// Lanes of one column pair (LP lanes, aligned) sum their partial values.
template <int LP>
SEED_DEV float pair_sum(float v) {
#pragma unroll
  for (int off = LP / 2; off >= 1; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
  return v;
}

SEED_DEV float warp_max(float v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, off));
  return v;
}

// One-sided Jacobi (Hestenes) on MP columns held in registers, as described at
// jacobi_regs below: lane (slot s, part h) holds rows h*NR .. h*NR+NR-1 of the pair
// (x, y) whose column indices are (ix, iy), initially (s, s + MP/2).  On return x, y
// hold the rotated columns now at (ix, iy).  NR * (64 / MP) may be below MP when the
// rows beyond it are zero in every column: rotations keep them zero, so they are
// not held.
template <int MP, int NR = MP / (64 / MP)>
SEED_DEV int jacobi_core(float (&x)[NR], float (&y)[NR], int& ix, int& iy, bool& conv) {
  constexpr int LP = 64 / MP;   // lanes per pair
  constexpr int NS = MP / 2;    // pair slots
  static_assert(NR % 4 == 0 && NR * LP <= MP, "rows per lane: whole float4s, at most MP in all");
  const int lane = threadIdx.x & 31;
  const int slot = lane / LP, h = lane % LP;
  const float tol = 8.f * sqrtf((float)MP) * 5.9604645e-8f;
  const float tol2 = tol * tol;
  float tiny = 0.f;
  int sweeps = 0;
  conv = false;
  for (int sweep = 0; sweep < kJacobiMaxSweeps; ++sweep) {
    // exact squared norms (the scales are 1 at the start of every sweep)
    float nx = 0.f, ny = 0.f;
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      nx = fmaf(x[i], x[i], nx);
      ny = fmaf(y[i], y[i], ny);
    }
    nx = pair_sum<LP>(nx);
    ny = pair_sum<LP>(ny);
    if (sweep == 0) tiny = 1e-10f * group_sum<32>(nx + ny) * (1.f / LP);
    // true column = s * stored column; r = 1 / s
    float sx = 1.f, sy = 1.f, rx = 1.f, ry = 1.f;
    bool rot = false, big = false;
#pragma unroll 1
    for (int G = NS; G >= 1; G >>= 1) {
#pragma unroll 1
      for (int r = 0; r < G; ++r) {
        float g0 = 0.f, g1 = 0.f, g2 = 0.f, g3 = 0.f;
#pragma unroll
        for (int i = 0; i < NR; i += 4) {
          g0 = fmaf(x[i], y[i], g0);
          g1 = fmaf(x[i + 1], y[i + 1], g1);
          g2 = fmaf(x[i + 2], y[i + 2], g2);
          g3 = fmaf(x[i + 3], y[i + 3], g3);
        }
        const float g = pair_sum<LP>((g0 + g1) + (g2 + g3)) * (sx * sy);
        const bool live = nx > tiny && ny > tiny;
        big |= live && g * g > 1e-6f * (nx * ny);
        if (live && g * g > tol2 * (nx * ny)) {
          // Rutishauser's rotation, t = sign(d) 2g / (|d| + sqrt(d^2 + 4 g^2)) with
          // d = |y|^2 - |x|^2 (the smaller root of t^2 + (d / g) t - 1 = 0); the
          // fast reciprocal only perturbs t, c = 1 / sqrt(1 + t^2) keeps it orthogonal
          const float d = ny - nx;
          const float e = fmaf(d, d, 4.f * g * g);
          const float t0 = __fdividef(2.f * g, fabsf(d) + e * rsqrtf(e));
          const float t = d >= 0.f ? t0 : -t0;
          const float u = fmaf(t, t, 1.f);
          const float c = rsqrtf(u);
          const float ic = u * c;
          // x' = c (x - t y), y' = c (y + t x) on the true columns; on the stored
          // ones xs' = xs - t (sy / sx) ys, ys' = ys + t (sx / sy) xs, s' = c s
          const float tx = t * sy * rx, ty = t * sx * ry;
#pragma unroll
          for (int i = 0; i < NR; ++i) {
            const float xo = x[i];
            x[i] = fmaf(-tx, y[i], xo);
            y[i] = fmaf(ty, xo, y[i]);
          }
          sx *= c;
          sy *= c;
          rx *= ic;
          ry *= ic;
          nx = fmaf(-t, g, nx);
          ny = fmaf(t, g, ny);
          rot = true;
        }
        if (r + 1 < G) {   // shift the first columns one slot along the group
          const int gb = slot & ~(G - 1);
          const int src = (gb + ((slot - gb - 1) & (G - 1))) * LP + h;
#pragma unroll
          for (int i = 0; i < NR; ++i) x[i] = __shfl_sync(kFull, x[i], src);
          ix = __shfl_sync(kFull, ix, src);
          nx = __shfl_sync(kFull, nx, src);
          sx = __shfl_sync(kFull, sx, src);
          rx = __shfl_sync(kFull, rx, src);
        }
      }
      if (G > 1) {   // halve the groups: first halves pair their x's, second halves their y's
        const int half = G >> 1;
        const bool first = (slot & half) == 0;
        const int pl = lane ^ (half * LP);
#pragma unroll
        for (int i = 0; i < NR; ++i) {
          const float got = __shfl_sync(kFull, first ? y[i] : x[i], pl);
          if (first) y[i] = got;
          else x[i] = got;
        }
        const int gi = __shfl_sync(kFull, first ? iy : ix, pl);
        const float gn = __shfl_sync(kFull, first ? ny : nx, pl);
        const float gs = __shfl_sync(kFull, first ? sy : sx, pl);
        const float gr = __shfl_sync(kFull, first ? ry : rx, pl);
        if (first) { iy = gi; ny = gn; sy = gs; ry = gr; }
        else { ix = gi; nx = gn; sx = gs; rx = gr; }
      }
    }
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      x[i] *= sx;
      y[i] *= sy;
    }
    sweeps = sweep + 1;
    // converged when nothing rotated, or when no pair was further from orthogonal
    // than 1e-3 (relative): quadratic convergence then leaves every pair below the
    // threshold after this sweep, so the sweep that would only confirm it is skipped
    if (!__any_sync(kFull, rot) || !__any_sync(kFull, big)) {
      conv = true;
      break;
    }
  }
  return sweeps;
}

// One-sided Jacobi on the MP x MP matrix in sM (column-major, stride LM), in
// registers.  Slot s = lane / LP holds the column pair (x, y); lane part h holds
// rows h*NR .. h*NR+NR-1 of both (NR below MP / LP: the rows from NR * LP on are
// zero and left as they are).  The matrix must be scaled so that its squared
// column norms stay far from the float32 range limits (entries of order one).
// Returns the sweeps run; `conv` is set when the last sweep rotated nothing.  On
// return sM holds M Z (columns in place).
template <int MP, int LM, int NR = MP / (64 / MP)>
SEED_DEV int jacobi_regs(float* sM, bool& conv) {
  constexpr int LP = 64 / MP;   // lanes per pair
  constexpr int NS = MP / 2;    // pair slots
  const int lane = threadIdx.x & 31;
  const int slot = lane / LP, h = lane % LP;
  int ix = slot, iy = slot + NS;
  float x[NR], y[NR];
#pragma unroll
  for (int f = 0; f < NR / 4; ++f) {
    const float4 a = ld4(sM + ix * LM + h * NR + 4 * f);
    const float4 b = ld4(sM + iy * LM + h * NR + 4 * f);
    x[4 * f] = a.x; x[4 * f + 1] = a.y; x[4 * f + 2] = a.z; x[4 * f + 3] = a.w;
    y[4 * f] = b.x; y[4 * f + 1] = b.y; y[4 * f + 2] = b.z; y[4 * f + 3] = b.w;
  }
  const int sweeps = jacobi_core<MP, NR>(x, y, ix, iy, conv);
  __syncwarp();
#pragma unroll
  for (int f = 0; f < NR / 4; ++f) {
    st4(sM + ix * LM + h * NR + 4 * f, make_float4(x[4 * f], x[4 * f + 1], x[4 * f + 2], x[4 * f + 3]));
    st4(sM + iy * LM + h * NR + 4 * f, make_float4(y[4 * f], y[4 * f + 1], y[4 * f + 2], y[4 * f + 3]));
  }
  __syncwarp();
  return sweeps;
}

// Chunk c of the panel stream (rows 32c .. 32c+31 of U, then of V) into buffer
// c & 1: one tensor copy of the box {32 rows, MP columns, 1 unit}, completing on
// bar[c & 1].  Columns m .. MP-1 lie outside the tensor and arrive as zeros.  In
// shared memory column j is a 128-byte row whose 16-byte pieces are permuted by
// the 128-byte swizzle: piece f sits at f ^ (j & 7).
// withhold: announce the bytes but issue no copy (the injected wait fault).  last:
// the second pass, the panel's last read (evict_first); the first pass keeps its
// lines in L2 (evict_last) for the second, which follows after the core SVD.
template <int NCU, int CHUNK>
SEED_DEV void issue_chunk(int c, float* sA, const CUtensorMap* tmU, const CUtensorMap* tmV, long long unit,
                          uint64_t* bar, bool withhold = false, bool last = false) {
  const int bb = c & 1;
  const bool isU = c < NCU;
  const int r0 = 32 * (isU ? c : c - NCU);
  if ((threadIdx.x & 31) == 0) {
    mbar_arrive_expect_tx(&bar[bb], (uint32_t)(CHUNK * 4));
    if (!withhold)
      tma_load_3d_hint(sA + bb * CHUNK, isU ? tmU : tmV, r0, 0, (int)unit, &bar[bb],
                       last ? l2_policy_evict_first() : l2_policy_evict_last());
  }
}

// Offset (in floats) of element e of column j in a swizzled chunk buffer.
SEED_DEV int swz(int j, int e) { return j * 32 + ((((e >> 2) ^ (j & 7)) << 2) | (e & 3)); }

// 16-bit factors.  Chunk c is copied as it is stored (lane l: 8 rows 8 (l & 3) ..
// of column 8 pass + (l >> 2), one 16-byte cp.async each) into staging buffer c & 1
// (the two take the place of float32 chunk buffer 1), then widened by the same
// lanes into float32 chunk buffer 0 in the swizzled layout of the tensor copies, so
// that the arithmetic below is the float32 path's.  Columns m .. MP-1 become zeros.
template <int DK, int DV, int MP, typename TS>
SEED_DEV void issue_chunk16(int c, float* sA, const FastParams& p, long long unit, int m) {
  constexpr int NCU = DK / 32, CHUNK = MP * 32;
  const int lane = threadIdx.x & 31, q = lane & 3;
  const bool isU = c < NCU;
  const int D = isU ? DK : DV;
  const int r0 = 32 * (isU ? c : c - NCU);
  const TS* src = static_cast<const TS*>(isU ? p.U : p.V) + unit * (long long)m * D + r0;
  TS* stg = reinterpret_cast<TS*>(sA + CHUNK) + (c & 1) * CHUNK;
#pragma unroll
  for (int pass = 0; pass < MP / 8; ++pass) {
    const int j = pass * 8 + (lane >> 2);
    if (j < m) cp_async16(stg + j * 32 + 8 * q, src + (long long)j * D + 8 * q);
  }
  cp_async_commit();
}

// Waits for chunk c (more: chunk c + 1 was issued after it) and widens it.
template <int MP, typename TS>
SEED_DEV void widen_chunk16(int c, float* sA, int m, bool more) {
  constexpr int CHUNK = MP * 32;
  if (more) cp_async_wait<1>();
  else cp_async_wait<0>();
  const int lane = threadIdx.x & 31, q = lane & 3;
  const TS* stg = reinterpret_cast<const TS*>(sA + CHUNK) + (c & 1) * CHUNK;
#pragma unroll
  for (int pass = 0; pass < MP / 8; ++pass) {
    const int j = pass * 8 + (lane >> 2);
    float lo[4] = {0.f, 0.f, 0.f, 0.f}, hi[4] = {0.f, 0.f, 0.f, 0.f};
    if (j < m) {
      fac_ld<TS, 4>(stg + j * 32 + 8 * q, lo);
      fac_ld<TS, 4>(stg + j * 32 + 8 * q + 4, hi);
    }
    st4(sA + j * 32 + (((2 * q) ^ (j & 7)) << 2), make_float4(lo[0], lo[1], lo[2], lo[3]));
    st4(sA + j * 32 + (((2 * q + 1) ^ (j & 7)) << 2), make_float4(hi[0], hi[1], hi[2], hi[3]));
  }
  __syncwarp();
}

// The next chunk of the stream: float32 factors wait for its tensor copy on the
// barrier of its buffer (uses[b]: phases of bar[b] completed so far; false on
// timeout, after waiting for the copies in flight); 16-bit factors widen it and
// issue chunk c + 2 into the staging buffer it leaves.  Returns the chunk's buffer
// through buf.
template <int DK, int DV, int MP, typename TS>
SEED_DEV bool next_chunk(int c, uint32_t (&uses)[2], float* sA, uint64_t* bar, const FastParams& p,
                         long long unit, int m, const float*& buf, uint64_t limit = kWaitLimitNs) {
  constexpr int NCH = (DK + DV) / 32, CHUNK = MP * 32;
  if constexpr (std::is_same<TS, float>::value) {
    const int bb = c & 1;
    const uint32_t ph = uses[bb] & 1u;
    if (!__all_sync(kFull, mbar_wait_bounded(&bar[bb], ph, limit))) {
      mbar_wait_bounded(&bar[bb], ph, kWaitLimitNs);
      if (c + 1 < NCH) mbar_wait_bounded(&bar[bb ^ 1], uses[bb ^ 1] & 1u, kWaitLimitNs);
      return false;
    }
    ++uses[bb];
    buf = sA + bb * CHUNK;
  } else {
    widen_chunk16<MP, TS>(c, sA, m, c + 1 < NCH);
    if (c + 2 < NCH) issue_chunk16<DK, DV, MP, TS>(c + 2, sA, p, unit, m);
    buf = sA;
  }
  return true;
}

// Tensor-core products in float32 accuracy: x = hi + lo with hi = tf32(x) and
// lo = tf32(x - hi), and a b ~ hi_a hi_b + hi_a lo_b + lo_a hi_b (the dropped
// lo_a lo_b is below 2^-21 of a b), each term one warp-level mma.sync m16n8k8 with
// float32 accumulation.
SEED_DEV void tf32_split(float x, uint32_t& hi, uint32_t& lo) {
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hi) : "f"(x));
  const float r = x - __uint_as_float(hi);
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(lo) : "f"(r));
}

SEED_DEV void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

SEED_DEV void mma3_tf32(float (&d)[4], const uint32_t (&ah)[4], const uint32_t (&al)[4], uint32_t bh0,
                        uint32_t bh1, uint32_t bl0, uint32_t bl1) {
  mma_tf32(d, ah, bl0, bl1);
  mma_tf32(d, al, bh0, bh1);
  mma_tf32(d, ah, bh0, bh1);
}

// Gram matrix of one panel, accumulated over its chunks c0 .. c1-1 as they arrive
// (chunk c + 2 is issued into a buffer once chunk c is read) with tensor-core tiles:
// G = P^T P as (MP x 32-row chunk) x (32-row chunk x MP) products, the upper block
// triangle only (m16n8 tiles with n-tile >= 2 m-tile), mirrored when written to Gs
// (row-major, stride LG).  The A operand of
// an m-tile is made of the B operands of n-tiles 2 mt and 2 mt + 1 (the same panel
// columns).  fold (KDA's U): entries weighted by P (true U = Diag(P) U).  Also
// checks the column scale.  Returns false if a copy did not arrive in time (after
// waiting for those in flight).
// Not inlined: both Grams use it, and one copy of the code keeps the kernel closer to
// the instruction cache.
template <bool KDA, int DK, int DV, int MP, int LG, typename TS>
__device__ __noinline__ bool gram_stream(int c0, int c1, bool fold, float* sA, const CUtensorMap* tmU,
                                         const CUtensorMap* tmV, const FastParams& p, long long unit, int m,
                                         uint64_t* bar, uint32_t (&uses)[2], const float* scl, float* Gs,
                                         bool& bad, bool fault) {
  constexpr int NCU = DK / 32, NCH = (DK + DV) / 32, CHUNK = MP * 32;
  constexpr int NT = MP / 8, MT = MP / 16;
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
  float acc[MT][NT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
  float mx[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) mx[nt] = 0.f;
#pragma unroll 1
  for (int c = c0; c < c1; ++c) {
    const float* buf;
    if (!next_chunk<DK, DV, MP, TS>(c, uses, sA, bar, p, unit, m, buf,
                                    (fault && c == c0) ? 0ull : kWaitLimitNs))
      return false;
    const int r0 = 32 * (c < NCU ? c : c - NCU);
#pragma unroll 1
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int row = ks * 8 + tq + 4 * h;
          float x = buf[swz(nt * 8 + gq, row)];
          if (KDA && fold) x *= scl[r0 + row];   // both operands carry P: P^2 in the product
          mx[nt] = fmaxf(mx[nt], fabsf(x));
          tf32_split(x, bh[nt][h], bl[nt][h]);
        }
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const uint32_t ah[4] = {bh[2 * mt][0], bh[2 * mt + 1][0], bh[2 * mt][1], bh[2 * mt + 1][1]};
        const uint32_t al[4] = {bl[2 * mt][0], bl[2 * mt + 1][0], bl[2 * mt][1], bl[2 * mt + 1][1]};
#pragma unroll
        for (int nt = 2 * mt; nt < NT; ++nt)
          mma3_tf32(acc[mt][nt], ah, al, bh[nt][0], bh[nt][1], bl[nt][0], bl[nt][1]);
      }
    }
    __syncwarp();   // every lane has read this chunk before the next copy overwrites it
    if (std::is_same<TS, float>::value && c + 2 < NCH) issue_chunk<NCU, CHUNK>(c + 2, sA, tmU, tmV, unit, bar);
  }
  // largest magnitude of column nt * 8 + gq, over the four lanes of the group
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float v = fmaxf(mx[nt], __shfl_xor_sync(kFull, mx[nt], 1));
    v = fmaxf(v, __shfl_xor_sync(kFull, v, 2));
    if (nt * 8 + gq < m && v > 0.f && (v < kColMin || v > kColMax)) bad = true;
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int nt = 2 * mt; nt < NT; ++nt) {
      const int row = mt * 16 + gq, col = nt * 8 + 2 * tq;
      Gs[row * LG + col] = acc[mt][nt][0];
      Gs[row * LG + col + 1] = acc[mt][nt][1];
      Gs[(row + 8) * LG + col] = acc[mt][nt][2];
      Gs[(row + 8) * LG + col + 1] = acc[mt][nt][3];
      if (nt >= 2 * mt + 2) {   // off the diagonal blocks: the transposed entries too
        Gs[col * LG + row] = acc[mt][nt][0];
        Gs[(col + 1) * LG + row] = acc[mt][nt][1];
        Gs[col * LG + row + 8] = acc[mt][nt][2];
        Gs[(col + 1) * LG + row + 8] = acc[mt][nt][3];
      }
    }
  }
  __syncwarp();
  return true;
}

// Shared memory.  Region A first holds two 32-row chunk buffers through which the
// panels stream (U chunks, then V chunks); after the V Gram it holds L_v, then M
// in place of it and the selected left vectors X, and at the end the chunks of the
// panels again.  L_u has its own region, used from the U Gram until the small
// right factors T_u and T_v replace it; the two chunk barriers come last.  Region A
// must start on a 1 KB boundary (the 128-byte swizzle of the tensor copies).
template <int FORM, int DK, int DV, int MP>
struct FastLayout {
  static constexpr int CHUNK = MP * 32;                         // one swizzled chunk (MP x 128 B)
  static constexpr int LG = MP + 4, LX = MP + 1;
  static constexpr int SL = (FORM == SEED_KDA ? DK : MP);
  static constexpr int OFF_M = 0, OFF_X = MP * LG;
  static constexpr int A_CH = 2 * CHUNK, A_B = OFF_X + kFastMaxR * LX;
  static constexpr int A = ((A_CH > A_B ? A_CH : A_B) + 3) & ~3;
  static constexpr int LU = A;                                  // L_u (MP x LG), then T_u | T_v
  static constexpr int LU_N = (MP * LG > 2 * MP * kFastMaxR ? MP * LG : 2 * MP * kFastMaxR);
  static constexpr int SMALL = LU + LU_N;
  static constexpr int FLOATS = SMALL + 4 * MP + SL;           // nu nv du nrm, scl
  static constexpr size_t BAR_OFF = FLOATS * sizeof(float) + kFastMaxR * sizeof(int);   // 8-byte aligned
  static constexpr size_t bytes = BAR_OFF + 2 * sizeof(uint64_t);
  // a block whose dynamic shared memory may start anywhere re-aligns region A
  static constexpr size_t bytes_aligned = bytes + 1024;
  static_assert(BAR_OFF % 8 == 0, "barrier alignment");
};

// Chunks 0 and 1 of a stream.
template <int DK, int DV, int MP, typename TS>
SEED_DEV void start_stream(float* sA, const CUtensorMap* tmU, const CUtensorMap* tmV, const FastParams& p,
                           long long unit, int m, uint64_t* bar, bool withhold = false, bool last = false) {
  if constexpr (std::is_same<TS, float>::value) {
    issue_chunk<DK / 32, MP * 32>(0, sA, tmU, tmV, unit, bar, withhold, last);
    issue_chunk<DK / 32, MP * 32>(1, sA, tmU, tmV, unit, bar, false, last);
  } else {
    issue_chunk16<DK, DV, MP, TS>(0, sA, p, unit, m);
    issue_chunk16<DK, DV, MP, TS>(1, sA, p, unit, m);
  }
}

// One unit (index idx within the call's scope) of the fast compression, by the
// whole warp, with the shared memory of FastLayout at sA (1 KB aligned) and the two
// chunk barriers bar; uses[b] counts the completed phases of bar[b] (the barriers
// may serve earlier units of the same warp).  The tensor maps describe float32
// factors; with 16-bit factors they are unused.  Returns false when a bulk copy
// did not arrive in time (the warp should then stop).
template <int FORM, int DK, int DV, int MP, typename TS>
SEED_DEV bool compress_fast_unit(const FastParams& p, const CUtensorMap& tmU, const CUtensorMap& tmV, int idx,
                                 float* sA, uint64_t* bar, uint32_t (&uses)[2]) {
  using Lay = FastLayout<FORM, DK, DV, MP>;
  constexpr bool KDA = FORM == SEED_KDA;
  constexpr int LG = Lay::LG, LX = Lay::LX, CHUNK = Lay::CHUNK;
  constexpr int NCU = DK / 32, NCV = DV / 32, NCH = NCU + NCV;
  float* sM = sA + Lay::OFF_M;       // L_v, then M (column-major), then T_u | T_v
  float* sX = sA + Lay::OFF_X;       // R x LX
  float* sLu = sA + Lay::LU;
  float* nu = sA + Lay::SMALL;
  float* nv = nu + MP;
  float* du = nv + MP;
  float* nrm = du + MP;
  float* scl = nrm + MP;
  int* sel = reinterpret_cast<int*>(scl + Lay::SL);

  const int lane = threadIdx.x;
  const int m = p.R + p.W;
  const int per = p.layer < 0 ? p.L * p.H : p.H;
  const int b = idx / per, rest = idx - b * per;
  const long long unit =
      p.layer < 0 ? (long long)idx : ((long long)b * p.L + p.layer) * p.H + rest;
  if (p.ncols[unit] != m) return true;   // not due (the fallback kernel flags invalid counts)

  // 1. the panels stream through two chunk buffers, 32 rows of every column per
  //    chunk (one tensor copy each); Gram rows accumulate in registers
  fence_proxy_async_smem();   // an earlier unit may have written the buffers with ordinary stores
  __syncwarp();
  for (int e = lane; e < p.slen; e += 32) scl[e] = p.scale[unit * p.slen + e];
  __syncwarp();
  // the injected wait fault (float32 factors: the only ones copied with mbarriers)
  const bool fault = std::is_same<TS, float>::value && wait_fault_injected(p.status);
  start_stream<DK, DV, MP, TS>(sA, &tmU, &tmV, p, unit, m, bar, fault);
  bool bad = false;   // ill-conditioned or badly scaled: left for the Householder kernel
  // U: chunks 0 .. NCU-1, then its Cholesky factor (to its own region); a copy that
  // does not arrive here leaves the unit untouched at R + W columns, for the
  // Householder kernel
  if (!gram_stream<KDA, DK, DV, MP, LG, TS>(0, NCU, true, sA, &tmU, &tmV, p, unit, m, bar, uses, scl, sLu,
                                            bad, fault)) {
    if (lane == 0) raise_flag(p.status, SEED_FLAG_TIMEOUT);
    return false;
  }
  // equilibrated Cholesky in shared memory; nrm is free until after both
  // factorisations and serves as its scratch
  cholesky_wide<MP, LG>(sLu, m, nu, nrm, bad);
  // V: chunks NCU .. NCH-1; L_v over the chunk buffers once the last one is read
  if (!gram_stream<KDA, DK, DV, MP, LG, TS>(NCU, NCH, false, sA, &tmU, &tmV, p, unit, m, bar, uses, scl, sM,
                                            bad, false)) {
    if (lane == 0) raise_flag(p.status, SEED_FLAG_TIMEOUT);
    return false;
  }
  cholesky_wide<MP, LG>(sM, m, nv, nrm, bad);
  if (__any_sync(kFull, bad)) {
    if (lane == 0) atomicAdd(p.status + 6, 1u);
    return true;
  }

  // D_u, D_v: true column norms (GDN / Mamba-2: with the lazy scale gamma_j; D_v is
  // nv); the core is formed with w_k = D_u D_v / max(D_u D_v) so that its entries
  // are of order one, and its singular values are scaled back by wmax
  float wl = 0.f;
  if (lane < MP) {
    const float gj = (KDA || lane >= m) ? 1.f : scl[lane];
    const float a = nu[lane] * gj;
    du[lane] = a;
    wl = a * nv[lane];
  }
  const float wmax = warp_max(wl);
  const float winv = wmax > 0.f ? 1.f / wmax : 0.f;
  __syncwarp();

  // 2. core M = L_u^T diag(w) L_v in place of L_v, column j in lane j:
  //    M[i][j] = sum_{k >= max(i, j)} L_u[k][i] w_k L_v[k][j]   (L_u, L_v lower triangular)
  {
    const int j = lane < MP ? lane : 0;
    float acc[MP];
#pragma unroll
    for (int i = 0; i < MP; ++i) acc[i] = 0.f;
#pragma unroll 2
    for (int k = 0; k < MP; ++k) {
      const float cf = sM[k * LG + j] * (du[k] * nv[k] * winv);
#pragma unroll
      for (int i4 = 0; i4 < MP; i4 += 4) {
        const float4 l = ld4(sLu + k * LG + i4);
        acc[i4] = fmaf(cf, l.x, acc[i4]);
        acc[i4 + 1] = fmaf(cf, l.y, acc[i4 + 1]);
        acc[i4 + 2] = fmaf(cf, l.z, acc[i4 + 2]);
        acc[i4 + 3] = fmaf(cf, l.w, acc[i4 + 3]);
      }
    }
    __syncwarp();   // every lane has read L_v before M overwrites it
    if (lane < MP) {
#pragma unroll
      for (int i = 0; i < MP; i += 4) st4(sM + lane * LG + i, make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]));
    }
  }
  __syncwarp();

  // 3. one-sided Jacobi on M
  bool converged;
  const int sweeps = jacobi_regs<MP, LG>(sM, converged);
  if (lane == 0) {
    atomicAdd(p.status + 1, (uint32_t)sweeps);
    atomicAdd(p.status + 5, 1u);
    if (!converged) raise_flag(p.status, SEED_FLAG_NOCONVERGE);
  }

  // 4. singular values (of the scaled core) = column norms of M Z; the R largest
  if (lane < MP) {
    float s2 = 0.f;
#pragma unroll
    for (int r = 0; r < MP; r += 4) {
      const float4 x = ld4(sM + lane * LG + r);
      s2 += dot4(x, x);
    }
    nrm[lane] = sqrtf(s2);
  }
  __syncwarp();
  if (lane < MP) {
    const float s = nrm[lane];
    int rank = 0;
    for (int k = 0; k < MP; ++k) {
      const float t = nrm[k];
      rank += (t > s) || (t == s && k < lane);
    }
    if (rank < p.R) sel[rank] = lane;
  }
  __syncwarp();
  const float smax = warp_max(lane < MP ? nrm[lane] : 0.f);
  const float szero = (float)(DK > DV ? DK : DV) * 1.1920929e-7f * smax;

  // 4b. the selected left vectors x_r = (M Z)_{sel r} / sigma_r, stored [r][i].
  //     Columns whose squared norm the Jacobi judged negligible (below 1e-10 of
  //     the total) are left unrotated, so they need not be orthogonal to the
  //     others; when every selected sigma is above 1e-4 sigma_max none of them is
  //     such a column and the x_r are orthonormal as they are.  Otherwise they are
  //     orthonormalised in descending order (modified Gram-Schmidt, two passes;
  //     lane = row), so that the result below is exactly the projection of U V^T on
  //     their span; a vector that loses more than half its norm to the earlier ones
  //     adds no new direction and is dropped.
  float sk = 0.f;   // lane r < R: the scaled sigma kept for output column r (0: dropped)
  if (nrm[sel[p.R - 1]] > 1e-4f * smax) {
    for (int r = 0; r < p.R; ++r) {
      const int j = sel[r];
      const float sj = nrm[j];
      if (lane < MP) sX[r * LX + lane] = sM[j * LG + lane] / sj;
      if (lane == r) sk = sj;
    }
    __syncwarp();
  } else {
    for (int r = 0; r < p.R; ++r) {
      const int j = sel[r];
      const float sj = nrm[j];
      float x = (lane < MP && sj > szero) ? sM[j * LG + lane] / sj : 0.f;
#pragma unroll 1
      for (int pass = 0; pass < 2; ++pass) {
#pragma unroll 1
        for (int k = 0; k < r; ++k) {   // r is the same in every lane
          const float xk = lane < MP ? sX[k * LX + lane] : 0.f;
          const float d = group_sum<32>(x * xk);
          x = fmaf(-d, xk, x);
        }
      }
      const float nx = sqrtf(group_sum<32>(x * x));
      const bool keep = nx > 0.5f;
      x = keep ? x / nx : 0.f;
      if (lane < MP) sX[r * LX + lane] = x;
      if (lane == r) sk = keep ? sj : 0.f;
      __syncwarp();
    }
  }

  // 5. small right factors on the stored panels, lane k holding row k of both:
  //    with sigma_r = wmax * sk_r the true singular value,
  //      GDN / Mamba-2 (a per-column scale exists): unit columns, the scale = sigma
  //        U' = U_st T_u, T_u = diag(1 / nu) L_u^{-T} X_R
  //        V' = V_st T_v, T_v = D_u L_u X_R Sigma^{-1}
  //      KDA: balanced, Sigma^{1/2} on each side (the row products P applied to U'
  //        after the product, and reset to 1)
  //    then stored [k][r] (stride 16) over L_u: T_u first, T_v after it
  {
    float fu[kFastMaxR], fv[kFastMaxR];
#pragma unroll
    for (int r = 0; r < kFastMaxR; ++r) {
      const float sr = __shfl_sync(kFull, sk, r) * wmax;
      const bool zero = !(sr > 0.f) || r >= p.R;
      fu[r] = zero ? 0.f : (KDA ? sqrtf(sr) : 1.f);
      fv[r] = zero ? 0.f : (KDA ? rsqrtf(sr) : 1.f / sr);
    }
    const int k = lane < MP ? lane : 0;
    float bu[kFastMaxR], bv[kFastMaxR];
#pragma unroll
    for (int r = 0; r < kFastMaxR; ++r) {
      bu[r] = (lane < MP && r < p.R) ? sX[r * LX + k] * fu[r] : 0.f;
      bv[r] = 0.f;
    }
    // T_v rows: (L_u X_R^T)_k = sum_{i <= k} L_u[k][i] x_r[i]  (L_u[k][i] = 0 above the diagonal)
#pragma unroll 2
    for (int i = 0; i < MP; ++i) {
      const float l = sLu[k * LG + i];
#pragma unroll
      for (int r = 0; r < kFastMaxR; ++r) bv[r] = fmaf(l, sX[r * LX + i], bv[r]);
    }
    // T_u: back substitution with L_u^T by columns: once row kk is final, remove its
    // part from every row above it
#pragma unroll 1
    for (int kk = MP - 1; kk >= 0; --kk) {
      const float lkk = sLu[kk * LG + kk];
      const float rl = lkk != 0.f ? 1.f / lkk : 0.f;
      const float lk = sLu[kk * LG + k];   // L_u[kk][k], used by rows k < kk
#pragma unroll
      for (int r = 0; r < kFastMaxR; ++r) {
        if (lane == kk) bu[r] *= rl;
        const float tk = __shfl_sync(kFull, bu[r], kk);
        if (lane < kk) bu[r] = fmaf(-lk, tk, bu[r]);
      }
    }
    const float nk = lane < MP ? nu[k] : 0.f;
    const float rn = nk > 0.f ? 1.f / nk : 0.f;
    const float dk = lane < MP ? du[k] : 0.f;
    __syncwarp();   // every lane has read L_u
    if (lane < MP) {
#pragma unroll
      for (int r = 0; r < kFastMaxR; r += 4) {
        st4(sLu + k * kFastMaxR + r, make_float4(bu[r] * rn, bu[r + 1] * rn, bu[r + 2] * rn, bu[r + 3] * rn));
        st4(sLu + MP * kFastMaxR + k * kFastMaxR + r,
            make_float4(dk * bv[r] * fv[r], dk * bv[r + 1] * fv[r + 1], dk * bv[r + 2] * fv[r + 2],
                        dk * bv[r + 3] * fv[r + 3]));
      }
    }
    __syncwarp();
  }
  const float* sTu = sLu;
  const float* sTv = sLu + MP * kFastMaxR;

  // 6. U' = U_st T_u, then V' = V_st T_v: the panels stream through the chunk
  //    buffers again (read a moment ago, normally still in L2); lane = row of the
  //    chunk.  A chunk's rows are written after they were read and no other chunk
  //    holds them, so slots 0..R-1 can be overwritten in place.
  fence_proxy_async_smem();   // the chunk buffers were written with ordinary stores
  __syncwarp();
  start_stream<DK, DV, MP, TS>(sA, &tmU, &tmV, p, unit, m, bar, false, true);
  bool nonfinite = false;
  TS* Uo = static_cast<TS*>(p.U) + unit * (long long)m * DK;
  TS* Vo = static_cast<TS*>(p.V) + unit * (long long)m * DV;
#pragma unroll 1
  for (int c = 0; c < NCH; ++c) {
    const float* buf;
    if (!next_chunk<DK, DV, MP, TS>(c, uses, sA, bar, p, unit, m, buf)) {
      // slots of the chunks before c already hold results: the unit no longer
      // represents its state, so it is marked invalid (column count -1) instead of
      // being left at R + W for the Householder kernel, which would compress the
      // mixture; later calls flag it with SEED_FLAG_BADCOLS and leave it alone
      if (lane == 0) {
        if (c > 0) p.ncols[unit] = -1;
        raise_flag(p.status, SEED_FLAG_TIMEOUT);
      }
      return false;
    }
    const bool isU = c < NCU;
    const int r0 = 32 * (isU ? c : c - NCU);
    const float* T = isU ? sTu : sTv;
    // out (32 rows x 16) = chunk (32 rows x MP) T (MP x 16): m16n8k8 tiles, rows
    // mt * 16 + .., output columns nt * 8 + ..; columns >= m are zero in both
    const int gq = lane >> 2, tq = lane & 3;
    float acc[2][2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < MP / 8; ++ks) {
      const int k = ks * 8 + tq;
      uint32_t bh[2][2], bl[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        tf32_split(T[k * kFastMaxR + nt * 8 + gq], bh[nt][0], bl[nt][0]);
        tf32_split(T[(k + 4) * kFastMaxR + nt * 8 + gq], bh[nt][1], bl[nt][1]);
      }
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const int r = mt * 16 + gq;
        uint32_t ah[4], al[4];
        tf32_split(buf[swz(k, r)], ah[0], al[0]);
        tf32_split(buf[swz(k, r + 8)], ah[1], al[1]);
        tf32_split(buf[swz(k + 4, r)], ah[2], al[2]);
        tf32_split(buf[swz(k + 4, r + 8)], ah[3], al[3]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) mma3_tf32(acc[mt][nt], ah, al, bh[nt][0], bh[nt][1], bl[nt][0], bl[nt][1]);
      }
    }
    __syncwarp();   // every lane has read this chunk before the next copy overwrites it
    if (std::is_same<TS, float>::value && c + 2 < NCH)
      issue_chunk<NCU, CHUNK>(c + 2, sA, &tmU, &tmV, unit, bar, false, true);
    TS* out = (isU ? Uo : Vo) + r0;
    const int ld = isU ? DK : DV;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int r = mt * 16 + gq + 8 * hh;
        const float rowf = (KDA && isU) ? scl[r0 + r] : 1.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int q = nt * 8 + 2 * tq + e;
            if (q < p.R) {
              const float v = acc[mt][nt][2 * hh + e] * rowf;
              nonfinite |= !isfinite(fac_round<TS>(v));
              fac_st_stream<TS>(out + (long long)q * ld + r, v);
            }
          }
        }
      }
    }
  }
  const float sig_true = (lane < p.R) ? nrm[sel[lane]] * wmax : 0.f;
  if (p.sigma_out && lane < p.R) p.sigma_out[(long long)idx * p.R + lane] = sig_true;
  const float sk_lane = __shfl_sync(kFull, sk, lane & 15);
  for (int e = lane; e < p.slen; e += 32)   // e < R <= 16 happens only with e == lane
    p.scale[unit * p.slen + e] = (!KDA && e < p.R) ? sk_lane * wmax : 1.f;
  if (lane == 0) p.ncols[unit] = p.R;
  if (__any_sync(kFull, nonfinite) && lane == 0) raise_flag(p.status, SEED_FLAG_NONFINITE);
  return true;
}

// A factor array [units][m][D] (float32) as the tensor map the chunk copies use
// (seed_compress_fast.cu).
bool make_panel_map(CUtensorMap* tm, const float* base, int D, int m, long long units, int MP);

}  // namespace seed
