// seed_compress_wide.cuh -- the compression of units with 32 < R + W <= 64, R <= 32.
//
// "Shallow Encoding Emits Deep Memories", SEED figures & tables (thelatestinai.com),
// Figure 1(b): every W steps the factors are compressed back to rank R.  The same
// route as seed_compress_fast.cuh (Cholesky QR of the two panels, the core
// M = R_u R_v^T, one-sided Jacobi on M, the top-R reconstruction), for cores of up to
// 64 columns, one warp per unit:
//
//   1. the panels stream through two shared-memory chunk buffers (32 rows of 64
//      columns per tensor copy; columns R + W .. 63 arrive as zeros) and their Gram
//      matrices accumulate on the tensor cores (split TF32, float32 accuracy), only
//      the tiles of columns below R + W;
//   2. each Gram is equilibrated and factored by Cholesky in shared memory,
//      right-looking in panels of four columns, lane i holding rows i and i + 32 (the
//      panel in registers, then a rank-4 update of the rows below it);
//   3. M = L_u^T diag(w) L_v is formed in place of L_v, lane j holding columns j and
//      j + 32;
//   4. one-sided Jacobi on M in registers, one column pair per lane (jacobi_regs),
//      each lane holding the first R + W rows rounded up to 8 (the rest are zero);
//   5. the R leading left vectors X_R (re-orthonormalised when some of them belong to
//      numerically negligible columns), T_v = D_u L_u X_R Sigma^{-1} and, by back
//      substitution in place of L_u, T_u = diag(1/nu) L_u^{-T} X_R;
//   6. U' = U_st T_u, V' = V_st T_v on the tensor cores from the panels streamed again.
// A unit whose Cholesky meets a pivot below 1e-2, or whose stored columns are badly
// scaled, is left to the Householder kernel, as in the fast path.
#pragma once

#include "seed_compress_fast.cuh"

namespace seed {

constexpr int kWideMP = 64;
constexpr int kWideMaxR = 32;

// Shared memory of one unit (floats).  Region A holds the two chunk buffers, then the
// V Gram, L_v and M in place (stride LG), then the transposed left vectors X_R^T
// (stride XS); region LU holds the U Gram and L_u, then T_u (columns 0..31 of each row)
// and T_v (columns 32..63).  Region A starts on a 1 KB boundary (128-byte swizzle).
template <int FORM, int DK, int DV>
struct WideLayout {
  static constexpr int MP = kWideMP;
  static constexpr int CHUNK = MP * 32;
  // 68 floats: rows start on 16 bytes, and 128-bit accesses of 8 lanes to 8 rows fall
  // on distinct banks (68 = 4 mod 32)
  static constexpr int LG = MP + 4;
  static constexpr int XS = kWideMaxR + 4;
  static constexpr int A = (2 * CHUNK > MP * LG ? 2 * CHUNK : MP * LG);
  static constexpr int LU = A;
  static constexpr int SMALL = LU + MP * LG;
  static constexpr int SL = FORM == SEED_KDA ? DK : MP;
  // nu nv du wk sg ninv (6 x MP), fu fv (2 x 32), scl
  static constexpr int FLOATS = SMALL + 6 * MP + 2 * kWideMaxR + SL;
  static constexpr size_t BAR_OFF = (FLOATS * sizeof(float) + kWideMaxR * sizeof(int) + 7) & ~size_t(7);
  static constexpr size_t bytes = BAR_OFF + 2 * sizeof(uint64_t);
  static_assert(MP * XS <= A, "the transposed left vectors fit region A");
  static_assert(LG % 32 == 4, "bank layout of the row stride");
};

// Gram matrix P^T P of one panel (chunks c0 .. c1-1, streamed as in gram_stream) into
// Gs (row-major, stride LG, both triangles), with m16n8k8 tiles of the upper block
// triangle whose columns lie below m (the rest is zero: those columns are).  fold
// (KDA's U): entries weighted by P.  Checks the column scale.  Returns false if a copy
// did not arrive in time (after waiting for those in flight).
// Not inlined (both Grams use it): one copy of the code keeps the kernel closer to the
// instruction cache.
template <bool KDA, int DK, int DV, int MP, int LG, typename TS>
__device__ __noinline__ bool gram_wide(int c0, int c1, bool fold, float* sA, const CUtensorMap* tmU, const CUtensorMap* tmV,
                        const FastParams& p, long long unit, int m, uint64_t* bar, uint32_t (&uses)[2],
                        const float* scl, float* Gs, bool& bad, bool fault) {
  constexpr int NCU = DK / 32, NCH = (DK + DV) / 32, CHUNK = MP * 32;
  constexpr int NT = MP / 8, MT = MP / 16;
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
  const int nt_end = (m + 7) >> 3;
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
    if (!next_chunk<DK, DV, MP, TS>(c, uses, sA, bar, p, unit, m, buf, (fault && c == c0) ? 0ull : kWaitLimitNs))
      return false;
    const int r0 = 32 * (c < NCU ? c : c - NCU);
#pragma unroll 1
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          bh[nt][h] = bl[nt][h] = 0u;
          if (nt < nt_end) {
            const int row = ks * 8 + tq + 4 * h;
            float x = buf[swz(nt * 8 + gq, row)];
            if (KDA && fold) x *= scl[r0 + row];   // both operands carry P: P^2 in the product
            mx[nt] = fmaxf(mx[nt], fabsf(x));
            tf32_split(x, bh[nt][h], bl[nt][h]);
          }
        }
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        if (2 * mt >= nt_end) continue;
        const uint32_t ah[4] = {bh[2 * mt][0], bh[2 * mt + 1][0], bh[2 * mt][1], bh[2 * mt + 1][1]};
        const uint32_t al[4] = {bl[2 * mt][0], bl[2 * mt + 1][0], bl[2 * mt][1], bl[2 * mt + 1][1]};
#pragma unroll
        for (int nt = 2 * mt; nt < NT; ++nt)
          if (nt < nt_end) mma3_tf32(acc[mt][nt], ah, al, bh[nt][0], bh[nt][1], bl[nt][0], bl[nt][1]);
      }
    }
    __syncwarp();   // every lane has read this chunk before the next copy overwrites it
    if (std::is_same<TS, float>::value && c + 2 < NCH) issue_chunk<NCU, CHUNK>(c + 2, sA, tmU, tmV, unit, bar);
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float v = fmaxf(mx[nt], __shfl_xor_sync(kFull, mx[nt], 1));
    v = fmaxf(v, __shfl_xor_sync(kFull, v, 2));
    if (nt * 8 + gq < m && v > 0.f && (v < kColMin || v > kColMax)) bad = true;
  }
  __syncwarp();   // the Gram may overwrite the chunk buffers (V's Gram does)
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

// One unit (index idx within the call's scope) of the wide compression, by the whole
// warp, with the shared memory of WideLayout at sA (1 KB aligned) and the two chunk
// barriers bar (uses[b]: completed phases of bar[b]).  Returns false when a bulk copy
// did not arrive in time.
template <int FORM, int DK, int DV, typename TS>
SEED_DEV bool compress_wide_unit(const FastParams& p, const CUtensorMap& tmU, const CUtensorMap& tmV, int idx,
                                 float* sA, uint64_t* bar, uint32_t (&uses)[2]) {
  using Lay = WideLayout<FORM, DK, DV>;
  constexpr bool KDA = FORM == SEED_KDA;
  constexpr int MP = Lay::MP, LG = Lay::LG, XS = Lay::XS, CHUNK = Lay::CHUNK;
  constexpr int NCU = DK / 32, NCV = DV / 32, NCH = NCU + NCV;
  constexpr int RPL = MP / 32;
  float* sM = sA;                    // V Gram, L_v, M, M Z (column j at j * LG)
  float* sXt = sA;                   // X_R^T: row i at i * XS, after M Z is read
  float* sLu = sA + Lay::LU;         // U Gram, L_u; then T_u | T_v
  float* nu = sA + Lay::SMALL;
  float* nv = nu + MP;
  float* du = nv + MP;
  float* wk = du + MP;
  float* sg = wk + MP;
  float* ninv = sg + MP;
  float* fu = ninv + MP;
  float* fv = fu + kWideMaxR;
  float* scl = fv + kWideMaxR;
  int* sel = reinterpret_cast<int*>(scl + Lay::SL);

  const int lane = threadIdx.x;
  const int m = p.R + p.W;
  const int R = p.R;
  const int per = p.layer < 0 ? p.L * p.H : p.H;
  const int b = idx / per, rest = idx - b * per;
  const long long unit = p.layer < 0 ? (long long)idx : ((long long)b * p.L + p.layer) * p.H + rest;
  if (p.ncols[unit] != m) return true;   // not due (the fallback kernel flags invalid counts)

  // 1-2. Grams on the tensor cores as the panels stream, then Cholesky in shared memory
  fence_proxy_async_smem();   // an earlier unit may have written the buffers with ordinary stores
  __syncwarp();
  for (int e = lane; e < p.slen; e += 32) scl[e] = p.scale[unit * p.slen + e];
  __syncwarp();
  const bool fault = std::is_same<TS, float>::value && wait_fault_injected(p.status);
  start_stream<DK, DV, MP, TS>(sA, &tmU, &tmV, p, unit, m, bar, fault);
  bool bad = false;
  if (!gram_wide<KDA, DK, DV, MP, LG, TS>(0, NCU, true, sA, &tmU, &tmV, p, unit, m, bar, uses, scl, sLu, bad,
                                          fault)) {
    if (lane == 0) raise_flag(p.status, SEED_FLAG_TIMEOUT);
    return false;
  }
  cholesky_wide<MP, LG>(sLu, m, nu, ninv, bad);
  if (!gram_wide<KDA, DK, DV, MP, LG, TS>(NCU, NCH, false, sA, &tmU, &tmV, p, unit, m, bar, uses, scl, sM, bad,
                                          false)) {
    if (lane == 0) raise_flag(p.status, SEED_FLAG_TIMEOUT);
    return false;
  }
  cholesky_wide<MP, LG>(sM, m, nv, ninv, bad);
  if (__any_sync(kFull, bad)) {
    if (lane == 0) atomicAdd(p.status + 6, 1u);
    return true;
  }

  // D_u (true U column norms: stored norm x lazy scale for GDN / Mamba-2) and the core
  // weights w_k = D_u D_v / max(D_u D_v), so that M's entries are of order one
  float wl = 0.f;
#pragma unroll
  for (int h = 0; h < RPL; ++h) {
    const int k = lane + 32 * h;
    const float gj = (KDA || k >= m) ? 1.f : scl[k];
    const float a = nu[k] * gj;
    du[k] = a;
    wl = fmaxf(wl, a * nv[k]);
  }
  const float wmax = warp_max(wl);
  const float winv = wmax > 0.f ? 1.f / wmax : 0.f;
  __syncwarp();
#pragma unroll
  for (int h = 0; h < RPL; ++h) {
    const int k = lane + 32 * h;
    wk[k] = du[k] * nv[k] * winv;
  }
  __syncwarp();

  // 3. M = L_u^T diag(w) L_v in place of L_v, column j = lane + 32 h in pass h:
  //    M[i][j] = sum_{k >= max(i, j)} L_u[k][i] w_k L_v[k][j].  Pass h reads rows
  //    k >= 32 h of L_v (L_v[k][j] = 0 for k < j) and overwrites rows 32 h .. 32 h + 31
  //    (the buffer row j holds M's column j) only after every lane has read them.
#pragma unroll 1
  for (int h = 0; h < RPL; ++h) {
    const int j = lane + 32 * h;
    float acc[MP];
#pragma unroll
    for (int i = 0; i < MP; ++i) acc[i] = 0.f;
#pragma unroll 1
    for (int k = 32 * h; k < m; ++k) {
      const float cf = sM[k * LG + j] * wk[k];
#pragma unroll
      for (int i4 = 0; i4 < MP; i4 += 4) {
        if (i4 <= k) {   // L_u[k][i] = 0 for i > k
          const float4 l = ld4(sLu + k * LG + i4);
          acc[i4] = fmaf(cf, l.x, acc[i4]);
          acc[i4 + 1] = fmaf(cf, l.y, acc[i4 + 1]);
          acc[i4 + 2] = fmaf(cf, l.z, acc[i4 + 2]);
          acc[i4 + 3] = fmaf(cf, l.w, acc[i4 + 3]);
        }
      }
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < MP; i += 4) st4(sM + j * LG + i, make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]));
    __syncwarp();
  }

  // 4. one-sided Jacobi on M; its rows from m on are zero, so the lanes hold only the
  //    first m rounded up to 8 (one copy of the sweep code per row count; m is the
  //    same for every unit of a launch)
  bool converged;
  int sweeps;
  if (m <= 40) sweeps = jacobi_regs<MP, LG, 40>(sM, converged);
  else if (m <= 48) sweeps = jacobi_regs<MP, LG, 48>(sM, converged);
  else if (m <= 56) sweeps = jacobi_regs<MP, LG, 56>(sM, converged);
  else sweeps = jacobi_regs<MP, LG, 64>(sM, converged);
  if (lane == 0) {
    atomicAdd(p.status + 1, (uint32_t)sweeps);
    atomicAdd(p.status + 5, 1u);
    if (!converged) raise_flag(p.status, SEED_FLAG_NOCONVERGE);
  }

  // singular values (of the scaled core) = column norms of M Z; the R largest
#pragma unroll
  for (int h = 0; h < RPL; ++h) {
    const int j = lane + 32 * h;
    float s2 = 0.f;
#pragma unroll
    for (int r = 0; r < MP; r += 4) {
      const float4 x = ld4(sM + j * LG + r);
      s2 += dot4(x, x);
    }
    sg[j] = sqrtf(s2);
  }
  __syncwarp();
#pragma unroll
  for (int h = 0; h < RPL; ++h) {
    const int j = lane + 32 * h;
    const float s = sg[j];
    int rank = 0;
    for (int k = 0; k < MP; ++k) {
      const float t = sg[k];
      rank += (t > s) || (t == s && k < j);
    }
    if (rank < R) sel[rank] = j;
  }
  __syncwarp();
  const float smax = warp_max(fmaxf(sg[lane], sg[lane + 32]));
  const float szero = (float)(DK > DV ? DK : DV) * 1.1920929e-7f * smax;

  // 5. the selected left vectors x_r = (M Z)_{sel r} / sigma_r, transposed into
  //    X^T[i][r] over M Z once every lane holds its rows.  Columns whose squared norm
  //    the Jacobi judged negligible are left unrotated; when every selected sigma is
  //    above 1e-4 sigma_max none of them is such a column and the x_r are orthonormal
  //    as they are, otherwise they are orthonormalised in descending order (modified
  //    Gram-Schmidt, two passes), a vector that loses more than half its norm to the
  //    earlier ones being dropped.
  const bool clean = sg[sel[R - 1]] > 1e-4f * smax;
  {
    float xr[RPL][kWideMaxR];
#pragma unroll
    for (int r = 0; r < kWideMaxR; ++r) {
      const int j = r < R ? sel[r] : 0;
      const float sj = sg[j];
      const float inv = (r < R && sj > szero) ? 1.f / sj : 0.f;
#pragma unroll
      for (int h = 0; h < RPL; ++h) xr[h][r] = sM[j * LG + lane + 32 * h] * inv;
    }
    __syncwarp();
#pragma unroll
    for (int h = 0; h < RPL; ++h) {
      const int i = lane + 32 * h;
#pragma unroll
      for (int r = 0; r < kWideMaxR; r += 4)
        st4(sXt + i * XS + r, make_float4(xr[h][r], xr[h][r + 1], xr[h][r + 2], xr[h][r + 3]));
    }
    __syncwarp();
  }
  float sk = lane < R ? sg[sel[lane]] : 0.f;   // lane r < R: scaled sigma kept for column r (0: dropped)
  if (!clean) {
#pragma unroll 1
    for (int r = 0; r < R; ++r) {
      float x[RPL];
#pragma unroll
      for (int h = 0; h < RPL; ++h) x[h] = sXt[(lane + 32 * h) * XS + r];
#pragma unroll 1
      for (int pass = 0; pass < 2; ++pass) {
#pragma unroll 1
        for (int k = 0; k < r; ++k) {
          float xk[RPL], part = 0.f;
#pragma unroll
          for (int h = 0; h < RPL; ++h) {
            xk[h] = sXt[(lane + 32 * h) * XS + k];
            part = fmaf(x[h], xk[h], part);
          }
          const float d = group_sum<32>(part);
#pragma unroll
          for (int h = 0; h < RPL; ++h) x[h] = fmaf(-d, xk[h], x[h]);
        }
      }
      float n2 = 0.f;
#pragma unroll
      for (int h = 0; h < RPL; ++h) n2 = fmaf(x[h], x[h], n2);
      const float nx = sqrtf(group_sum<32>(n2));
      const bool keep = nx > 0.5f;
#pragma unroll
      for (int h = 0; h < RPL; ++h) sXt[(lane + 32 * h) * XS + r] = keep ? x[h] / nx : 0.f;
      if (lane == r && !keep) sk = 0.f;
      __syncwarp();
    }
  }

  // 6. small right factors, lane k holding rows k and k + 32, with sigma_r = wmax sk_r:
  //      GDN / Mamba-2 (a per-column scale exists): unit columns, the scale = sigma
  //        T_u = diag(1 / nu) L_u^{-T} X_R,   T_v = D_u L_u X_R Sigma^{-1}
  //      KDA: Sigma^{1/2} on each side (the row products P applied to U' after the
  //        product, and reset to 1)
  {
    const float sr = sk * wmax;
    const bool zero = !(sr > 0.f) || lane >= R;
    fu[lane] = zero ? 0.f : (KDA ? sqrtf(sr) : 1.f);
    fv[lane] = zero ? 0.f : (KDA ? rsqrtf(sr) : 1.f / sr);
  }
  __syncwarp();
  float bv[RPL][kWideMaxR];
#pragma unroll
  for (int h = 0; h < RPL; ++h)
#pragma unroll
    for (int r = 0; r < kWideMaxR; ++r) bv[h][r] = 0.f;
  // (L_u X_R)_k = sum_{i <= k} L_u[k][i] x_r[i]  (L_u[k][i] = 0 above the diagonal)
#pragma unroll 1
  for (int i4 = 0; i4 < m; i4 += 4) {
    float4 l4[RPL];
#pragma unroll
    for (int h = 0; h < RPL; ++h) l4[h] = ld4(sLu + (lane + 32 * h) * LG + i4);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float* xrow = sXt + (i4 + e) * XS;
#pragma unroll
      for (int r4 = 0; r4 < kWideMaxR; r4 += 4) {
        const float4 x = ld4(xrow + r4);
#pragma unroll
        for (int h = 0; h < RPL; ++h) {
          const float l = e == 0 ? l4[h].x : e == 1 ? l4[h].y : e == 2 ? l4[h].z : l4[h].w;
          bv[h][r4] = fmaf(l, x.x, bv[h][r4]);
          bv[h][r4 + 1] = fmaf(l, x.y, bv[h][r4 + 1]);
          bv[h][r4 + 2] = fmaf(l, x.z, bv[h][r4 + 2]);
          bv[h][r4 + 3] = fmaf(l, x.w, bv[h][r4 + 3]);
        }
      }
    }
  }
  // T_u: back substitution with L_u^T, in place of L_u (row kk of L_u is read for the
  // last time at step kk, then holds row kk of the solution in its columns 0..31)
  float bu[RPL][kWideMaxR];
#pragma unroll
  for (int h = 0; h < RPL; ++h) {
    const float* xrow = sXt + (lane + 32 * h) * XS;
#pragma unroll
    for (int r4 = 0; r4 < kWideMaxR; r4 += 4) {
      const float4 x = ld4(xrow + r4);
      const float4 f = ld4(fu + r4);
      bu[h][r4] = x.x * f.x;
      bu[h][r4 + 1] = x.y * f.y;
      bu[h][r4 + 2] = x.z * f.z;
      bu[h][r4 + 3] = x.w * f.w;
    }
  }
#pragma unroll 1
  for (int kk = m - 1; kk >= 0; --kk) {
    const float lkk = sLu[kk * LG + kk];
    const float rl = lkk != 0.f ? 1.f / lkk : 0.f;
    const int ho = kk >> 5, owner = kk & 31;
    float lk[RPL];
#pragma unroll
    for (int h = 0; h < RPL; ++h) {
      const int k = lane + 32 * h;
      lk[h] = k < kk ? sLu[kk * LG + k] : 0.f;   // L_u[kk][k]
    }
    __syncwarp();   // row kk of L_u is read; it now receives row kk of the solution
#pragma unroll
    for (int h = 0; h < RPL; ++h) {
      if (h == ho && lane == owner) {
#pragma unroll
        for (int r4 = 0; r4 < kWideMaxR; r4 += 4) {
          bu[h][r4] *= rl;
          bu[h][r4 + 1] *= rl;
          bu[h][r4 + 2] *= rl;
          bu[h][r4 + 3] *= rl;
          st4(sLu + kk * LG + r4, make_float4(bu[h][r4], bu[h][r4 + 1], bu[h][r4 + 2], bu[h][r4 + 3]));
        }
      }
    }
    __syncwarp();
#pragma unroll
    for (int r4 = 0; r4 < kWideMaxR; r4 += 4) {
      const float4 t = ld4(sLu + kk * LG + r4);
#pragma unroll
      for (int h = 0; h < RPL; ++h) {
        bu[h][r4] = fmaf(-lk[h], t.x, bu[h][r4]);
        bu[h][r4 + 1] = fmaf(-lk[h], t.y, bu[h][r4 + 1]);
        bu[h][r4 + 2] = fmaf(-lk[h], t.z, bu[h][r4 + 2]);
        bu[h][r4 + 3] = fmaf(-lk[h], t.w, bu[h][r4 + 3]);
      }
    }
  }
  __syncwarp();
  // final rows: T_u row k scaled by 1 / nu_k (columns 0..31), T_v row k = D_u[k] (L_u
  // X_R)_k (.) fv (columns 32..63); rows at or beyond m are zero
#pragma unroll
  for (int h = 0; h < RPL; ++h) {
    const int k = lane + 32 * h;
    const float rn = (k < m && nu[k] > 0.f) ? 1.f / nu[k] : 0.f;
    const float dk = k < m ? du[k] : 0.f;
#pragma unroll
    for (int r4 = 0; r4 < kWideMaxR; r4 += 4) {
      float4 t = ld4(sLu + k * LG + r4);
      if (k >= m) t = zero4();
      st4(sLu + k * LG + r4, make_float4(t.x * rn, t.y * rn, t.z * rn, t.w * rn));
      const float4 f = ld4(fv + r4);
      st4(sLu + k * LG + 32 + r4, make_float4(dk * bv[h][r4] * f.x, dk * bv[h][r4 + 1] * f.y,
                                              dk * bv[h][r4 + 2] * f.z, dk * bv[h][r4 + 3] * f.w));
    }
  }
  __syncwarp();

  // 7. U' = U_st T_u, then V' = V_st T_v: the panels stream through the chunk buffers
  //    again; lane = row of the chunk.  A chunk's rows are written after they were
  //    read and no other chunk holds them, so slots 0..R-1 can be overwritten in place.
  fence_proxy_async_smem();   // the chunk buffers were written with ordinary stores
  __syncwarp();
  start_stream<DK, DV, MP, TS>(sA, &tmU, &tmV, p, unit, m, bar, false, true);
  bool nonfinite = false;
  TS* Uo = static_cast<TS*>(p.U) + unit * (long long)m * DK;
  TS* Vo = static_cast<TS*>(p.V) + unit * (long long)m * DV;
  const int gq = lane >> 2, tq = lane & 3;
  const int ks_end = (m + 7) >> 3;
#pragma unroll 1
  for (int c = 0; c < NCH; ++c) {
    const float* buf;
    if (!next_chunk<DK, DV, MP, TS>(c, uses, sA, bar, p, unit, m, buf)) {
      // slots of the chunks before c already hold results: mark the unit invalid
      if (lane == 0) {
        if (c > 0) p.ncols[unit] = -1;
        raise_flag(p.status, SEED_FLAG_TIMEOUT);
      }
      return false;
    }
    const bool isU = c < NCU;
    const int r0 = 32 * (isU ? c : c - NCU);
    const float* T = sLu + (isU ? 0 : 32);
    // out (32 rows x R) = chunk (32 rows x MP) T (MP x R): m16n8k8 tiles, output
    // columns nt * 8 + .. below R, k-steps over the columns below m
    float acc[2][4][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
#pragma unroll 1
    for (int ks = 0; ks < ks_end; ++ks) {
      const int k = ks * 8 + tq;
      uint32_t bh[4][2], bl[4][2];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        bh[nt][0] = bh[nt][1] = bl[nt][0] = bl[nt][1] = 0u;
        if (nt * 8 < R) {
          tf32_split(T[k * LG + nt * 8 + gq], bh[nt][0], bl[nt][0]);
          tf32_split(T[(k + 4) * LG + nt * 8 + gq], bh[nt][1], bl[nt][1]);
        }
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
        for (int nt = 0; nt < 4; ++nt)
          if (nt * 8 < R) mma3_tf32(acc[mt][nt], ah, al, bh[nt][0], bh[nt][1], bl[nt][0], bl[nt][1]);
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
        for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int q = nt * 8 + 2 * tq + e;
            if (q < R) {
              const float v = acc[mt][nt][2 * hh + e] * rowf;
              nonfinite |= !isfinite(fac_round<TS>(v));
              fac_st_stream<TS>(out + (long long)q * ld + r, v);
            }
          }
        }
      }
    }
  }
  const float sig_true = (lane < R) ? sg[sel[lane]] * wmax : 0.f;
  if (p.sigma_out && lane < R) p.sigma_out[(long long)idx * R + lane] = sig_true;
  for (int e = lane; e < p.slen; e += 32)   // e < R <= 32 happens only with e == lane
    p.scale[unit * p.slen + e] = (!KDA && e < R) ? sk * wmax : 1.f;
  if (lane == 0) p.ncols[unit] = R;
  if (__any_sync(kFull, nonfinite) && lane == 0) raise_flag(p.status, SEED_FLAG_NONFINITE);
  return true;
}

// One warp per block and per unit of the scope, as compress_fast_kernel: the dynamic
// shared memory starts the block's window; a block that finds it off a 1 KB boundary
// leaves its unit to the Householder kernel.
template <int FORM, int DK, int DV, typename TS>
__global__ void __launch_bounds__(32)
    compress_wide_kernel(const FastParams p, const __grid_constant__ CUtensorMap tmU,
                         const __grid_constant__ CUtensorMap tmV) {
  using Lay = WideLayout<FORM, DK, DV>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  if (smem_addr(smem_raw) & 1023u) {
    if (threadIdx.x == 0) {
      const int per = p.layer < 0 ? p.L * p.H : p.H;
      const int b = blockIdx.x / per, rest = blockIdx.x - b * per;
      const long long unit = p.layer < 0 ? (long long)blockIdx.x : ((long long)b * p.L + p.layer) * p.H + rest;
      if (p.ncols[unit] == p.R + p.W) atomicAdd(p.status + 6, 1u);
    }
    return;
  }
  float* sA = reinterpret_cast<float*>(smem_raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem_raw + Lay::BAR_OFF);
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  __syncwarp();
  uint32_t uses[2] = {0u, 0u};
  compress_wide_unit<FORM, DK, DV, TS>(p, tmU, tmV, blockIdx.x, sA, bar, uses);
}

template <int FORM, int DK, int DV, typename TS>
static int launch_wide_t(const FastParams& p, int blocks, cudaStream_t st) {
  using Lay = WideLayout<FORM, DK, DV>;
  auto kern = compress_wide_kernel<FORM, DK, DV, TS>;
  static LaunchCache cache;
  int dev = 0;
  if (const int rc = cache.prepare(reinterpret_cast<const void*>(kern), Lay::bytes, &dev)) return rc;
  const long long units = (long long)p.B * p.L * p.H;
  const int m = p.R + p.W;
  CUtensorMap tmU, tmV;
  memset(&tmU, 0, sizeof(tmU));
  memset(&tmV, 0, sizeof(tmV));
  if (std::is_same<TS, float>::value &&
      (!make_panel_map(&tmU, static_cast<const float*>(p.U), DK, m, units, kWideMP) ||
       !make_panel_map(&tmV, static_cast<const float*>(p.V), DV, m, units, kWideMP)))
    return SEED_ERR_CUDA;
  kern<<<blocks, 32, Lay::bytes, st>>>(p, tmU, tmV);
  return cudaGetLastError() == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
}

// The wide compression launch for factor type TS (one translation unit per type).
template <typename TS>
int launch_wide_typed(const seed_dims& d, const FastParams& p, int blocks, cudaStream_t st) {
#define SEED_WIDE_DIMS(FORM)                                                                         \
  do {                                                                                               \
    if (d.d_k == 128 && d.d_v == 128) return launch_wide_t<FORM, 128, 128, TS>(p, blocks, st);       \
    if (d.d_k == 128 && d.d_v == 64) return launch_wide_t<FORM, 128, 64, TS>(p, blocks, st);         \
    if (d.d_k == 64 && d.d_v == 128) return launch_wide_t<FORM, 64, 128, TS>(p, blocks, st);         \
    if (d.d_k == 64 && d.d_v == 64) return launch_wide_t<FORM, 64, 64, TS>(p, blocks, st);           \
    return SEED_ERR_SHAPE;                                                                           \
  } while (0)
  switch (d.form) {
    case SEED_GDN: SEED_WIDE_DIMS(SEED_GDN);
    case SEED_KDA: SEED_WIDE_DIMS(SEED_KDA);
    case SEED_MAMBA2: SEED_WIDE_DIMS(SEED_MAMBA2);
  }
#undef SEED_WIDE_DIMS
  return SEED_ERR_INVALID_ARG;
}

int launch_wide_f32(const seed_dims& d, const FastParams& p, int blocks, cudaStream_t st);
int launch_wide_f16(const seed_dims& d, const FastParams& p, int blocks, cudaStream_t st);
int launch_wide_bf16(const seed_dims& d, const FastParams& p, int blocks, cudaStream_t st);

}  // namespace seed
