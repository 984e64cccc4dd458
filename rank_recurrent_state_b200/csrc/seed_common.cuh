// seed_common.cuh -- device helpers shared by the libseed kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <type_traits>

#include "../../include/seed.h"
#include "seed_launch.h"

#define SEED_DEV __device__ __forceinline__

namespace seed {

constexpr int kWarp = 32;

// ------------------------------------------------------------------ status word
SEED_DEV void raise_flag(uint32_t* status, uint32_t flag) { atomicOr(status, flag); }

// Workspace word (32-bit index from the status word) that, when nonzero, makes the
// kernels with bounded copy waits fail their first wait on purpose: each warp
// (decode) or block (fast compression) withholds its first bulk copy and gives up
// on it at once.  No copy is then in flight when the wait fails.  Set only by
// seed_debug_wait_fault, for the tests of the timeout path.
constexpr int kWsWaitFaultWord = 8;
static_assert(kWsWaitFaultWord == kWsWaitFaultWordHost, "one workspace layout");
SEED_DEV bool wait_fault_injected(const uint32_t* status) {
  return *reinterpret_cast<const volatile uint32_t*>(status + kWsWaitFaultWord) != 0u;
}

// Programmatic dependent launch (sm_90 and later).  griddep_wait: block until the
// grids this launch depends on have completed and their writes are visible (returns
// at once for a launch made without the programmatic-serialization attribute).
// griddep_launch_dependents: let the launch that depends on this grid begin; its
// blocks take SM slots as this grid's blocks retire.
SEED_DEV void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
SEED_DEV void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ vector helpers
SEED_DEV float4 ld_stream4(const float* p) { return __ldcs(reinterpret_cast<const float4*>(p)); }
SEED_DEV float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
SEED_DEV void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
SEED_DEV void st_stream4(float* p, float4 v) { __stcs(reinterpret_cast<float4*>(p), v); }
SEED_DEV float dot4(float4 a, float4 b) { return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w; }
SEED_DEV float4 mul4(float4 a, float4 b) { return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w); }
SEED_DEV float4 fma4(float s, float4 x, float4 y) {
  return make_float4(fmaf(s, x.x, y.x), fmaf(s, x.y, y.y), fmaf(s, x.z, y.z), fmaf(s, x.w, y.w));
}
SEED_DEV float4 zero4() { return make_float4(0.f, 0.f, 0.f, 0.f); }
SEED_DEV bool finite4(float4 v) {
  return isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w);
}

// ------------------------------------------------------------------ factor storage
// U and V hold float32 or 16-bit values (seed_factors); every kernel computes in
// float32, converting when it reads a factor and rounding to nearest, ties to even,
// when it writes one.
SEED_DEV float fac_to_f(float x) { return x; }
SEED_DEV float fac_to_f(__half x) { return __half2float(x); }
SEED_DEV float fac_to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
SEED_DEV T fac_from_f(float x) {
  if constexpr (std::is_same<T, __half>::value) return __float2half_rn(x);
  else if constexpr (std::is_same<T, __nv_bfloat16>::value) return __float2bfloat16_rn(x);
  else return x;
}

// One factor value stored with the streaming hint (evict first: not read again soon).
template <typename T>
SEED_DEV void fac_st_stream(T* p, float x) {
  if constexpr (std::is_same<T, float>::value) __stcs(p, x);
  else *p = fac_from_f<T>(x);
}

// The value x has once stored as T.
template <typename T>
SEED_DEV float fac_round(float x) { return fac_to_f(fac_from_f<T>(x)); }

// P consecutive factor values (P = 1, 2, 4) at p, aligned to P * sizeof(T).
template <typename T, int P>
SEED_DEV void fac_ld(const T* p, float (&e)[P]) {
  static_assert(P == 1 || P == 2 || P == 4, "P");
  if constexpr (std::is_same<T, float>::value) {
    if constexpr (P == 4) {
      const float4 t = *reinterpret_cast<const float4*>(p);
      e[0] = t.x; e[1] = t.y; e[2] = t.z; e[3] = t.w;
    } else if constexpr (P == 2) {
      const float2 t = *reinterpret_cast<const float2*>(p);
      e[0] = t.x; e[1] = t.y;
    } else {
      e[0] = *p;
    }
  } else {
    using W = typename std::conditional<P == 4, uint2, typename std::conditional<P == 2, uint32_t, uint16_t>::type>::type;
    const W raw = *reinterpret_cast<const W*>(p);
    T t[P];
    memcpy(t, &raw, sizeof(raw));
#pragma unroll
    for (int i = 0; i < P; ++i) e[i] = fac_to_f(t[i]);
  }
}

template <typename T, int P>
SEED_DEV void fac_st(T* p, const float (&e)[P]) {
  static_assert(P == 1 || P == 2 || P == 4, "P");
  if constexpr (std::is_same<T, float>::value) {
    if constexpr (P == 4) *reinterpret_cast<float4*>(p) = make_float4(e[0], e[1], e[2], e[3]);
    else if constexpr (P == 2) *reinterpret_cast<float2*>(p) = make_float2(e[0], e[1]);
    else *p = e[0];
  } else {
    using W = typename std::conditional<P == 4, uint2, typename std::conditional<P == 2, uint32_t, uint16_t>::type>::type;
    T t[P];
#pragma unroll
    for (int i = 0; i < P; ++i) t[i] = fac_from_f<T>(e[i]);
    W raw;
    memcpy(&raw, t, sizeof(raw));
    *reinterpret_cast<W*>(p) = raw;
  }
}

SEED_DEV float4 fac_ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
template <typename T>
SEED_DEV float4 fac_ld4(const T* p) {
  float e[4];
  fac_ld<T, 4>(p, e);
  return make_float4(e[0], e[1], e[2], e[3]);
}

template <int WIDTH>
SEED_DEV float group_sum(float x) {
#pragma unroll
  for (int off = WIDTH / 2; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

SEED_DEV float group_sum_rt(float x, int width) {
  for (int off = width / 2; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// ------------------------------------------------------------------ Philox4x32-10
// Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3" (SC'11):
// per round, two 32x32->64 products of counter words 0 and 2 by the round
// multipliers; the high halves are xor-ed with the other counter word and a key
// word; the key advances by the Weyl constants between rounds.
SEED_DEV uint4 philox4x32_10(uint4 ctr, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * ctr.x, hi0 = __umulhi(0xD2511F53u, ctr.x);
    const uint32_t lo1 = 0xCD9E8D57u * ctr.z, hi1 = __umulhi(0xCD9E8D57u, ctr.z);
    ctr = make_uint4(hi1 ^ ctr.y ^ k0, lo1, hi0 ^ ctr.w ^ k1, lo0);
  }
  return ctr;
}

// (x + 1/2) 2^-32: exact in double, strictly inside (0, 1).
SEED_DEV double word_to_unit(uint32_t x) { return ((double)x + 0.5) * 2.3283064365386963e-10; }

// Box-Muller on the word pairs (w0, w1), (w2, w3) of one Philox block -> 4 normals.
SEED_DEV void block_normals(uint4 w, double z[4]) {
  const double two_pi = 6.283185307179586;
  const double r0 = sqrt(__dmul_rn(-2.0, log(word_to_unit(w.x))));
  const double a0 = __dmul_rn(two_pi, word_to_unit(w.y));
  const double r1 = sqrt(__dmul_rn(-2.0, log(word_to_unit(w.z))));
  const double a1 = __dmul_rn(two_pi, word_to_unit(w.w));
  z[0] = __dmul_rn(r0, cos(a0));
  z[1] = __dmul_rn(r0, sin(a0));
  z[2] = __dmul_rn(r1, cos(a1));
  z[3] = __dmul_rn(r1, sin(a1));
}

SEED_DEV void block_uniforms(uint4 w, double u[4]) {
  u[0] = word_to_unit(w.x);
  u[1] = word_to_unit(w.y);
  u[2] = word_to_unit(w.z);
  u[3] = word_to_unit(w.w);
}

// ------------------------------------------------------------------ one-sided Jacobi
// Hestenes one-sided Jacobi SVD of an n_rows x n_cols matrix A held column-major
// in shared memory (column j at A + j * lda), accumulating the right rotations in
// Z (n_cols x n_cols, column-major, ldz).  On return the columns of A are mutually
// orthogonal (A_out = A_in Z), so sigma_j = ||A_out[:, j]||.
//
// Pairs are visited in the round-robin tournament order: n_cols/2 disjoint pairs
// per round, n_cols - 1 rounds per sweep, every pair once per sweep.  A pair is
// rotated when |x^T y| > tol sqrt(x^T x y^T y), with the rotation of Rutishauser:
// zeta = (y^T y - x^T x) / (2 x^T y), t = sign(zeta) / (|zeta| + sqrt(1 + zeta^2)),
// c = 1 / sqrt(1 + t^2), s = c t, x <- c x - s y, y <- s x + c y.  Iterates until a
// sweep rotates nothing or `max_sweeps` sweeps ran (then returns false).
//
// n_cols must be even (callers pad with a zero column).  Called by all threads of
// the block; each pair is handled by a group of G lanes (G a power of two <= 32).
//
// Columns whose squared norm is below tiny_rel ||A||_F^2 are treated as zero:
// their pairs are not rotated.  Such columns are rounding noise (or exact zeros)
// where n_cols exceeds the rank, and a relative threshold alone would keep
// rotating them for ever; their contribution is below sqrt(tiny_rel) ||A||_F.
// Returns the number of sweeps run (max_sweeps + 1 if it did not converge).
template <int NT>
__device__ int jacobi_svd(float* A, int lda, int n_rows, float* Z, int ldz, int n_cols, float tol,
                          int max_sweeps, float* s_red, float tiny_rel) {
  const int tid = threadIdx.x;
  const int npairs = n_cols / 2;
  int G = 32;
  while (G > 1 && G * npairs > NT) G >>= 1;
  const int groups = NT / G;
  const int grp = tid / G, gl = tid % G;

  float f2 = 0.f;
  for (int j = tid; j < n_cols * n_rows; j += NT) {
    const float x = A[(j / n_rows) * lda + (j % n_rows)];
    f2 = fmaf(x, x, f2);
  }
  f2 = group_sum<32>(f2);
  if ((tid & 31) == 0) s_red[tid >> 5] = f2;
  for (int j = tid; j < n_cols * n_cols; j += NT) {
    const int col = j / n_cols, row = j % n_cols;
    Z[col * ldz + row] = (row == col) ? 1.f : 0.f;
  }
  __syncthreads();
  float frob2 = 0.f;
  for (int w = 0; w < NT / 32; ++w) frob2 += s_red[w];
  const float tiny = tiny_rel * frob2;
  __syncthreads();

  for (int sweep = 0; sweep < max_sweeps; ++sweep) {
    int rotated = 0;
    for (int round = 0; round < n_cols - 1; ++round) {
      // every lane runs the same number of iterations so that the full-warp
      // shuffles below always see all 32 lanes; lanes without a pair add zeros
      for (int base = 0; base < npairs; base += groups) {
        const int pr = base + grp;
        const bool active = pr < npairs;
        int p = 0, q = 0;
        if (pr == 0) {
          p = n_cols - 1;
          q = round;
        } else if (active) {
          p = (round + pr) % (n_cols - 1);
          q = (round - pr + (n_cols - 1)) % (n_cols - 1);
        }
        float* x = A + p * lda;
        float* y = A + q * lda;
        float xx = 0.f, yy = 0.f, xy = 0.f;
        if (active) {
          for (int e = gl; e < n_rows; e += G) {
            const float xe = x[e], ye = y[e];
            xx = fmaf(xe, xe, xx);
            yy = fmaf(ye, ye, yy);
            xy = fmaf(xe, ye, xy);
          }
        }
        if (G > 1) {
          xx = group_sum_rt(xx, G);
          yy = group_sum_rt(yy, G);
          xy = group_sum_rt(xy, G);
        }
        if (active && xx > tiny && yy > tiny && fabsf(xy) > tol * sqrtf(xx) * sqrtf(yy)) {
          rotated = 1;
          const float zeta = (yy - xx) / (2.f * xy);
          float t;
          if (fabsf(zeta) > 1e18f) {
            t = 0.5f / zeta;
          } else {
            t = copysignf(1.f, zeta) / (fabsf(zeta) + sqrtf(fmaf(zeta, zeta, 1.f)));
          }
          const float cs = rsqrtf(fmaf(t, t, 1.f));
          const float sn = cs * t;
          for (int e = gl; e < n_rows; e += G) {
            const float xe = x[e], ye = y[e];
            x[e] = cs * xe - sn * ye;
            y[e] = fmaf(sn, xe, cs * ye);
          }
          float* zx = Z + p * ldz;
          float* zy = Z + q * ldz;
          for (int e = gl; e < n_cols; e += G) {
            const float xe = zx[e], ye = zy[e];
            zx[e] = cs * xe - sn * ye;
            zy[e] = fmaf(sn, xe, cs * ye);
          }
        }
      }
      __syncthreads();
    }
    if (!__syncthreads_or(rotated)) return sweep + 1;
  }
  return max_sweeps + 1;
}

}  // namespace seed
