// seed_compress.cu -- periodic compression, end-of-prefill conversion, to_dense.
//
// Compression ("Shallow Encoding Emits Deep Memories", SEED figures & tables
// (thelatestinai.com), Figure 1(b): every W steps the factors are compressed back
// to rank R; SEED summary (picx.dev), Corollary 4 bounds its open-loop error).
// One CTA per unit that holds m = R + W columns:
//   1. one TMA bulk copy per factor panel (U: m x d_k, V: m x d_v) into shared
//      memory; the lazy decay scales are folded in (true U);
//   2. Householder QR of both panels: U = Q_u R_u, V = Q_v R_v (R_* m x m upper);
//   3. the core M = R_u R_v^T (m x m) and its one-sided Jacobi SVD, M Z = X Sigma;
//   4. the R largest singular triplets: U' = Q_u X_R Sigma_R^{1/2},
//      V' = Q_v Z_R Sigma_R^{1/2}, applied as reflector products to the small
//      m-vectors, written to slots 0..R-1; scales reset; ncols <- R.
// U' V'^T is the best rank-R approximation of U V^T (Eckart-Young); the sink a is
// never touched.
//
// Conversion (SEED figures & tables, Figure 1(a), Table 1; SEED summary, Lemma 1):
// a = S vbar / ||vbar||^2, C = S - a vbar^T, one-sided Jacobi SVD of C^T (its
// columns are the rows of C), U = X_R Sigma^{1/2}, V = Y_R Sigma^{1/2}.
#include "seed_common.cuh"
#include "seed_launch.h"
#include "seed_tma.cuh"

namespace seed {

// ------------------------------------------------------------------ Householder QR
// In-place QR of an n x m panel A (column-major, lda = n, m <= n) by m Householder
// reflections H_j = I - tau_j v_j v_j^T, v_j = [0..0, 1, A[j+1:n, j]] stored below
// the diagonal, R on and above it (LAPACK's convention, Golub & Van Loan 5.2).
template <int NT>
__device__ void householder_qr(float* A, int n, int m, float* tau, float* s_red) {
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float prev_scale = 0.f;
  for (int j = 0; j < m; ++j) {
    float* x = A + j * n;
    // scale the previous reflector in place while summing this column's tail
    if (j > 0) {
      float* xp = A + (j - 1) * n;
      for (int i = j + tid; i < n; i += NT) xp[i] *= prev_scale;
    }
    float part = 0.f;
    for (int i = j + 1 + tid; i < n; i += NT) part = fmaf(x[i], x[i], part);
    part = group_sum<32>(part);
    if (lane == 0) s_red[warp] = part;
    __syncthreads();
    float sig2 = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) sig2 += s_red[w];
    const float x0 = x[j];
    float t = 0.f, beta = x0, vscale = 0.f;
    if (sig2 > 0.f) {
      const float nrm = sqrtf(fmaf(x0, x0, sig2));
      beta = -copysignf(nrm, x0);
      t = (beta - x0) / beta;
      vscale = 1.f / (x0 - beta);
    }
    // apply H_j to the trailing columns: warp per column, lanes over rows
    for (int k = j + 1 + warp; k < m; k += NW) {
      float* y = A + k * n;
      float w = 0.f;
      for (int i = j + 1 + lane; i < n; i += 32) w = fmaf(x[i], y[i], w);
      w = group_sum<32>(w);
      w = t * fmaf(w, vscale, y[j]);   // tau * v^T y with v = [1, x * vscale]
      if (lane == 0) y[j] -= w;
      const float wv = w * vscale;
      for (int i = j + 1 + lane; i < n; i += 32) y[i] = fmaf(-wv, x[i], y[i]);
    }
    __syncthreads();
    if (tid == 0) {
      x[j] = beta;
      tau[j] = t;
    }
    prev_scale = vscale;
  }
  for (int i = m + threadIdx.x; i < n; i += NT) A[(m - 1) * n + i] *= prev_scale;
  __syncthreads();
}

// y <- Q y for Q = H_0 ... H_{m-1} from householder_qr, one warp per vector of
// length n (n <= 32 * PER), y distributed as y[lane + 32 r].
template <int PER>
SEED_DEV void apply_q_warp(const float* A, int n, int m, const float* tau, float (&y)[PER]) {
  const int lane = threadIdx.x & 31;
  for (int j = m - 1; j >= 0; --j) {
    const float t = tau[j];
    if (t == 0.f) continue;
    const float* v = A + j * n;
    float w = 0.f;
#pragma unroll
    for (int r = 0; r < PER; ++r) {
      const int e = lane + 32 * r;
      if (e > j && e < n) w = fmaf(v[e], y[r], w);
      if (e == j) w += y[r];
    }
    w = group_sum<32>(w) * t;
#pragma unroll
    for (int r = 0; r < PER; ++r) {
      const int e = lane + 32 * r;
      if (e > j && e < n) y[r] = fmaf(-w, v[e], y[r]);
      if (e == j) y[r] -= w;
    }
  }
}

// ------------------------------------------------------------------ compress
struct CompressParams {
  void* U;   // element type: the kernel's factor type
  void* V;
  float* scale;
  int32_t* ncols;
  float* sigma_out;
  uint32_t* status;
  int B, L, H, layer, R, W, slen;  // layer < 0: all layers
};

template <int NT>
SEED_DEV int select_top(const float* sig, int n, int R, int* sel) {
  // rank of each value in descending order (ties broken by index); writes sel[rank] = j
  for (int j = threadIdx.x; j < n; j += NT) {
    const float s = sig[j];
    int rank = 0;
    for (int k = 0; k < n; ++k) {
      const float t = sig[k];
      rank += (t > s) || (t == s && k < j);
    }
    if (rank < R) sel[rank] = j;
  }
  return 0;
}

// One unit whose column count is R + W (checked by the caller), whole CTA.
// `phase` is the parity of this unit's use of the CTA's mbarrier.
template <int FORM, int DK, int DV, int NT, typename TS>
__device__ void compress_unit(const CompressParams& p, long long unit, long long srow,
                              unsigned char* smem_raw, uint64_t& bar, uint32_t phase) {
  constexpr int NW = NT / 32;
  constexpr bool KDA = FORM == SEED_KDA;
  const int m = p.R + p.W;
  const int mp = m + (m & 1);          // Jacobi needs an even column count
  const int ldm = m + 1;
  float* sU = reinterpret_cast<float*>(smem_raw);          // m x DK
  float* sV = sU + m * DK;                                   // m x DV
  float* sM = sV + m * DV;                                   // mp columns x ldm
  float* sZ = sM + mp * ldm;                                 // mp columns x mp (ld mp+1)
  const int ldz = mp + 1;
  float* tau_u = sZ + mp * ldz;
  float* tau_v = tau_u + m;
  float* sig = tau_v + m;                                    // mp
  float* s_red = sig + mp;                                   // NW
  float* s_scale = s_red + NW;                               // KDA ? DK : m
  float* cs_u = s_scale + (KDA ? DK : ((m + 3) & ~3));      // m: column scales of U
  float* cs_v = cs_u + m;                                    // m: column scales of V
  int* sel = reinterpret_cast<int*>(cs_v + m);               // R
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // 1. panels -> shared memory as float32 (TMA bulk copies, no multicast; 16-bit
  //    factors are read and widened by the threads)
  constexpr bool F32 = std::is_same<TS, float>::value;
  if constexpr (F32) {
    if (tid == 0) {
      mbar_arrive_expect_tx(&bar, (uint32_t)(m * (DK + DV) * sizeof(float)));
      bulk_g2s(sU, static_cast<const float*>(p.U) + unit * (long long)m * DK, (uint32_t)(m * DK * sizeof(float)),
               &bar);
      bulk_g2s(sV, static_cast<const float*>(p.V) + unit * (long long)m * DV, (uint32_t)(m * DV * sizeof(float)),
               &bar);
    }
  } else {
    const TS* Us = static_cast<const TS*>(p.U) + unit * (long long)m * DK;
    const TS* Vs = static_cast<const TS*>(p.V) + unit * (long long)m * DV;
    for (int idx = tid; idx < m * DK; idx += NT) sU[idx] = fac_to_f(Us[idx]);
    for (int idx = tid; idx < m * DV; idx += NT) sV[idx] = fac_to_f(Vs[idx]);
  }
  const int slen = p.slen;
  for (int i = tid; i < slen; i += NT) s_scale[i] = p.scale[unit * slen + i];
  __syncthreads();
  // every thread polls, and the outcome is made uniform so no barrier below diverges
  if constexpr (F32) {
    if (!__syncthreads_and(mbar_wait_bounded(&bar, phase, kWaitLimitNs))) {
      if (tid == 0) raise_flag(p.status, SEED_FLAG_TIMEOUT);
      mbar_wait_bounded(&bar, phase, kWaitLimitNs);
      __syncthreads();
      return;
    }
  }
  // KDA's per-row decay is folded into the panel (P >= 0.85^W stays far from
  // underflow); the per-column decay of GDN / Mamba-2 stays a column factor
  if constexpr (KDA) {
    for (int idx = tid; idx < m * DK; idx += NT) {
      const int i = idx % DK;
      sU[idx] *= s_scale[i];
    }
    __syncthreads();
  }
  // column equilibration by the largest magnitude: the QR then never squares
  // values near the float32 underflow (a long-decayed column may hold 1e-30), where
  // reflectors built from denormals lose their orthogonality
  for (int j = warp; j < 2 * m; j += NW) {
    const bool isU = j < m;
    const int col = isU ? j : j - m;
    float* x = isU ? sU + col * DK : sV + col * DV;
    const int n = isU ? DK : DV;
    float mx = 0.f;
    for (int i = lane; i < n; i += 32) mx = fmaxf(mx, fabsf(x[i]));
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float inv = mx > 0.f ? 1.f / mx : 0.f;
    for (int i = lane; i < n; i += 32) x[i] *= inv;
    if (lane == 0) {
      if (isU) cs_u[col] = mx * (KDA ? 1.f : s_scale[col]);
      else cs_v[col] = mx;
    }
  }
  __syncthreads();

  // 2. QR of both equilibrated panels
  householder_qr<NT>(sU, DK, m, tau_u, s_red);
  householder_qr<NT>(sV, DV, m, tau_v, s_red);

  // 3. core M = R_u R_v^T = Rhat_u diag(cs_u cs_v) Rhat_v^T, column-major with ld
  //    m+1 (plus a zero column if m is odd)
  for (int idx = tid; idx < mp * m; idx += NT) {
    const int j = idx / m, i = idx - j * m;   // M[i][j]
    float acc = 0.f;
    if (j < m) {
      for (int k = max(i, j); k < m; ++k)
        acc = fmaf(sU[k * DK + i] * (cs_u[k] * cs_v[k]), sV[k * DV + j], acc);
    }
    sM[j * ldm + i] = acc;
  }
  __syncthreads();
  const float tol = 8.f * sqrtf((float)m) * 5.9604645e-8f;
  const int sweeps = jacobi_svd<NT>(sM, ldm, m, sZ, ldz, mp, tol, 40, s_red, 1e-10f);
  const bool conv = sweeps <= 40;
  if (tid == 0) {
    atomicAdd(p.status + 1, (uint32_t)sweeps);
    atomicAdd(p.status + 2, 1u);
  }
  for (int j = tid; j < mp; j += NT) {
    float s2 = 0.f;
    for (int i = 0; i < m; ++i) s2 = fmaf(sM[j * ldm + i], sM[j * ldm + i], s2);
    sig[j] = sqrtf(s2);
  }
  __syncthreads();
  select_top<NT>(sig, mp, p.R, sel);
  __syncthreads();
  float smax = 0.f;
  for (int j = 0; j < mp; ++j) smax = fmaxf(smax, sig[j]);
  const float szero = (float)max(DK, DV) * 1.1920929e-7f * smax;

  // 4. U' = Q_u (M Z)_R Sigma^{-1/2}, V' = Q_v Z_R Sigma^{1/2}: warp per output column
  TS* Ug = static_cast<TS*>(p.U) + unit * (long long)m * DK;
  TS* Vg = static_cast<TS*>(p.V) + unit * (long long)m * DV;
  bool bad = !conv;
  for (int task = warp; task < 2 * p.R; task += NW) {
    const bool isU = task < p.R;
    const int r = isU ? task : task - p.R;
    const int j = sel[r];
    const float s = sig[j];
    const bool zero = !(s > szero);
    const float f = zero ? 0.f : (isU ? rsqrtf(s) : sqrtf(s));
    if (isU) {
      constexpr int PER = (DK + 31) / 32;
      float y[PER];
#pragma unroll
      for (int q = 0; q < PER; ++q) {
        const int e = lane + 32 * q;
        y[q] = e < m ? f * sM[j * ldm + e] : 0.f;
      }
      apply_q_warp<PER>(sU, DK, m, tau_u, y);
#pragma unroll
      for (int q = 0; q < PER; ++q) {
        const int e = lane + 32 * q;
        if (e < DK) {
          bad |= !isfinite(fac_round<TS>(y[q]));
          Ug[(long long)r * DK + e] = fac_from_f<TS>(y[q]);
        }
      }
    } else {
      constexpr int PER = (DV + 31) / 32;
      float y[PER];
#pragma unroll
      for (int q = 0; q < PER; ++q) {
        const int e = lane + 32 * q;
        y[q] = e < m ? f * sZ[j * ldz + e] : 0.f;
      }
      apply_q_warp<PER>(sV, DV, m, tau_v, y);
#pragma unroll
      for (int q = 0; q < PER; ++q) {
        const int e = lane + 32 * q;
        if (e < DV) {
          bad |= !isfinite(fac_round<TS>(y[q]));
          Vg[(long long)r * DV + e] = fac_from_f<TS>(y[q]);
        }
      }
    }
  }
  if (p.sigma_out) {
    for (int r = tid; r < p.R; r += NT) p.sigma_out[srow * p.R + r] = sig[sel[r]];
  }
  for (int i = tid; i < slen; i += NT) p.scale[unit * slen + i] = 1.f;
  if (tid == 0) p.ncols[unit] = p.R;
  if (!conv && tid == 0) raise_flag(p.status, SEED_FLAG_NOCONVERGE);
  if (bad && conv) raise_flag(p.status, SEED_FLAG_NONFINITE);
  __syncthreads();
}

// Scans the scope in chunks of NT units, collects those holding R + W columns and
// compresses them one after the other with the whole CTA.  A modest grid suffices:
// after the fast kernel this pass normally finds nothing left to do.
template <int FORM, int DK, int DV, int NT, typename TS>
__global__ void __launch_bounds__(NT) compress_kernel(const CompressParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_list[NT];
  __shared__ int s_cnt;
  const int tid = threadIdx.x;
  const int m = p.R + p.W;
  const int per = p.layer < 0 ? p.L * p.H : p.H;
  const long long total = (long long)p.B * per;
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  uint32_t phase = 0;
  for (long long base = (long long)blockIdx.x * NT; base < total; base += (long long)gridDim.x * NT) {
    if (tid == 0) s_cnt = 0;
    __syncthreads();
    const long long idx = base + tid;
    if (idx < total) {
      const long long b = idx / per, rest = idx - b * per;
      const long long unit = p.layer < 0 ? idx : (b * p.L + p.layer) * p.H + rest;
      const int c = p.ncols[unit];
      if (c == m) s_list[atomicAdd(&s_cnt, 1)] = (int)(idx - base);
      else if (c < 0 || c > m) raise_flag(p.status, SEED_FLAG_BADCOLS);
    }
    __syncthreads();
    const int n = s_cnt;
    for (int k = 0; k < n; ++k) {
      const long long i2 = base + s_list[k];
      const long long b = i2 / per, rest = i2 - b * per;
      const long long unit = p.layer < 0 ? i2 : (b * p.L + p.layer) * p.H + rest;
      compress_unit<FORM, DK, DV, NT, TS>(p, unit, i2, smem_raw, bar, phase);
      phase ^= 1u;
    }
    __syncthreads();
  }
}

static size_t compress_smem_bytes(int form, int dk, int dv, int R, int W, int nt) {
  const int m = R + W, mp = m + (m & 1);
  size_t f = (size_t)m * dk + (size_t)m * dv + (size_t)mp * (m + 1) + (size_t)mp * (mp + 1) +
             2 * m + mp + nt / 32 + (form == SEED_KDA ? dk : ((m + 3) & ~3)) + 2 * m + R;
  return f * sizeof(float) + 16;
}

template <int FORM, int DK, int DV, typename TS>
static int launch_compress_tt(const CompressParams& p, int blocks, cudaStream_t st) {
  constexpr int NT = 128;
  const size_t smem = compress_smem_bytes(FORM, DK, DV, p.R, p.W, NT);
  auto kern = compress_kernel<FORM, DK, DV, NT, TS>;
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return SEED_ERR_CUDA;
  }
  const int grid = (blocks + NT - 1) / NT < 1184 ? (blocks + NT - 1) / NT : 1184;
  kern<<<grid, NT, smem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
}

template <int FORM, int DK, int DV>
static int launch_compress_t(const CompressParams& p, int blocks, int factors, cudaStream_t st) {
  switch (factors) {
    case SEED_FACTORS_F32: return launch_compress_tt<FORM, DK, DV, float>(p, blocks, st);
    case SEED_FACTORS_F16: return launch_compress_tt<FORM, DK, DV, __half>(p, blocks, st);
    case SEED_FACTORS_BF16: return launch_compress_tt<FORM, DK, DV, __nv_bfloat16>(p, blocks, st);
  }
  return SEED_ERR_INVALID_ARG;
}

#define SEED_DISPATCH_DIMS(FN, FORM, ...)                                     \
  do {                                                                        \
    if (d.d_k == 16 && d.d_v == 16) return FN<FORM, 16, 16>(__VA_ARGS__);     \
    if (d.d_k == 32 && d.d_v == 32) return FN<FORM, 32, 32>(__VA_ARGS__);     \
    if (d.d_k == 64 && d.d_v == 64) return FN<FORM, 64, 64>(__VA_ARGS__);     \
    if (d.d_k == 128 && d.d_v == 128) return FN<FORM, 128, 128>(__VA_ARGS__); \
    if (d.d_k == 128 && d.d_v == 64) return FN<FORM, 128, 64>(__VA_ARGS__);   \
    if (d.d_k == 64 && d.d_v == 128) return FN<FORM, 64, 128>(__VA_ARGS__);   \
    return SEED_ERR_SHAPE;                                                    \
  } while (0)

int launch_compress(const seed_dims& d, const seed_state& s, int layer, float* sigma_out,
                    uint32_t* status, cudaStream_t st) {
  if (compress_fast_supported(d)) {
    const int rc = launch_compress_fast(d, s, layer, sigma_out, status, st);
    if (rc != SEED_OK) return rc;
  } else if (compress_wide_supported(d)) {
    const int rc = launch_compress_wide(d, s, layer, sigma_out, status, st);
    if (rc != SEED_OK) return rc;
  }
  return launch_compress_householder(d, s, layer, sigma_out, status, st);
}

int launch_compress_householder(const seed_dims& d, const seed_state& s, int layer, float* sigma_out,
                                uint32_t* status, cudaStream_t st) {
  CompressParams p{s.U, s.V, s.scale, s.ncols, sigma_out, status,
                   d.batch, d.layers, d.heads, layer, d.R, d.W, scale_len(d)};
  const int blocks = d.batch * d.heads * (layer < 0 ? d.layers : 1);
  switch (d.form) {
    case SEED_GDN: SEED_DISPATCH_DIMS(launch_compress_t, SEED_GDN, p, blocks, d.factors, st);
    case SEED_KDA: SEED_DISPATCH_DIMS(launch_compress_t, SEED_KDA, p, blocks, d.factors, st);
    case SEED_MAMBA2: SEED_DISPATCH_DIMS(launch_compress_t, SEED_MAMBA2, p, blocks, d.factors, st);
  }
  return SEED_ERR_INVALID_ARG;
}

// ------------------------------------------------------------------ conversion
struct InitParams {
  const float* S;
  float* a;
  void* U;   // element type: the kernel's factor type
  void* V;
  float* scale;
  int32_t* ncols;
  const float* vbar;
  float* sigma_out;
  uint32_t* status;
  int B, L, H, layer, R, W, form, slen, factors;
};

// The one-sided Jacobi runs over the shorter side of C so that the columns it
// orthogonalises are at most as many as their length: over the d_v columns of C
// when d_k >= d_v, else over the d_k columns of C^T.  Either way at most one
// column is a structural null direction (C vbar = 0), not many.
template <int DK, int DV, int NT, typename TS>
__global__ void __launch_bounds__(NT) init_kernel(const InitParams p) {
  constexpr int NW = NT / 32;
  constexpr bool COLS = DK >= DV;       // Jacobi over the columns of C
  constexpr int NC = COLS ? DV : DK;    // Jacobi columns
  constexpr int NR = COLS ? DK : DV;    // their length
  constexpr int LDC = NR + 1;
  constexpr int LDZ = NC + 1;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  float* sC = reinterpret_cast<float*>(smem_raw);   // NC columns of length NR
  float* sZ = sC + NC * LDC;                         // NC x NC
  float* s_vb = sZ + NC * LDZ;                       // DV
  float* s_a = s_vb + DV;                            // DK
  float* sig = s_a + DK;                             // NC
  float* s_red = sig + NC;                           // NW
  int* sel = reinterpret_cast<int*>(s_red + NW);     // R
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int units_in_scope = p.layer < 0 ? p.L * p.H : p.H;
  const int b = blockIdx.x / units_in_scope;
  const int rest = blockIdx.x - b * units_in_scope;
  const int l = p.layer < 0 ? rest / p.H : p.layer;
  const int h = p.layer < 0 ? rest - (rest / p.H) * p.H : rest;
  const long long unit = ((long long)b * p.L + l) * p.H + h;
  const int m = p.R + p.W;
  const float* S = p.S + (long long)blockIdx.x * DK * DV;

  for (int i = tid; i < DV; i += NT) s_vb[i] = p.vbar[((long long)l * p.H + h) * DV + i];
  for (int idx = tid; idx < DK * DV / 4; idx += NT) {
    const float4 x = ld4(S + 4 * idx);
    const int i = (4 * idx) / DV, j = (4 * idx) - i * DV;   // S[i][j .. j+3]
    const float xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (COLS) sC[(j + e) * LDC + i] = xv[e];
      else sC[i * LDC + j + e] = xv[e];
    }
  }
  __syncthreads();
  float vv = 0.f;
  for (int j = tid; j < DV; j += NT) vv = fmaf(s_vb[j], s_vb[j], vv);
  vv = group_sum<32>(vv);
  if (lane == 0) s_red[warp] = vv;
  __syncthreads();
  float vbvb = 0.f;
#pragma unroll
  for (int w = 0; w < NW; ++w) vbvb += s_red[w];
  if (!(vbvb > 0.f)) {
    if (tid == 0) raise_flag(p.status, SEED_FLAG_ZERO_VBAR);
    return;
  }
  // a = S vbar / ||vbar||^2, then C = S - a vbar^T in place
  if (COLS) {
    for (int i = tid; i < DK; i += NT) {
      float acc = 0.f;
      for (int j = 0; j < DV; ++j) acc = fmaf(sC[j * LDC + i], s_vb[j], acc);
      acc /= vbvb;
      for (int j = 0; j < DV; ++j) sC[j * LDC + i] = fmaf(-acc, s_vb[j], sC[j * LDC + i]);
      s_a[i] = acc;
    }
  } else {
    for (int i = warp; i < DK; i += NW) {
      float acc = 0.f;
      for (int j = lane; j < DV; j += 32) acc = fmaf(sC[i * LDC + j], s_vb[j], acc);
      acc = group_sum<32>(acc) / vbvb;
      for (int j = lane; j < DV; j += 32) sC[i * LDC + j] = fmaf(-acc, s_vb[j], sC[i * LDC + j]);
      if (lane == 0) s_a[i] = acc;
    }
  }
  __syncthreads();
  const float tol = 8.f * sqrtf((float)NR) * 5.9604645e-8f;
  const int sweeps = jacobi_svd<NT>(sC, LDC, NR, sZ, LDZ, NC, tol, 60, s_red, 1e-12f);
  const bool conv = sweeps <= 60;
  if (tid == 0) {
    atomicAdd(p.status + 3, (uint32_t)sweeps);
    atomicAdd(p.status + 4, 1u);
  }
  for (int j = tid; j < NC; j += NT) {
    float s2 = 0.f;
    for (int i = 0; i < NR; ++i) s2 = fmaf(sC[j * LDC + i], sC[j * LDC + i], s2);
    sig[j] = sqrtf(s2);
  }
  __syncthreads();
  select_top<NT>(sig, NC, p.R, sel);
  __syncthreads();
  float smax = 0.f;
  for (int j = 0; j < NC; ++j) smax = fmaxf(smax, sig[j]);
  const float szero = (float)max(DK, DV) * 1.1920929e-7f * smax;

  // COLS: U[:, r] = (C Z)[:, j] / sqrt(s), V[:, r] = Z[:, j] sqrt(s)
  // else: U[:, r] = Z[:, j] sqrt(s),       V[:, r] = (C^T Z)[:, j] / sqrt(s)
  TS* Ug = static_cast<TS*>(p.U) + unit * (long long)m * DK;
  TS* Vg = static_cast<TS*>(p.V) + unit * (long long)m * DV;
  bool bad = !conv;
  for (int r = warp; r < p.R; r += NW) {
    const bool valid = r < NC;
    const int j = valid ? sel[r] : 0;
    const float s = valid ? sig[j] : 0.f;
    const bool zero = !(s > szero);
    const float fz = zero ? 0.f : sqrtf(s), fc = zero ? 0.f : rsqrtf(s);
    for (int e = lane; e < DK; e += 32) {
      const float x = COLS ? fc * sC[j * LDC + e] : fz * sZ[j * LDZ + e];
      bad |= !isfinite(fac_round<TS>(x));
      Ug[(long long)r * DK + e] = fac_from_f<TS>(x);
    }
    for (int e = lane; e < DV; e += 32) {
      const float x = COLS ? fz * sZ[j * LDZ + e] : fc * sC[j * LDC + e];
      bad |= !isfinite(fac_round<TS>(x));
      Vg[(long long)r * DV + e] = fac_from_f<TS>(x);
    }
    if (p.sigma_out && lane == 0) p.sigma_out[(long long)blockIdx.x * p.R + r] = s;
  }
  for (int i = tid; i < DK; i += NT) {
    bad |= !isfinite(s_a[i]);
    p.a[unit * DK + i] = s_a[i];
  }
  for (int i = tid; i < p.slen; i += NT) p.scale[unit * p.slen + i] = 1.f;
  if (tid == 0) p.ncols[unit] = p.R;
  if (!conv && tid == 0) raise_flag(p.status, SEED_FLAG_NOCONVERGE);
  if (bad && conv) raise_flag(p.status, SEED_FLAG_NONFINITE);
}

template <int DK, int DV, typename TS>
static int launch_init_tt(const InitParams& p, int blocks, cudaStream_t st) {
  constexpr int NT = 256;
  constexpr int NC = DK >= DV ? DV : DK, NR = DK >= DV ? DK : DV;
  const size_t smem = ((size_t)NC * (NR + 1) + (size_t)NC * (NC + 1) + DV + DK + NC + NT / 32 +
                       p.R) * sizeof(float) + 16;
  auto kern = init_kernel<DK, DV, NT, TS>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return SEED_ERR_CUDA;
  kern<<<blocks, NT, smem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
}

template <int FORM, int DK, int DV>
static int launch_init_t(const InitParams& p, int blocks, cudaStream_t st) {
  switch (p.factors) {
    case SEED_FACTORS_F32: return launch_init_tt<DK, DV, float>(p, blocks, st);
    case SEED_FACTORS_F16: return launch_init_tt<DK, DV, __half>(p, blocks, st);
    case SEED_FACTORS_BF16: return launch_init_tt<DK, DV, __nv_bfloat16>(p, blocks, st);
  }
  return SEED_ERR_INVALID_ARG;
}

int launch_init_from_dense(const seed_dims& d, const seed_state& s, int layer, const float* S,
                           float* sigma_out, uint32_t* status, cudaStream_t st) {
  InitParams p{S, s.a, s.U, s.V, s.scale, s.ncols, s.vbar, sigma_out, status,
               d.batch, d.layers, d.heads, layer, d.R, d.W, d.form, scale_len(d), d.factors};
  const int blocks = d.batch * d.heads * (layer < 0 ? d.layers : 1);
  SEED_DISPATCH_DIMS(launch_init_t, 0, p, blocks, st);
}

// ------------------------------------------------------------------ to_dense
struct ToDenseParams {
  const float* a;
  const void* U;   // element type: the kernel's factor type
  const void* V;
  const float* scale;
  const int32_t* ncols;
  const float* vbar;
  const int32_t* units;
  float* S;
  uint32_t* status;
  int B, L, H, layer, R, W, form, slen, factors;
};

template <int DK, int DV, int NT, typename TS>
__global__ void __launch_bounds__(NT) to_dense_kernel(const ToDenseParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const int m = p.R + p.W;
  float* sU = reinterpret_cast<float*>(smem_raw);   // m x DK (true columns)
  float* sV = sU + m * DK;                           // m x DV
  float* s_a = sV + m * DV;
  float* s_vb = s_a + DK;
  const int per = p.layer < 0 ? p.L * p.H : p.H;
  const int scope = p.units ? p.units[blockIdx.x] : (int)blockIdx.x;
  if (scope < 0 || scope >= p.B * per) {   // the unit list lives on the device: check it here
    if (threadIdx.x == 0) raise_flag(p.status, SEED_FLAG_BADINDEX);
    return;
  }
  const int b = scope / per, rest = scope - b * per;
  const int l = p.layer < 0 ? rest / p.H : p.layer;
  const int h = p.layer < 0 ? rest - (rest / p.H) * p.H : rest;
  const long long unit = ((long long)b * p.L + l) * p.H + h;
  const bool kda = p.form == SEED_KDA;
  int c = p.ncols[unit];
  if (c < 0 || c > m) {
    if (threadIdx.x == 0) raise_flag(p.status, SEED_FLAG_BADCOLS);
    c = 0;
  }
  for (int idx = threadIdx.x; idx < c * DK; idx += NT) {
    const int j = idx / DK, i = idx - j * DK;
    const float sc = kda ? p.scale[unit * DK + i] : p.scale[unit * p.slen + j];
    sU[idx] = sc * fac_to_f(static_cast<const TS*>(p.U)[unit * (long long)m * DK + idx]);
  }
  for (int idx = threadIdx.x; idx < c * DV; idx += NT)
    sV[idx] = fac_to_f(static_cast<const TS*>(p.V)[unit * (long long)m * DV + idx]);
  for (int i = threadIdx.x; i < DK; i += NT) s_a[i] = p.a[unit * DK + i];
  for (int i = threadIdx.x; i < DV; i += NT) s_vb[i] = p.vbar[((long long)l * p.H + h) * DV + i];
  __syncthreads();
  float* S = p.S + (long long)blockIdx.x * DK * DV;
  for (int idx = threadIdx.x; idx < DK * DV; idx += NT) {
    const int i = idx / DV, j = idx - i * DV;
    float acc = s_a[i] * s_vb[j];
    for (int r = 0; r < c; ++r) acc = fmaf(sU[r * DK + i], sV[r * DV + j], acc);
    S[idx] = acc;
  }
}

template <int DK, int DV, typename TS>
static int launch_to_dense_tt(const ToDenseParams& p, int blocks, cudaStream_t st) {
  constexpr int NT = 256;
  const size_t smem = ((size_t)(p.R + p.W) * (DK + DV) + DK + DV) * sizeof(float);
  auto kern = to_dense_kernel<DK, DV, NT, TS>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return SEED_ERR_CUDA;
  kern<<<blocks, NT, smem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? SEED_OK : SEED_ERR_CUDA;
}

template <int FORM, int DK, int DV>
static int launch_to_dense_t(const ToDenseParams& p, int blocks, cudaStream_t st) {
  switch (p.factors) {
    case SEED_FACTORS_F32: return launch_to_dense_tt<DK, DV, float>(p, blocks, st);
    case SEED_FACTORS_F16: return launch_to_dense_tt<DK, DV, __half>(p, blocks, st);
    case SEED_FACTORS_BF16: return launch_to_dense_tt<DK, DV, __nv_bfloat16>(p, blocks, st);
  }
  return SEED_ERR_INVALID_ARG;
}

int launch_to_dense(const seed_dims& d, const seed_state& s, int layer, const int32_t* units,
                    int n_units, float* S_out, uint32_t* status, cudaStream_t st) {
  ToDenseParams p{s.a, s.U, s.V, s.scale, s.ncols, s.vbar, units, S_out, status,
                  d.batch, d.layers, d.heads, layer, d.R, d.W, d.form, scale_len(d), d.factors};
  SEED_DISPATCH_DIMS(launch_to_dense_t, 0, p, n_units, st);
}

}  // namespace seed
