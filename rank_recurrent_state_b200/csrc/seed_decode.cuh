// seed_decode.cuh -- what the decode-step kernels share: launch parameters, the
// per-unit shared-memory stage that TMA bulk copies fill, and a warp reduction.
#pragma once

#include "seed_common.cuh"

namespace seed {

struct DecodeParams {
  const float* q;
  const float* k;
  const float* v;
  const float* alpha;
  const float* beta;
  float* o;
  float* a;
  void* U;   // element type: the kernel's factor type
  void* V;
  float* scale;
  int32_t* ncols;
  const float* vbar;
  uint32_t* status;
  int B, L, H, layer, R, W, slen;
  int overlap;   // host side only: launch with programmatic stream serialization
};

// One pipeline stage: everything a unit's step reads (U and V in their stored type).
template <int FORM, int DK, int DV, int MAXC, typename TS>
struct DecodeStage {
  static constexpr bool KDA = FORM == SEED_KDA;
  static constexpr int GPAD = (MAXC + 3) & ~3;
  alignas(16) TS U[MAXC * DK];
  alignas(16) TS V[MAXC * DV];
  float a[DK];
  float k[DK];
  float q[DK];
  float v[DV];
  float vb[DV];
  float al[KDA ? DK : 4];
  float P[KDA ? DK : 4];
  float gam[GPAD];
  float g;
  float beta;
  int c;
  int pad;
};

// Sum of NV per-lane values over the 32 lanes of a warp by recursive halving:
// 2 NV - 2 shuffles for NV <= 32 instead of 5 NV.  Lane l ends up holding the
// total of value (l >> (5 - log2 NV)) & (NV - 1).
template <int NV>
SEED_DEV float warp_xreduce(float (&v)[NV]) {
  const int lane = threadIdx.x & 31;
  int n = NV;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    if (n > 1) {
      const bool hi = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < NV / 2; ++i) {
        if (i < n / 2) {
          const float send = hi ? v[i] : v[i + n / 2];
          const float keep = hi ? v[i + n / 2] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      n >>= 1;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
    }
  }
  return v[0];
}

template <int NV>
SEED_DEV constexpr int log2c() { return NV <= 1 ? 0 : 1 + log2c<NV / 2>(); }

// The one-warp-per-unit decode kernel with a ring of column chunks
// (seed_decode_ring.cu), for R + W - 1 <= 64: the decode step's kernel there.
int launch_decode_ring(const DecodeParams& p, int form, int dk, int dv, int factors, cudaStream_t st);
// The whole-unit one-warp kernel for 16-bit factors (seed_decode_warp.cu).
int launch_decode_warp16(const DecodeParams& p, int form, int dk, int dv, int factors, cudaStream_t st);

}  // namespace seed
