/*
 * seed_synth.h -- synthetic workload generation on the device (libseed.so).
 *
 * Not part of the method: these calls build seeded synthetic inputs and the dense
 * end-of-prefill states that the method starts from.  They stand in for a model's
 * q/k/v/alpha/beta projections and for the prefill, neither of which the pages
 * describe beyond the recurrences themselves.
 *
 * Generator: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers:
 * as easy as 1, 2, 3", SC'11), key = (seed, workload), counter = (block,
 * field | phase << 8, t, unit).  Transforms are evaluated in float64 and rounded
 * to float32 once; the value distributions per form are:
 *   GDN, KDA   k, q ~ N(0, I) L2-normalised; v = 3 vbar + 0.3 z; beta = sigmoid(z);
 *              GDN g = exp(-softplus(-3 + 0.5 z)); KDA alpha_i = 0.85 + 0.15 u_i
 *   Mamba-2    k, q ~ N(0, I) / sqrt(d_k); v = vbar + 0.5 z; Delta = softplus(-2 + 0.5 z);
 *              alpha = exp(-Delta A), A = 1 + 15 u per head
 *   vbar       random direction, norm 1 (vbar_unit) or 1 + 3 u
 * A host implementation of the same counters lives in the Python package
 * `workloads`; the two are written independently and tested against each other.
 *
 * Memory, alignment, streams and return codes as in seed.h.
 */
#ifndef SEED_SYNTH_H_
#define SEED_SYNTH_H_

#include <stdint.h>

#include "seed.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  uint32_t seed;      /* master seed, first key word */
  uint32_t workload;  /* workload id, second key word */
  int32_t vbar_unit;  /* 1: vbar has unit norm; 0: norm 1 + 3u */
  int32_t b0;         /* global index of the first request of this batch (sharding) */
} seed_synth_key;

#define SEED_PHASE_PREFILL 0
#define SEED_PHASE_DECODE 1
#define SEED_PHASE_LEADIN 2   /* decode steps a request took before the others joined it
                                 (ragged compression schedules); t counts them from 0 */

/* vbar [L][H][d_v] for every head. */
int seed_synth_vbar(const seed_dims* dims, seed_synth_key key, float* vbar, void* stream);

/* Inputs of decode step / prefill token t of `phase` for every unit of `layer`:
 * q, k [B][H][d_k]; v [B][H][d_v]; alpha [B][H] (KDA [B][H][d_k]); beta [B][H].
 * q may be NULL (not generated).  vbar is the table from seed_synth_vbar.        */
int seed_synth_token_inputs(const seed_dims* dims, seed_synth_key key, int32_t phase, int32_t t,
                            int32_t layer, const float* vbar, float* q, float* k, float* v,
                            float* alpha, float* beta, void* stream);

/* Dense prefill: from S_0 = 0, n_tokens tokens of the form's dense recurrence for
 * every unit of `layer` (or all layers), inputs generated in the kernel (phase 0).
 * S_out [B][H][d_k][d_v] for one layer, [B][L][H][d_k][d_v] for all.               */
int seed_synth_dense_prefill(const seed_dims* dims, seed_synth_key key, int32_t n_tokens,
                             int32_t layer, const float* vbar, float* S_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SEED_SYNTH_H_ */
