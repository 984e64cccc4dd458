/*
 * seed.h -- C ABI of the sink-plus-low-rank recurrent-state decode path (libseed.so).
 *
 * What the library computes ("Shallow Encoding Emits Deep Memories", SEED):
 * each per-head d_k x d_v recurrent state of a Gated DeltaNet, Kimi Delta
 * Attention or Mamba-2 layer is stored as
 *
 *     S = a vbar^T + U V^T                                              (1)
 *
 * (SEED summary (picx.dev), Methodology, "SEED Architecture": decode, shallow in
 * representation), where vbar (d_v) is a fixed per-head direction shared by all
 * requests, a (d_k) the sink coefficient and U (d_k x c), V (d_v x c) the content
 * factors.  A decode step reads out o = S^T q, applies the exact factored update
 * (same page, "Exact Update (Lemma 2)"; the sink split of Lemma 1 under
 * "Theoretical and Practical Implications"), and appends one column pair; every
 * W steps the factors are compressed back to rank R (SEED figures & tables
 * (thelatestinai.com), Figure 1(b) and Table 1).
 *
 * Conventions shared by every entry point
 *  - Memory: every pointer is a DEVICE pointer owned by the caller.  The library
 *    never allocates, frees or keeps a pointer after a call returns.
 *  - Alignment: every array pointer must be 16-byte aligned (float4 access).
 *  - Streams: `stream` is a cudaStream_t (NULL = the legacy default stream).
 *    Calls only enqueue work and return; they never synchronise, except
 *    seed_get_status.
 *  - Errors: arguments are validated on the host before anything is enqueued;
 *    a negative seed_status is returned and nothing is launched.  Conditions
 *    that only the device can see set bits in the status word that lives in the
 *    caller's workspace; kernels never trap.  Read them with seed_get_status.
 *  - Units: one unit is one (request b, layer l, head h).  State arrays are
 *    request-major: unit index u = ((b * layers) + l) * heads + h.
 *  - Precision: float32 arithmetic throughout; float32 storage, except that the
 *    content factors U and V may be stored in 16 bits (seed_dims.factors).
 */
#ifndef SEED_H_
#define SEED_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Recurrent-layer forms.  Dense recurrences (orientation d_k x d_v, o = S^T q):
 *   SEED_GDN     S+ = g (I - beta k k^T) S + beta k v^T
 *   SEED_KDA     S+ = (I - beta k k^T) Diag(alpha) S + beta k v^T
 *   SEED_MAMBA2  S+ = alpha S + Delta k v^T   (k = B_t, v = x_t; d_k = d_state, d_v = headdim,
 *                the orientation of SEED figures & tables, Table 17)                         */
typedef enum { SEED_GDN = 0, SEED_KDA = 1, SEED_MAMBA2 = 2 } seed_form;

/* Host-side return codes. */
typedef enum {
  SEED_OK = 0,
  SEED_ERR_INVALID_ARG = -1, /* null pointer, bad enum, non-positive size, layer out of range */
  SEED_ERR_SHAPE = -2,       /* unsupported d_k / d_v / R / W combination                    */
  SEED_ERR_ALIGN = -3,       /* a pointer is not 16-byte aligned                             */
  SEED_ERR_CUDA = -4,        /* a CUDA runtime call or kernel launch failed                  */
  SEED_ERR_WORKSPACE = -5    /* workspace missing or smaller than seed_workspace_bytes       */
} seed_status;

/* Device-side status bits, accumulated in the workspace, read by seed_get_status. */
#define SEED_FLAG_FULL 0x1u       /* decode_step met a unit already holding R+W columns;
                                     that unit was left unchanged and its o not written    */
#define SEED_FLAG_NONFINITE 0x2u  /* a non-finite value was produced                       */
#define SEED_FLAG_NOCONVERGE 0x4u /* a Jacobi SVD reached its sweep cap                     */
#define SEED_FLAG_BADCOLS 0x8u    /* a unit's column count was outside [0, R+W]            */
#define SEED_FLAG_ZERO_VBAR 0x10u /* a head's vbar has zero norm; its units were left
                                     unchanged (decode_step also leaves o unwritten)      */
#define SEED_FLAG_BADINDEX 0x20u  /* seed_state_to_dense met a unit index outside the scope;
                                     that output slab was not written                      */
#define SEED_FLAG_TIMEOUT 0x40u   /* a bounded wait for a bulk copy gave up (1 s); the unit
                                     being worked on was left unchanged, except that a
                                     compression that had already written part of its
                                     result sets the unit's column count to -1 (later
                                     calls flag it SEED_FLAG_BADCOLS and skip it)          */

/* Supported shapes: (d_k, d_v) equal and in {16, 32, 64, 128}, or (128, 64), or
 * (64, 128); R >= 1, W >= 1, R + W <= SEED_MAX_COLS and R + W <= min(d_k, d_v).
 * Anything else returns SEED_ERR_SHAPE. */
#define SEED_MAX_COLS 96
#define SEED_ALL_LAYERS (-1)

/* Storage format of the content factors U and V (seed_dims.factors).  The SEED
 * figures & tables page, Table 9 (and Table 4's 16-bit rows), keeps the shallow
 * state's factors in fp16 or bf16, rounded when a compression writes them, with the
 * same drift as fp32; the SEED summary's key points add that fp16 factors halve the
 * state's bytes again.  Here every value written to U or V -- a conversion's or a
 * compression's result and every appended column pair -- is rounded to the nearest
 * value of the format, ties to even; all arithmetic stays float32, and the sink a,
 * the scales and the column counts stay float32 / int32.  A 16-bit factor array
 * holds 2-byte elements in the layout below (pointers still 16-byte aligned).
 * A value beyond the format's range is stored as +-inf and raises
 * SEED_FLAG_NONFINITE (fp16's largest finite value is 65504).                      */
typedef enum { SEED_FACTORS_F32 = 0, SEED_FACTORS_F16 = 1, SEED_FACTORS_BF16 = 2 } seed_factors;

/* Problem dimensions: batch of requests x layers x heads, head dims, rank, window. */
typedef struct {
  int32_t form;   /* seed_form */
  int32_t batch;  /* requests B */
  int32_t layers; /* recurrent layers L */
  int32_t heads;  /* heads per layer H */
  int32_t d_k;    /* key / state dimension */
  int32_t d_v;    /* value dimension */
  int32_t R;      /* rank kept after a compression */
  int32_t W;      /* steps between compressions; a unit holds at most R + W columns */
  int32_t factors; /* seed_factors: element type of U and V (0 = float32)          */
} seed_dims;

/* The stored state of all B x L x H units (device pointers, caller-owned).
 *   a      [B][L][H][d_k]            sink coefficient a
 *   U      [B][L][H][R+W][d_k]       content factor U (element type: dims->factors), one
 *                                    contiguous d_k column per slot;
 *                                    slot j holds column j, so appends never move data
 *   V      [B][L][H][R+W][d_v]       content factor V, same slots
 *   scale  GDN, Mamba-2: [B][L][H][ceil4(R+W)] per-column scales gamma_j: the true
 *                                    U column j is gamma_j * U[:, j] (decay applied lazily,
 *                                    and a singular value kept by seed_compress);
 *                                    the per-unit stride is R+W rounded up to a multiple of 4
 *          KDA:          [B][L][H][d_k] per-channel decay products P: the true U is
 *                                    Diag(P) U (per-row decay applied lazily)
 *   ncols  [B][L][H] int32            columns held, R <= ncols <= R+W after a conversion
 *   vbar   [L][H][d_v]                per-head mean value, shared by all requests
 * The represented dense state of a unit is (1) with the true U; seed_state_to_dense
 * returns it.  seed_scale_len() gives the per-unit length of `scale`.               */
typedef struct {
  float* a;
  void* U;   /* float, or 16-bit elements (dims->factors) */
  void* V;
  float* scale;
  int32_t* ncols;
  const float* vbar;
} seed_state;

/* Per-unit length of seed_state.scale: R+W rounded up to a multiple of 4 for GDN and
 * Mamba-2, d_k for KDA.  Returns -1 for unsupported dims. */
int32_t seed_scale_len(const seed_dims* dims);

/* Bytes of device workspace every call below needs (the device status word).
 * Zero it once with seed_workspace_init before first use. */
size_t seed_workspace_bytes(const seed_dims* dims);
int seed_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* End-of-prefill conversion (SEED figures & tables, Figure 1(a) and Table 1: the
 * states the prefill leaves are compressed to the shallow form; SEED summary,
 * Lemma 1: the split along vbar).  For every unit of `layer` (or of all layers
 * with SEED_ALL_LAYERS):
 *     a = S vbar / ||vbar||^2,   C = S - a vbar^T,   U V^T = best rank-R approximation of C
 * with Sigma^{1/2} on each side (one-sided Jacobi SVD of C); scale <- 1; ncols <- R.
 * Columns of a rank-deficient C are zero.
 *   S_dense    [B][H][d_k][d_v] row-major for one layer, [B][L][H][d_k][d_v] for all
 *   sigma_out  optional (may be NULL): the kept singular values, [units in scope][R]
 * A unit whose vbar is zero is left unchanged and raises SEED_FLAG_ZERO_VBAR.          */
int seed_state_init_from_dense(const seed_dims* dims, const seed_state* state, int32_t layer,
                               const float* S_dense, float* sigma_out, void* ws, size_t ws_bytes,
                               void* stream);

/* One exact decode step of one layer for all B x H units, then the read-out
 * (SEED summary, "Exact Update (Lemma 2)" and Lemma 1; read-out o = S+^T q with
 * S+ the updated state).  For Gated DeltaNet, with omega = v^T vbar / ||vbar||^2 and
 * eps = v - omega vbar:
 *     a+ = g a + beta (omega - g k^T a) k
 *     U+ = [g U, k],   V+ = [V, beta (eps - g V U^T k)]
 *     o  = vbar (a+^T q) + V+ (U+^T q)
 * KDA applies Diag(alpha) on the key side before the erase; Mamba-2 has no erase
 * and writes with Delta (V+ = [V, Delta eps]).  The new column pair goes to slot
 * ncols, which then grows by one.  A unit already at R+W columns is skipped and
 * SEED_FLAG_FULL is raised: call seed_compress after the step that fills R+W.
 *   q, k   [B][H][d_k]           v, o [B][H][d_v]
 *   alpha  GDN: decay g [B][H];  KDA: per-channel decay [B][H][d_k];  Mamba-2: alpha [B][H]
 *   beta   GDN, KDA: write strength [B][H];  Mamba-2: Delta [B][H]                        */
int seed_decode_step(const seed_dims* dims, const seed_state* state, int32_t layer,
                     const float* q, const float* k, const float* v, const float* alpha,
                     const float* beta, float* o, void* ws, size_t ws_bytes, void* stream);

/* seed_decode_step, with the same arguments and results, for a stream on which the
 * launch just before this call does not write this layer's stored state (a, U, V,
 * scale, ncols), e.g. the decode step of another layer.  The step may then begin
 * streaming this layer's stored columns while that launch finishes (programmatic
 * dependent launch, R + W <= 65; larger shapes launch as seed_decode_step does).  It reads q, k, v, alpha, beta and the state's scalars,
 * and writes anything, only after that launch has completed, so the inputs may be
 * its outputs.  The caller owns the guarantee: if the launch before writes this
 * layer's state (a seed_compress or a conversion of this layer, for instance), call
 * seed_decode_step instead.                                                          */
int seed_decode_step_overlapped(const seed_dims* dims, const seed_state* state, int32_t layer,
                                const float* q, const float* k, const float* v, const float* alpha,
                                const float* beta, float* o, void* ws, size_t ws_bytes, void* stream);

/* Periodic compression (SEED figures & tables, Figure 1(b): every W steps the
 * factors are compressed back to rank R; SEED summary, Corollary 4 bounds its
 * open-loop error).  For every unit of `layer` (or all layers) whose ncols equals
 * R+W: QR of U and V (true U, scales applied), the (R+W) x (R+W) core
 * M = R_u R_v^T, a one-sided Jacobi SVD M = X Sigma Y^T, and the rank-R truncation
 * (Q_u X_R) Sigma_R (Q_v Y_R)^T written to slots 0..R-1; ncols <- R.  The sink a
 * is not touched.  Units with ncols != R+W are left unchanged.
 * How Sigma_R is stored depends on the path a unit takes (both represent the same
 * state): with d_k, d_v in {64, 128} and either R + W <= 32 and R <= 16, or
 * 32 < R + W <= 64 and R <= 32, a well-conditioned, well-scaled unit takes
 * Cholesky QR, which for GDN and Mamba-2 stores the unit
 * columns Q_u X_R, Q_v Y_R and scale_r = sigma_r (scale 1 beyond R), and for KDA
 * Sigma^{1/2} on each side with P <- 1; every other unit takes Householder QR,
 * which stores Sigma^{1/2} on each side and resets the scales to 1.
 *   sigma_out  optional: [units in scope][R] singular values kept (only compressed
 *              units' rows are written)                                              */
int seed_compress(const seed_dims* dims, const seed_state* state, int32_t layer,
                  float* sigma_out, void* ws, size_t ws_bytes, void* stream);

/* One decode step of one layer (as seed_decode_step) fused with the compression of
 * the units it brings to R + W columns (as seed_compress on that layer): call it
 * instead of seed_decode_step for the step after which a compression is due (every
 * step with ragged per-request schedules); no separate seed_compress is needed.
 * Where R + W <= 32, R <= 16 and d_k, d_v are in {64, 128}, one launch does both:
 * the warp that stepped a unit compresses it right away (SEED figures & tables,
 * Figure 1(b): the step, then every W steps the compression), its columns read
 * again from L2 instead of HBM; units that launch's Cholesky-QR path declines are
 * compressed by the Householder path in a second launch over the layer.  Other
 * shapes: a decode launch and a compression launch.  Results, their storage and
 * the errors as with seed_decode_step followed by seed_compress(layer).
 *   sigma_out  optional: [B * H][R] singular values kept (rows of compressed units)  */
int seed_decode_step_compress(const seed_dims* dims, const seed_state* state, int32_t layer,
                              const float* q, const float* k, const float* v, const float* alpha,
                              const float* beta, float* o, float* sigma_out, void* ws,
                              size_t ws_bytes, void* stream);

/* Dense state S = a vbar^T + U V^T (true U, scales applied) of units of `layer`
 * (or all layers).  units: optional list of unit indices within the scope
 * (b * H + h for one layer, the global unit index for all layers); NULL = every
 * unit in scope.  S_out [n][d_k][d_v] row-major.                                */
int seed_state_to_dense(const seed_dims* dims, const seed_state* state, int32_t layer,
                        const int32_t* units, int32_t n_units, float* S_out, void* ws,
                        size_t ws_bytes, void* stream);

/* Energies of the stored states (SEED figures & tables, Figure 3 (f)-(g): the sink
 * holds most of a state's energy; Figure 12 (f): the content energy beyond rank R).
 * For the listed units of `layer` (or all layers; units and n_units as in
 * seed_state_to_dense, NULL = every unit in scope), out[n][4] (float32) receives
 *     [0] ||a vbar^T||_F^2   [1] ||U V^T||_F^2 (true U)   [2] 2 <a vbar^T, U V^T>_F
 *     [3] ||S||_F^2 = [0] + [1] + [2]
 * The sink's share of the state's energy is [0] / [3]; the content C = S - a vbar^T
 * has energy [1] + [2] (the cross term vanishes up to rounding: every update keeps
 * V^T vbar = 0), so with the kept singular values sigma_1..R of the content (returned
 * by the conversion and the compression) the energy beyond rank R is
 * [1] + [2] - sum sigma_i^2.  Reads the state only.                                  */
int seed_state_energy(const seed_dims* dims, const seed_state* state, int32_t layer,
                      const int32_t* units, int32_t n_units, float* out, void* ws, size_t ws_bytes,
                      void* stream);

/* Singular spectra and the top output direction of the stored states (SEED figures &
 * tables, Figure 3 (e): the spectra of the state and of the content, divided by the
 * head's top singular value; Figure 3 (h): |cos| between the head's top output
 * direction v* and vbar; Figure 13 (a): the energy share of the state's i-th
 * singular direction, sigma_i^2 / sum_j sigma_j^2; Figure 13 (d): the rank that holds
 * 90% and 99% of the content's energy).  For the listed units of `layer` (or all
 * layers; units and n_units as in seed_state_to_dense, NULL = every unit in scope):
 *   sigma_state    [n][R+W+1] float  the largest R+W+1 singular values of
 *                                    S = a vbar^T + U V^T (true U), descending; S has
 *                                    rank at most ncols + 1 <= R+W+1
 *   sigma_content  [n][R+W+1] float  the same for the content C = U V^T
 *   cos_top        [n] float         |v*^T vbar| / ||vbar||, v* the right singular vector
 *                                    of S's largest singular value (o = S^T q lies in the
 *                                    span of the right singular vectors)
 *   ranks          [n][2] int32      the smallest k whose k largest singular values of C
 *                                    hold 90% (ranks[.][0]) and 99% ([.][1]) of
 *                                    ||C||_F^2; 0 for a zero content
 * Computed in float32 by a one-sided Jacobi SVD of the explicit d_k x d_v matrices (a
 * diagnostic: about a millisecond per hundred 128 x 128 units, not for the decode
 * loop).  Reads the state only.  Device flags: SEED_FLAG_BADINDEX for a unit index
 * outside the scope (its rows are not written), SEED_FLAG_BADCOLS for a column count
 * outside [0, R+W] (the unit is taken as holding none), SEED_FLAG_NOCONVERGE if a
 * Jacobi SVD reached its sweep cap.                                               */
int seed_state_spectrum(const seed_dims* dims, const seed_state* state, int32_t layer,
                        const int32_t* units, int32_t n_units, float* sigma_state,
                        float* sigma_content, float* cos_top, int32_t* ranks, void* ws,
                        size_t ws_bytes, void* stream);

/* The dense-state step that SEED replaces, kept as the in-run comparison: every
 * decode step loads and stores whole recurrent states (SEED abstract, readsearch.ai).
 * One step of `layer` on a dense state S [B][L][H][d_k][d_v] with the form's dense
 * recurrence, then o = S+^T q.  Arguments as in seed_decode_step.                  */
int seed_dense_step(const seed_dims* dims, float* S, int32_t layer, const float* q,
                    const float* k, const float* v, const float* alpha, const float* beta,
                    float* o, void* ws, size_t ws_bytes, void* stream);

/* Synchronises `stream`, returns the accumulated SEED_FLAG_* bits in *flags and
 * clears them.  Returns SEED_OK or SEED_ERR_CUDA.                                   */
int seed_get_status(void* ws, void* stream, uint32_t* flags);

/* Synchronises `stream`, copies six diagnostic counters kept next to the status
 * word into counters[0..5] and clears them: [0] Jacobi sweeps run by seed_compress,
 * [1] units compressed by its Householder path, [2] Jacobi sweeps run by
 * seed_state_init_from_dense, [3] units it converted, [4] units compressed by the
 * Cholesky-QR path, [5] units the Cholesky-QR path left to the Householder path.
 * Returns SEED_OK or SEED_ERR_CUDA.                                                 */
int seed_get_diagnostics(void* ws, void* stream, uint32_t* counters);

/* Test hook for the bounded waits (no counterpart in the pages).  With enable != 0,
 * every later call on this workspace that waits for bulk copies with a bounded wait
 * -- seed_decode_step's and seed_decode_step_compress's decode warps, and
 * seed_compress's Cholesky-QR blocks with float32 factors -- withholds its first
 * copy and gives up on it at once: the warp raises SEED_FLAG_TIMEOUT, waits (at
 * most 1 s) in vain for the withheld bytes with no copy in flight, and stops, so
 * the units it had not finished are left unchanged (a decode warp fails on its
 * first unit, before touching any unit; a compression block's unit goes to the
 * Householder path as usual).  enable = 0 turns it off; seed_workspace_init clears
 * it.  The workspace word lies past the status word and the counters.              */
int seed_debug_wait_fault(void* ws, size_t ws_bytes, int32_t enable, void* stream);

/* Static description of a seed_status code. */
const char* seed_status_string(int status);

/* ---- Decode step without a caller workspace.  The SEED paper has no counterpart:
 * this is a library convenience for callers that cannot allocate device memory
 * (a host program without a device allocator, an engine that fixes every buffer
 * before serving).  It runs the same kernel as seed_decode_step, with the status
 * word in a 256-byte array that lives in libseed.so's device image (one per
 * device, zero at module load); it calls no allocator.
 *
 * Arguments as in seed_decode_step, without ws / ws_bytes, plus
 *   status_out  optional DEVICE pointer (4-byte aligned) that receives, in stream
 *               order, the SEED_FLAG_* bits this call raised; NULL discards them.
 * After the launch the call copies the status word to status_out and clears it,
 * so every call starts from zero.
 * Returns seed_decode_step's codes, and SEED_ERR_WORKSPACE if the decode step
 * for these dims needs more workspace than the fixed 256 bytes (no supported
 * shape does).  Nothing is enqueued when an argument is rejected.
 * The first call on each device looks up the array's address and may load the
 * module onto the device: make it before any stream capture on that device.
 * The address is kept per device together with the id of the context it was
 * looked up in; after a device reset (cudaDeviceReset, or the primary context
 * released and created again) the next call sees a new context and looks the
 * address up again, so that call too should come before any stream capture.
 * All calls on a device share the one array: calls that can run at the same time
 * (other streams, other host threads) race on the status word; serialise them,
 * or use seed_decode_step with a workspace each.                                  */
size_t seed_noalloc_workspace_bytes(void);
int seed_decode_step_noalloc(const seed_dims* dims, const seed_state* state, int32_t layer,
                             const float* q, const float* k, const float* v, const float* alpha,
                             const float* beta, float* o, uint32_t* status_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SEED_H_ */
