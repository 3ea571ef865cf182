/*
 * kvsculpt.h - C ABI of the B200 library for the KVSculpt distillation solve.
 *
 * Method: "KVSculpt: KV Cache Compression as Distillation" (arXiv 2603.27819).
 * Given a RoPE'd KV cache of N pairs, the compress zone (oldest z = N - m
 * pairs) is replaced by k free pairs (K_c, V_c) that reproduce the zone's
 * attention output Y and log-sum-exp l for a set of training queries
 * (section 2 "Methodology", "Problem Formulation" and "Loss Function").  Keys
 * are optimised by L-BFGS, values are re-solved in closed form by ridge
 * regression, alternating every few steps (Abstract; section 2 "Optimization
 * Strategy"); the keys start from the top-k positions by attention importance
 * ("Initialization"); a pilot run redistributes the budget k across
 * problems ("Adaptive Budget Allocation").
 *
 * Conventions shared by every call
 * --------------------------------
 * - A batch holds B independent head-problems (one per layer x KV head x
 *   sequence).  Per-problem tensors are concatenated along rows; problem b
 *   owns rows [off[b], off[b+1]) of each array.  Three offset arrays describe
 *   a batch: q_off (training queries, n_q_b rows), z_off (compress zone, z_b
 *   rows), c_off (compressed pairs, k_b rows).  Each is given twice: a device
 *   copy (read by kernels) and a host copy (read for validation and launch
 *   sizes); the two must hold the same values.
 * - Every matrix is row-major float32 with d = 64 or 128 columns; "device"
 *   pointers are CUDA global memory of the current device and must be 16-byte
 *   aligned.  The caller owns all memory: the library allocates no device
 *   memory.  Scratch comes from the caller's workspace `ws`
 *   (kvs_workspace_bytes) and L-BFGS state from `state`
 *   (kvs_lbfgs_state_bytes); both must be 256-byte aligned.
 * - Score scale s = 1/sqrt(d).  LSE is the natural-log log-sum-exp of the
 *   scaled scores.  Attention of a training query covers one chunk only (the
 *   compress zone for targets, the k compressed pairs for the distilled
 *   cache), so chunk results merge with the retain zone and future tokens by
 *   their LSE.
 * - All calls except kvs_pilot_allocate are asynchronous on `stream` (a
 *   cudaStream_t passed as void*; NULL = legacy default stream) and never
 *   synchronise the host.  Return value: KVS_OK or a negative KVS_E* code for
 *   a call error (nothing was launched for KVS_EINVAL / KVS_EWORKSPACE).
 *   Numerical outcomes are reported per problem as bits in int32 status[B]
 *   (KVS_ST_*); no kernel traps or asserts.
 * - Calls on distinct workspaces/state buffers may run concurrently; calls
 *   sharing a workspace must be ordered on one stream.
 */
#ifndef KVSCULPT_H
#define KVSCULPT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* call errors */
#define KVS_OK          0
#define KVS_EINVAL     -1   /* bad argument: null/unaligned pointer, bad shape or offsets */
#define KVS_ECUDA      -2   /* a CUDA runtime call failed (kvs_last_cuda_error() tells which) */
#define KVS_ENOTSUP    -3   /* unsupported configuration (e.g. d not 64/128, no sm_100 device) */
#define KVS_EWORKSPACE -4   /* workspace or state buffer smaller than required */

/* per-problem status bits */
#define KVS_ST_NONFINITE 1  /* a loss, gradient or solve produced inf/nan */
#define KVS_ST_NOT_PD    2  /* ridge Gram matrix not positive definite (Cholesky pivot <= 0) */
#define KVS_ST_LS_FAIL   4  /* max_bt Armijo trials failed: x kept, history cleared */
#define KVS_ST_TIMEOUT   8  /* a kernel's bounded wait expired (results of the call unreliable) */

typedef struct kvs_batch {
  int32_t B;                 /* number of head-problems, >= 1 */
  int32_t d;                 /* head dimension: 64 or 128 */
  const int64_t *q_off;      /* device [B+1] training-query row offsets (q_off[0] = 0) */
  const int64_t *z_off;      /* device [B+1] compress-zone row offsets */
  const int64_t *c_off;      /* device [B+1] compressed-pair row offsets (ragged k_b) */
  const int64_t *q_off_h;    /* host copies of the three arrays above */
  const int64_t *z_off_h;
  const int64_t *c_off_h;
} kvs_batch;

typedef struct kvs_schedule {
  int32_t outer;             /* outer iterations: value re-fits after the initial one */
  int32_t steps;             /* L-BFGS steps per outer iteration */
  int32_t history;           /* L-BFGS pairs kept (1..15) */
  int32_t max_bt;            /* Armijo trials per step (1..64) */
  int32_t persist_history;   /* 1: keep (s,y) pairs across value re-fits; 0: clear them */
  float lambda;              /* ridge penalty, absolute */
  float w_out;               /* weight of the output term, mean over n_q*d */
  float w_lse;               /* weight of the LSE term, mean over n_q */
  float c1;                  /* Armijo sufficient-decrease constant */
  float backtrack;           /* step factor per rejected trial (0,1) */
} kvs_schedule;

/* Geometry of the training-query construction (uniform across the batch). */
typedef struct kvs_query_spec {
  int32_t B, d;
  int32_t g;                 /* query heads per KV head */
  int32_t m_q;               /* retain queries per query head */
  int32_t n_syn;             /* synthetic future queries per query head */
  int32_t N;                 /* context length: synthetic query j goes to position N + j */
  float rope_base;           /* RoPE base (rotate-half pairing, theta_i = base^(-2i/d)) */
} kvs_query_spec;

/* Library version / diagnostics. */
const char *kvs_version(void);
const char *kvs_last_cuda_error(void);     /* text of the last CUDA error seen by this thread */
uint64_t kvs_launch_count(void);           /* kernels this library has launched in this process */

/* Failure detection.  Every wait inside the tensor-core kernels is bounded: a
 * kernel whose pipeline wait spins longer than the limit stops, lets the
 * copies and MMAs it already issued complete, and raises the call's timeout
 * flag.  Calls with a status array report it as KVS_ST_TIMEOUT in every
 * problem; kvs_targets, kvs_loss_grad and kvs_loss_grad_static, which have no
 * status array, then write NaN into every element of their outputs instead.
 * kvs_set_wait_limit sets the limit in SM clock cycles for launches issued
 * after it, process-wide (0 restores the default, about 2 s; a CUDA graph
 * keeps the limit it was recorded with).  It exists to test this path with a
 * limit too short for any wait to succeed; KVS_EINVAL for cycles < 0. */
int kvs_set_wait_limit(int64_t cycles);

/* Bytes of scratch workspace needed by every call below for this batch
 * (and schedule; may be NULL when no L-BFGS call will use the workspace),
 * kvs_compress_batch's sub-batches included.  Returns 0 for an invalid batch. */
size_t kvs_workspace_bytes(const kvs_batch *batch, const kvs_schedule *sched);

/* Bytes of persistent L-BFGS state for this batch and history length (enough
 * for kvs_lbfgs_reset / kvs_lbfgs_step and for kvs_compress_batch). */
size_t kvs_lbfgs_state_bytes(const kvs_batch *batch, int32_t history);

/* Where the L-BFGS state of kvs_lbfgs_step lives inside a state buffer
 * (host only; for inspection and tests: the solver needs none of it).  All
 * offsets are in bytes from the start of the buffer.
 *   scalars + b * scalar_bytes: problem b's record, holding at off_f the
 *     float loss f at x, at off_count the int32 number of stored pairs and at
 *     off_head the int32 ring slot the next pair goes to;
 *   x, g, dir: float [sum k_b * d] vectors (problem b at c_off[b] * d): the
 *     accepted keys, the gradient there and the last search direction;
 *   ring_s, ring_y: `slots` = history + 1 vectors each, ring_stride bytes
 *     apart, holding s = x_new - x_old and y = g_new - g_old of the stored
 *     pairs: pair p (p = 0 the newest, p < count) of a problem sits in slot
 *     (head - 1 - p) mod slots.
 * KVS_EINVAL for a null `out`, an invalid batch or history outside 1..15. */
typedef struct kvs_lbfgs_layout {
  uint64_t scalars, scalar_bytes, off_f, off_count, off_head;
  uint64_t x, g, dir, ring_s, ring_y, ring_stride;
  int32_t slots;
} kvs_lbfgs_layout;
int kvs_lbfgs_state_layout(const kvs_batch *batch, int32_t history, kvs_lbfgs_layout *out);

/* Training queries (section 2 "Training Query Construction").
 * q_retain [B*g*m_q, d]: retain queries, already RoPE'd at their positions,
 *   copied through.  q_ctx [B*g*n_syn, d]: sampled context queries RoPE'd at
 *   pos [B*g*n_syn] (int32, the method's uniform draw); each is de-RoPE'd at
 *   its position and re-embedded at position N + j (j = its rank within its
 *   query head).  Q [B*g*(m_q+n_syn), d] receives rows ordered by problem,
 *   query head, then retain rows, then synthetic rows. */
int kvs_build_queries(const kvs_query_spec *spec, const float *q_retain, const float *q_ctx,
                      const int32_t *pos, float *Q, void *stream);

/* Distillation targets over the compress zone (section 2 "Problem Formulation",
 * "Loss Function"): S0 = s Q Kz^T, lse[i] = LSE_j S0[i,j],
 * Y = softmax(S0) Vz.  If `importance` is non-NULL it also receives
 * importance[j] = sum_i exp(S0[i,j] - lse[i]) over the problem's z_b keys
 * (section 2 "Initialization": attention importance), rows by z_off.
 * Q [sum n_q, d], Kz/Vz [sum z, d]; Y [sum n_q, d]; lse [sum n_q].
 * If a kernel's bounded wait gave up, Y, lse and importance are all NaN. */
int kvs_targets(const kvs_batch *batch, const float *Q, const float *Kz, const float *Vz,
                float *Y, float *lse, float *importance, void *ws, size_t ws_bytes, void *stream);

/* Top-k initialisation (section 2 "Initialization"): per problem, the k_b
 * positions with the largest importance (ties to the lower position), in
 * ascending order, into idx [sum k_b] (int32, position within the problem's
 * zone), and Kc[c_off[b] + r] = Kz[z_off[b] + idx[r]].  Requires
 * 1 <= k_b <= z_b and z_b <= 16384. */
int kvs_init_topk(const kvs_batch *batch, const float *importance, const float *Kz,
                  int32_t *idx, float *Kc, void *stream);

/* Distillation loss and its gradient with respect to K_c (section 2 "Loss
 * Function"):  A = softmax(s Q Kc^T), Yh = A Vc, lh = LSE(s Q Kc^T),
 * loss[b] = w_out/(n_q d) ||Yh - Y||_F^2 + w_lse/n_q ||lh - lse||^2, and
 * dKc = dloss/dKc [sum k_b, d].  dKc may be NULL (loss only).
 * parts (nullable) [B,2] receives the unweighted output-MSE and LSE-MSE.
 * If a kernel's bounded wait gave up, loss, parts and dKc are all NaN. */
int kvs_loss_grad(const kvs_batch *batch, const float *Q, const float *Kc, const float *Vc,
                  const float *Y, const float *lse, float w_out, float w_lse,
                  float *loss, float *parts, float *dKc, void *ws, size_t ws_bytes,
                  void *stream);

/* kvs_loss_grad for callers that cannot allocate device memory.  The paper
 * has no counterpart to this call; it exists for deployment.  Some callers
 * cannot call cudaMalloc to provide a workspace: a plug-in inside a host
 * application that owns all device memory through its own pool and forbids
 * side allocations, or a service that must fix its device footprint when the
 * library loads.  This call computes exactly what kvs_loss_grad computes, with
 * its scratch taken from one array compiled into the library: 32 MiB
 * (KVS_STATIC_WS_BYTES in kvs_static.cu) of device memory on every GPU that
 * loads the library, held until the process exits.  It allocates nothing.
 * - Batches whose kvs_workspace_bytes() exceeds 32 MiB return KVS_EWORKSPACE
 *   (one head-problem with d = 128, n_q = 3840 and k = 960 fits; two do not).
 * - The first call on a device looks up the array's device address with that
 *   device current (cudaGetSymbolAddress) and caches it with the context it
 *   belongs to; a call under another context (after cudaDeviceReset, or with
 *   another driver context current) looks it up again.  Make the first call
 *   in each context before any stream capture.
 * - Every call on a device shares the one array and the array keeps the last
 *   call's contents.  No part of it needs to start at zero for this call.
 *   Calls whose work overlaps on the GPU (other streams, other host threads)
 *   race on it: order them, e.g. on one stream.
 * Arguments, outputs and errors are those of kvs_loss_grad. */
int kvs_loss_grad_static(const kvs_batch *batch, const float *Q, const float *Kc,
                         const float *Vc, const float *Y, const float *lse, float w_out,
                         float w_lse, float *loss, float *parts, float *dKc, void *stream);

/* Closed-form values (section 2 "Value Optimization"): with A = softmax(s Q Kc^T)
 * fixed, Vc = (A^T A + lambda I)^-1 A^T Y, by Cholesky.  A problem whose Gram
 * matrix is not positive definite gets KVS_ST_NOT_PD in status[b] (OR-ed in)
 * and keeps its previous Vc; so does a problem whose solution is not finite,
 * which gets KVS_ST_NONFINITE (a Gram matrix with a non-finite entry counts
 * as not positive definite).
 * The factorisation forks part of its work onto one internal high-priority
 * stream (created once per host thread and device) through events recorded on
 * `stream`, and joins it back to `stream` before returning, so the call stays
 * ordered on `stream` (every entry point that fits values, kvs_compress_batch
 * too, behaves this way). */
int kvs_fit_values(const kvs_batch *batch, const float *Q, const float *Kc, const float *Y,
                   float lambda, float *Vc, int32_t *status, void *ws, size_t ws_bytes,
                   void *stream);

/* (Re)start L-BFGS at the current Kc and Vc: evaluates loss and gradient into
 * `state`, clears the (s, y) history when clear_history != 0 (always on the
 * first call for a state buffer) and zeroes the step counters. */
int kvs_lbfgs_reset(const kvs_batch *batch, const kvs_schedule *sched, const float *Q,
                    const float *Y, const float *lse, const float *Vc, const float *Kc,
                    void *state, size_t state_bytes, int32_t clear_history,
                    void *ws, size_t ws_bytes, void *stream);

/* One L-BFGS iteration on Kc for every problem (section 2 "Key Optimization"):
 * two-loop direction from the history (H0 = gamma I), deterministic
 * backtracking Armijo search (first trial 1, or min(1, 1/||g||) with empty
 * history; factor sched->backtrack; at most sched->max_bt trials), history
 * update when s^T y > 1e-10 y^T y.  Kc is updated in place; a failed search
 * leaves Kc unchanged, clears the history and sets KVS_ST_LS_FAIL.  A loss
 * that evaluates to inf or NaN (at a trial point, or at the point the last
 * reset started from) sets KVS_ST_NONFINITE; such a trial is rejected.
 * f_out (nullable) [B] receives the loss after the step. */
int kvs_lbfgs_step(const kvs_batch *batch, const kvs_schedule *sched, const float *Q,
                   const float *Y, const float *lse, const float *Vc, float *Kc,
                   void *state, size_t state_bytes, int32_t *status, float *f_out,
                   void *ws, size_t ws_bytes, void *stream);

/* One Adam step on Kc, the ablation of the key optimiser (section 4 "Optimizer
 * Efficacy": Adam in place of L-BFGS leaves a much larger per-layer error).
 * With g = dKc [sum_c, d] (e.g. from kvs_loss_grad), elementwise over all
 * sum_c x d values of the batch:
 *   m <- beta1 m + (1 - beta1) g,   v <- beta2 v + (1 - beta2) g^2,
 *   Kc <- Kc - lr (m / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + eps).
 * m, v: caller buffers [sum_c, d] (float32, 16-byte aligned), zero before the
 * first step and carried between steps; t >= 1 counts the steps taken so far
 * including this one.  Errors: KVS_EINVAL for a null or unaligned pointer,
 * t < 1, lr <= 0, beta outside [0, 1) or eps <= 0. */
int kvs_adam_step(const kvs_batch *batch, float *Kc, const float *dKc, float *m, float *v,
                  int32_t t, float lr, float beta1, float beta2, float eps, void *stream);

/* The whole alternating solve for a batch (Abstract; section 2): targets,
 * importance, top-k keys, ridge values (the Select+Fit state), then
 * sched->outer times { sched->steps L-BFGS steps; ridge re-fit }.
 * Outputs Kc, Vc [sum k_b, d]; idx (nullable) [sum k_b] the top-k positions;
 * loss_trace (nullable) [B, outer+1] the loss after every fit; parts
 * (nullable) [B, 2] final unweighted output-MSE and LSE-MSE; status [B].
 * After its first step each L-BFGS step runs as one CUDA graph whose trial
 * loop is a conditional node; with the environment variable
 * KVS_STEP_GRAPHS=0 (read once per process) the same kernels are launched
 * one by one instead, for kernel-level profilers.
 * A batch of 8 or more problems is solved as sub-batches of contiguous
 * problems (two from 8 problems, four from 16; cut where the work
 * n_q k (d + k) splits evenly), all but the first on internal streams forked
 * from and joined back to `stream`, so that the latency-bound steps of one
 * overlap the tensor-core work of the others; the results are those of solving
 * each problem on its own.  `state` is then
 * scratch laid out per sub-batch (kvs_lbfgs_state_layout does not apply). */
int kvs_compress_batch(const kvs_batch *batch, const kvs_schedule *sched, const float *Q,
                       const float *Kz, const float *Vz, float *Kc, float *Vc, int32_t *idx,
                       float *loss_trace, float *parts, int32_t *status,
                       void *state, size_t state_bytes, void *ws, size_t ws_bytes,
                       void *stream);

/* Adaptive budget (section 2 "Adaptive Budget Allocation"; host only, no CUDA):
 * k_out[b] shares `total` in proportion to pilot_mse[b]^alpha, clamped to
 * [k_min, k_max[b]] (the clamped real shares x_b = clip(c w_b) with sum =
 * total), then rounded by largest remainder (ties to the lower index) so that
 * sum k_out = total.  Non-finite or non-positive MSEs weigh 0; all-zero
 * weights share uniformly.  KVS_EINVAL if total is outside
 * [B*k_min, sum k_max]. */
int kvs_pilot_allocate(int32_t B, const float *pilot_mse, int64_t total, int32_t k_min,
                       const int32_t *k_max, float alpha, int32_t *k_out);

#ifdef __cplusplus
}
#endif

#endif /* KVSCULPT_H */
