// Internal launchers shared by the C-ABI layer (not part of the public ABI).
#pragma once

#include <cuda_bf16.h>

#include "kvs_common.cuh"

namespace kvs {

// Most sub-batches a solve runs concurrently (kvs_compress_batch).
constexpr int KVS_MAX_PARTS = 4;

// L-BFGS line-search phase of a problem.
enum Phase : int { PH_IDLE = 0, PH_SEARCH = 1, PH_ACCEPT = 2, PH_FAIL = 3 };

// Per-problem scalar state of L-BFGS (lives in the caller's state buffer).
struct LbfgsScal {
  float f;        // loss at x
  float ft;       // loss at the current trial point
  float t;        // current trial step
  float gtd;      // g . d of the current direction
  float gamma;    // s . y / y . y of the newest stored pair (H0 = gamma I)
  float rho[16];  // 1 / (s_i . y_i) per ring slot
  int count;      // valid pairs in the ring
  int head;       // next ring slot to write
  int phase;      // Phase
  int trials;     // trials of the current search
  int lse_stale;  // 1: the workspace l_hat is not that of the accepted keys (failed search)
  int nonfinite;  // 1: a loss or gradient evaluated since the last report was inf / NaN
  int pad;
};

// Scratch buffers carved from the caller's workspace.
// The bf16 operand copies hold each problem's rows at padded offsets (rows
// rounded up to 128 per problem) with zero rows in the padding.
struct Work {
  __nv_bfloat16 *qh = nullptr, *ql = nullptr;    // [sum_qpad, d]        training queries, hi/lo
  __nv_bfloat16 *kh = nullptr, *kl = nullptr;    // [max(zpad, cpad), d] keys, hi/lo
  __nv_bfloat16 *vh = nullptr, *vl = nullptr;    // [max(zpad, cpad), d] values, hi/lo
  __nv_bfloat16 *go = nullptr;                   // [sum_qpad, d]        dloss/dY_hat
  __nv_bfloat16 *yh = nullptr, *yl = nullptr;    // [sum_qpad, d]        targets Y, hi/lo
  __nv_bfloat16 *ahi = nullptr, *alo = nullptr;  // [sum_qpad, ld_a]     attention weights for the ridge fit
  float *lse_h = nullptr;          // [sum_q]              row lse of the compressed keys
  float *delta = nullptr;          // [sum_q]
  float *partials = nullptr;       // [B, max q tiles, 2]  per-CTA loss sums
  int64_t *a_pad_off = nullptr;    // [B+1]                padded query-row offsets (qh, ql, go,
                                   //                      yh, yl, ahi, alo): n_q rounded up to 128
  int64_t *z_pad = nullptr, *c_pad = nullptr;  // [B+1] each  padded zone / pair rows of kh .. vl
  float *gram = nullptr;           // [sum_c, ld_g]        A^T A + lam I, then its Cholesky factor
  float *R = nullptr;              // [sum_c, d]           A^T Y, then the forward-solved rows
  float *X = nullptr;              // [sum_c, d]           solution of the ridge system
  float *dkp = nullptr;            // [4, sum_c, d]        key-gradient partial sums of query splits
  float *chol_t = nullptr;         // [B, panels, 64, 64]  transposed inverses of the diagonal blocks
  float *chol_p = nullptr;         // [2, 2, sum_c, 64]    tf32 hi / lo of a panel's factor rows;
                                   //                      shares dkp's memory (the fit and the key
                                   //                      gradient never run at once on one workspace)
  float *chol_y = nullptr;         // [2, 2, B d, 64]      tf32 hi / lo of the forward-solved rows
  int *dead = nullptr;             // [B]                  factorisation failed
  float *fbuf = nullptr;           // [B]                  loss scratch
  float *Yt = nullptr;             // [sum_q, d]           targets (kvs_compress_batch)
  float *lset = nullptr;           // [sum_q]              target log-sum-exp (kvs_compress_batch)
  float *imp = nullptr;            // [sum_z]              importance (kvs_compress_batch)
  int32_t *idx = nullptr;          // [sum_c]              top-k positions (kvs_compress_batch)
  int *err = nullptr;              // [1]                  set when a kernel wait timed out
  size_t bytes = 0;
};

// Persistent L-BFGS state carved from the caller's state buffer.
// Inner products of the stored pairs, indexed by ring slot: sy[i][j] = s_i . y_j
// (filled for s older than y and on the diagonal), yy[i][j] = y_i . y_j.
struct LbfgsGram {
  double sy[16][16];
  double yy[16][16];
};

// The next search direction as a combination d = cg g + sum_p (cy[p] y_p + cs[p] s_p)
// over the cnt newest pairs (p = 0 newest), with g . d and the first trial step.
struct DirCoef {
  float cg, gtd, t0;
  int cnt;
  float cy[16], cs[16];
};

constexpr int LBFGS_CHUNK = 2048;  // elements of a problem's vector per CTA
constexpr int LBFGS_NDOT = 65;     // inner products one CTA reports (h <= 15)

struct State {
  LbfgsScal *sc;   // [B]
  LbfgsGram *gram; // [B]
  DirCoef *dc;     // [B]
  float *part;     // [B][cmax][LBFGS_NDOT] per-CTA partial inner products
  int *ticket;     // [B] CTAs of the current pass that have finished
  int cmax;        // chunks of the longest problem
  float *x;        // [sum_c*d] accepted keys
  float *g;        // [sum_c*d] gradient at x
  float *dir;      // [sum_c*d] search direction
  float *gn;       // [sum_c*d] gradient at the accepted trial point
  float *ring_s;   // [h+1][sum_c*d]  ring of step differences (slot `head` is scratch)
  float *ring_y;   // [h+1][sum_c*d]  ring of gradient differences
  int h;
  size_t bytes;
};

size_t carve_work(const HostGeom &g, void *base, Work *w);
size_t carve_state(const HostGeom &g, int h, void *base, State *s);

struct Batch {
  HostGeom g;
  const kvs_batch *b;
  cudaStream_t st;
  int slot = 0;   // sub-batch index of a partitioned solve (its own internal streams)
  int share = 1;  // sub-batches that run at the same time (each sizes its grids for 1/share of the SMs)
};

// ---- attention contractions (kvs_attn.cu) ----
// Padded row offsets of the batch's queries, zones and (if any) pairs into the
// workspace (w.a_pad_off, w.z_pad, w.c_pad).
int launch_pad_offsets(const Batch &B, const Work &w);
// targets: Y, lse and (optionally) importance; leaves the Q split in w.qh/ql
// and the Y split in w.yh/yl.
int launch_targets(const Batch &B, const float *Q, const float *Kz, const float *Vz, float *Y,
                   float *lse, float *imp, const Work &w);
// Loss forward over the compressed pairs for the problems selected by `flt`:
// writes loss[b] (and parts[2b..2b+1] if non-null) and leaves lse_h, go and
// delta (plus the bf16 copies of Kc) for launch_backward.  q_ready: the
// Q split in w.qh/ql is current.
int launch_forward(const Batch &B, const float *Q, const float *Kc, const float *Vc,
                   const float *Y, const float *lse, float w_out, float w_lse, float *loss,
                   float *parts, Filter flt, bool q_ready, const Work &w,
                   bool pairs_ready = false, bool reduce = true);
// bf16 hi/lo copies of the compressed pairs (keys; values unless Vc is null).
// kflt: the problems whose K_c split is redone (all by default).
int launch_split_pairs(const Batch &B, const float *Kc, const float *Vc, const Work &w,
                       Filter kflt = Filter{nullptr, 0, 0});
// dKc from the state left by launch_forward for the same problems (with the same
// values Vc and output weight w_out).
int launch_backward(const Batch &B, const float *Vc, float w_out, float *dKc, Filter flt,
                    const Work &w);
// Ridge fit: Vc = (A^T A + lam I)^-1 A^T Y (y_ready: the Y split is current).  The
// row log-sum-exp of Kc is recomputed for the problems `stats` selects; the others
// take the one the last loss forward left in the workspace.
int launch_fit(const Batch &B, const float *Q, const float *Kc, const float *Y, float lam,
               float *Vc, int32_t *status, bool q_ready, bool y_ready, const Work &w,
               Filter stats = Filter{nullptr, 0, 0});

// Multiprocessor count of the current device (cached).
int sm_count();

// ---- other kernels ----
int launch_build_queries(const kvs_query_spec *sp, const float *q_retain, const float *q_ctx,
                         const int32_t *pos, float *Q, cudaStream_t st);
int launch_topk(const Batch &B, const float *imp, const float *Kz, int32_t *idx, float *Kc);
int launch_chol_solve(const Batch &B, float *Vc, int32_t *status, const Work &w);

// L-BFGS pieces (kvs_lbfgs.cu)
int launch_lbfgs_reset(const Batch &B, const State &s, const float *Kc, const float *f,
                       const float *g, int clear);
int launch_lbfgs_direction(const Batch &B, const State &s, const kvs_schedule &sc);
// Kc = x + t d for searching problems, with its bf16 hi/lo split into w.kh/w.kl
// (at the padded pair rows).
int launch_lbfgs_trial(const Batch &B, const State &s, float *Kc, const Work &w);
// Armijo test on the trial loss summed from the forward's per-CTA partials;
// with `cond`, also sets that graph condition to "a problem is still searching".
int launch_lbfgs_armijo(const Batch &B, const State &s, const kvs_schedule &sc, const Work &w,
                        const cudaGraphConditionalHandle *cond = nullptr);
int launch_lbfgs_update(const Batch &B, const State &s, float *Kc, int32_t *status,
                        float *f_out);
int launch_copy_f(const Batch &B, const State &s, float *dst, int64_t stride, int64_t col);

// Adam ablation (kvs_adam.cu): one elementwise Adam step over n key values
// (bc1, bc2: the bias corrections 1 - beta^t).
int launch_adam(float *Kc, const float *dKc, float *m, float *v, int64_t n, float lr, float b1,
                float b2, float eps, float bc1, float bc2, cudaStream_t st);

}  // namespace kvs
