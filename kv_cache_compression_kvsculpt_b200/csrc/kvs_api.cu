// C ABI of the KVSculpt library: argument validation, workspace layout and
// the orchestration of the kernels for each call (see include/kvsculpt.h).
#include <stdlib.h>
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <map>
#include <mutex>
#include <cstddef>
#include <vector>

#include "kvs_internal.cuh"

namespace kvs {

static thread_local char g_err[256] = "no error";
static std::atomic<uint64_t> g_launches{0};
static std::atomic<long long> g_wait_limit{0};  // 0: the default limit

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

long long wait_limit() {
  const long long v = g_wait_limit.load(std::memory_order_relaxed);
  return v > 0 ? v : tc_wait_default();
}

cudaError_t set_smem_once_impl(const void *kern, int bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void *, int>, int> done;  // (kernel, device) -> bytes set
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto it = done.find({kern, dev});
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done[{kern, dev}] = bytes;
  return e;
}

void set_cuda_error(cudaError_t e, const char *where) {
  snprintf(g_err, sizeof g_err, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

void set_driver_error(int code, const char *where) {
  snprintf(g_err, sizeof g_err, "%s: CUresult %d", where, code);
}

static bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

static int check_offsets(const int64_t *off, int B, int64_t *sum, int *mx, bool allow_empty) {
  if (!off || off[0] != 0) return KVS_EINVAL;
  int64_t m = 0;
  for (int b = 0; b < B; ++b) {
    const int64_t n = off[b + 1] - off[b];
    if (n < (allow_empty ? 0 : 1) || n > (1 << 30)) return KVS_EINVAL;
    m = std::max(m, n);
  }
  *sum = off[B];
  *mx = (int)m;
  return KVS_OK;
}

int geom_from_batch(const kvs_batch *b, HostGeom *g, bool need_c) {
  if (!b || b->B < 1 || (b->d != 64 && b->d != 128)) return b && b->B >= 1 ? KVS_ENOTSUP : KVS_EINVAL;
  if (!b->q_off || !b->z_off || !b->q_off_h || !b->z_off_h) return KVS_EINVAL;
  *g = HostGeom{};
  g->B = b->B;
  g->d = b->d;
  if (check_offsets(b->q_off_h, b->B, &g->sum_q, &g->max_q, false)) return KVS_EINVAL;
  if (check_offsets(b->z_off_h, b->B, &g->sum_z, &g->max_z, false)) return KVS_EINVAL;
  if (need_c) {
    if (!b->c_off || !b->c_off_h) return KVS_EINVAL;
    if (check_offsets(b->c_off_h, b->B, &g->sum_c, &g->max_c, false)) return KVS_EINVAL;
  } else if (b->c_off_h) {
    if (check_offsets(b->c_off_h, b->B, &g->sum_c, &g->max_c, true)) return KVS_EINVAL;
  }
  for (int bb = 0; bb < b->B; ++bb) {
    g->sum_qpad += align_up(b->q_off_h[bb + 1] - b->q_off_h[bb], 128);
    g->sum_zpad += align_up(b->z_off_h[bb + 1] - b->z_off_h[bb], 128);
    if (b->c_off_h) g->sum_cpad += align_up(b->c_off_h[bb + 1] - b->c_off_h[bb], 128);
  }
  g->ld_a = align_up(std::max(g->max_c, 1), 128);
  g->ld_g = align_up(std::max(g->max_c, 1), 4);
  return KVS_OK;
}

// Bump allocator over a caller buffer (256-byte aligned pieces).
struct Carver {
  char *base;
  size_t off = 0;
  template <class T>
  T *take(int64_t count) {
    off = (size_t)align_up((int64_t)off, 256);
    T *p = base ? reinterpret_cast<T *>(base + off) : nullptr;
    off += (size_t)std::max<int64_t>(count, 0) * sizeof(T);
    return p;
  }
};

size_t carve_work(const HostGeom &g, void *base, Work *w) {
  Carver c{static_cast<char *>(base)};
  // tensor-core operands: rows padded to 128 per problem (zero rows), so that no
  // tile reaches into another problem's rows
  const int64_t kz = std::max(g.sum_zpad, g.sum_cpad);
  w->qh = c.take<__nv_bfloat16>(g.sum_qpad * g.d);
  w->ql = c.take<__nv_bfloat16>(g.sum_qpad * g.d);
  w->kh = c.take<__nv_bfloat16>(kz * g.d);
  w->kl = c.take<__nv_bfloat16>(kz * g.d);
  w->vh = c.take<__nv_bfloat16>(kz * g.d);
  w->vl = c.take<__nv_bfloat16>(kz * g.d);
  w->go = c.take<__nv_bfloat16>(g.sum_qpad * g.d);
  w->yh = c.take<__nv_bfloat16>(g.sum_qpad * g.d);
  w->yl = c.take<__nv_bfloat16>(g.sum_qpad * g.d);
  w->ahi = c.take<__nv_bfloat16>(g.sum_qpad * g.ld_a);
  w->alo = c.take<__nv_bfloat16>(g.sum_qpad * g.ld_a);
  w->lse_h = c.take<float>(g.sum_q);
  w->delta = c.take<float>(g.sum_q);
  w->partials = c.take<float>((int64_t)g.B * ((g.max_q + 127) / 128) * 2);
  w->a_pad_off = c.take<int64_t>(g.B + 1);
  w->z_pad = c.take<int64_t>(g.B + 1);
  w->c_pad = c.take<int64_t>(g.B + 1);
  w->gram = c.take<float>(g.sum_c * g.ld_g);
  w->R = c.take<float>(g.sum_c * g.d);
  w->X = c.take<float>(g.sum_c * g.d);
  w->dkp = c.take<float>(4 * g.sum_c * g.d);  // 4 d >= 2 x 2 x 64 floats per row (d >= 64)
  w->chol_p = w->dkp;
  w->chol_t = c.take<float>((int64_t)g.B * ((g.max_c + 63) / 64) * 64 * 64);
  w->chol_y = c.take<float>(4 * (int64_t)g.B * g.d * 64);
  w->dead = c.take<int>(g.B);
  w->fbuf = c.take<float>(g.B);
  w->Yt = c.take<float>(g.sum_q * g.d);
  w->lset = c.take<float>(g.sum_q);
  w->imp = c.take<float>(g.sum_z);
  w->idx = c.take<int32_t>(g.sum_c);
  w->err = c.take<int>(1);
  w->bytes = align_up((int64_t)c.off, 256);
  return w->bytes;
}

size_t carve_state(const HostGeom &g, int h, void *base, State *s) {
  Carver c{static_cast<char *>(base)};
  const int64_t n = g.sum_c * g.d;
  s->sc = c.take<LbfgsScal>(g.B);
  s->gram = c.take<LbfgsGram>(g.B);
  s->dc = c.take<DirCoef>(g.B);
  s->cmax = (int)(((int64_t)g.max_c * g.d + LBFGS_CHUNK - 1) / LBFGS_CHUNK);
  s->part = c.take<float>((int64_t)g.B * s->cmax * LBFGS_NDOT);
  s->ticket = c.take<int>(g.B);
  s->x = c.take<float>(n);
  s->g = c.take<float>(n);
  s->dir = c.take<float>(n);
  s->gn = c.take<float>(n);
  s->ring_s = c.take<float>((int64_t)(h + 1) * n);
  s->ring_y = c.take<float>((int64_t)(h + 1) * n);
  s->h = h;
  s->bytes = align_up((int64_t)c.off, 256);
  return s->bytes;
}

static int prep(const kvs_batch *b, bool need_c, void *ws, size_t ws_bytes, void *stream,
                Batch *Bt, Work *w) {
  int rc = geom_from_batch(b, &Bt->g, need_c);
  if (rc) return rc;
  Bt->b = b;
  Bt->st = static_cast<cudaStream_t>(stream);
  if (!ws || !aligned(ws, 256)) return KVS_EINVAL;
  if (carve_work(Bt->g, nullptr, w) > ws_bytes) return KVS_EWORKSPACE;
  carve_work(Bt->g, ws, w);
  return KVS_OK;
}

// First device work of a call, after every argument check has passed: clear the
// timeout flag and lay out the padded operand rows.
static int begin(const Batch &Bt, const Work &w) {
  KVS_CUDA_TRY(cudaMemsetAsync(w.err, 0, sizeof(int), Bt.st));
  return launch_pad_offsets(Bt, w);
}

// status[b] |= KVS_ST_TIMEOUT when a kernel of the call gave up waiting.
__global__ void k_fold_err(const int *err, int32_t *status, int B) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B && *err) status[b] |= KVS_ST_TIMEOUT;
}

static int fold_err(const Batch &Bt, const Work &w, int32_t *status) {
  if (!status) return KVS_OK;
  k_fold_err<<<(Bt.g.B + 127) / 128, 128, 0, Bt.st>>>(w.err, status, Bt.g.B);
  KVS_LAUNCH_CHECK("k_fold_err");
  return KVS_OK;
}

// For the calls without a status array: when a kernel of the call gave up
// waiting, every output element becomes NaN, so partial results cannot pass
// for finite ones.
struct NanOut {
  float *p[3];
  int64_t n[3];
};

__global__ void k_nan_if_err(const int *err, NanOut o) {
  if (!*err) return;
  for (int k = 0; k < 3; ++k)
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < o.n[k];
         i += (int64_t)gridDim.x * blockDim.x)
      o.p[k][i] = __int_as_float(0x7fc00000);
}

static int nan_if_err(const Batch &Bt, const Work &w, float *p0, int64_t n0, float *p1, int64_t n1,
                      float *p2, int64_t n2) {
  NanOut o{{p0, p1, p2}, {p0 ? n0 : 0, p1 ? n1 : 0, p2 ? n2 : 0}};
  k_nan_if_err<<<64, 256, 0, Bt.st>>>(w.err, o);
  KVS_LAUNCH_CHECK("k_nan_if_err");
  return KVS_OK;
}

static bool ok_ptr(const void *p) { return p && aligned(p, 16); }

static bool ok_sched(const kvs_schedule *s) {
  return s && s->outer >= 0 && s->steps >= 0 && s->history >= 1 && s->history <= 15 &&
         s->max_bt >= 1 && s->max_bt <= 64 && s->backtrack > 0.f && s->backtrack < 1.f &&
         s->c1 > 0.f && s->c1 < 1.f && isfinite(s->lambda) && s->w_out >= 0.f && s->w_lse >= 0.f;
}

static Filter phase_filter(const State &s, int want) {
  return Filter{reinterpret_cast<const int *>(reinterpret_cast<const char *>(s.sc) +
                                              offsetof(LbfgsScal, phase)),
                (int)(sizeof(LbfgsScal) / sizeof(int)), want};
}

static const Filter ALL{nullptr, 0, 0};

// Problems whose last L-BFGS search failed: the loss forward left l_hat of a
// rejected trial in the workspace, so the ridge fit recomputes theirs.
static Filter stale_filter(const State &s) {
  return Filter{reinterpret_cast<const int *>(reinterpret_cast<const char *>(s.sc) +
                                              offsetof(LbfgsScal, lse_stale)),
                (int)(sizeof(LbfgsScal) / sizeof(int)), 1};
}

// Loss and gradient at Kc into (w.fbuf, s.gn), then the state reset.
static int lbfgs_restart(const Batch &Bt, const kvs_schedule &sc, const float *Q, const float *Y,
                         const float *lse, const float *Vc, const float *Kc, const State &s,
                         int clear, bool q_ready, const Work &w) {
  int rc = launch_forward(Bt, Q, Kc, Vc, Y, lse, sc.w_out, sc.w_lse, w.fbuf, nullptr, ALL, q_ready,
                          w);
  if (rc) return rc;
  rc = launch_backward(Bt, Vc, sc.w_out, s.gn, ALL, w);
  if (rc) return rc;
  return launch_lbfgs_reset(Bt, s, Kc, w.fbuf, s.gn, clear);
}

// One L-BFGS step in three parts: direction (and the bf16 split of the pairs),
// the Armijo trial loop, then dK_c at the accepted points and the history update.
// When the caller keeps the splits resident (inside kvs_compress_batch: the reset
// after each value fit split K_c and V_c, and every accepted trial leaves its own
// split), only the problems whose last search failed, and so left a rejected
// trial's split in the workspace, split K_c again; otherwise K_c and V_c are split.
static int step_head(const Batch &Bt, const kvs_schedule &sc, const float *Kc, const float *Vc,
                     const State &s, const Work &w, bool resident) {
  int rc = launch_lbfgs_direction(Bt, s, sc);
  if (rc) return rc;
  if (resident) return launch_split_pairs(Bt, Kc, nullptr, w, stale_filter(s));
  return launch_split_pairs(Bt, Kc, Vc, w);
}

static int step_trial(const Batch &Bt, const kvs_schedule &sc, const float *Q, const float *Y,
                      const float *lse, const float *Vc, float *Kc, const State &s,
                      bool q_ready, const Work &w, const cudaGraphConditionalHandle *cond) {
  int rc = launch_lbfgs_trial(Bt, s, Kc, w);
  if (rc) return rc;
  if ((rc = launch_forward(Bt, Q, Kc, Vc, Y, lse, sc.w_out, sc.w_lse, w.fbuf, nullptr,
                           phase_filter(s, PH_SEARCH), q_ready, w, true, false)))
    return rc;
  return launch_lbfgs_armijo(Bt, s, sc, w, cond);
}

static int step_tail(const Batch &Bt, const kvs_schedule &sc, const float *Vc, float *Kc,
                     const State &s, int32_t *status, float *f_out, const Work &w) {
  int rc = launch_backward(Bt, Vc, sc.w_out, s.gn, phase_filter(s, PH_ACCEPT), w);
  if (rc) return rc;
  return launch_lbfgs_update(Bt, s, Kc, status, f_out);
}

static int lbfgs_one_step(const Batch &Bt, const kvs_schedule &sc, const float *Q,
                          const float *Y, const float *lse, const float *Vc, float *Kc,
                          const State &s, int32_t *status, float *f_out, bool q_ready,
                          const Work &w) {
  int rc = step_head(Bt, sc, Kc, Vc, s, w, q_ready);
  if (rc) return rc;
  for (int t = 0; t < sc.max_bt; ++t)  // problems that have left the search skip each trial
    if ((rc = step_trial(Bt, sc, Q, Y, lse, Vc, Kc, s, q_ready || t > 0, w, nullptr))) return rc;
  return step_tail(Bt, sc, Vc, Kc, s, status, f_out, w);
}

// One L-BFGS step as a CUDA graph whose trial loop is a conditional WHILE node:
// trials run only while some problem is still searching (at most max_bt, since
// every trial either accepts, backtracks or, at max_bt, fails the search).
// The graph is recorded on two internal streams (the caller's stream may be the
// legacy default stream, which cannot be captured) and launched on the caller's.
struct StepGraph {
  uint64_t kernels = 0;  // kernel nodes captured (the trial loop body counted once)
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  cudaStream_t cap = nullptr, side = nullptr;
  ~StepGraph() {
    if (exec) cudaGraphExecDestroy(exec);
    if (graph) cudaGraphDestroy(graph);
    if (side) cudaStreamDestroy(side);
    if (cap) cudaStreamDestroy(cap);
  }
};

static int build_step_graph(const Batch &Bcaller, const kvs_schedule &sc, const float *Q,
                            const float *Y, const float *lse, const float *Vc, float *Kc,
                            const State &s, int32_t *status, const Work &w, StepGraph *sg) {
  KVS_CUDA_TRY(cudaStreamCreateWithFlags(&sg->side, cudaStreamNonBlocking));
  KVS_CUDA_TRY(cudaStreamCreateWithFlags(&sg->cap, cudaStreamNonBlocking));
  Batch Bt = Bcaller;
  Bt.st = sg->cap;
  const uint64_t n0 = g_launches.load(std::memory_order_relaxed);
  KVS_CUDA_TRY(cudaStreamBeginCapture(Bt.st, cudaStreamCaptureModeThreadLocal));
  int rc = step_head(Bt, sc, Kc, Vc, s, w, true);
  cudaStreamCaptureStatus cst;
  cudaGraph_t g = nullptr;
  const cudaGraphNode_t *deps = nullptr;
  size_t ndeps = 0;
  cudaGraphConditionalHandle cond{};
  cudaGraphNode_t cnode = nullptr;
  cudaGraphNodeParams cp = {};
  cudaError_t e = cudaSuccess;
  if (!rc) e = cudaStreamGetCaptureInfo(Bt.st, &cst, nullptr, &g, &deps, &ndeps);
  if (!rc && e == cudaSuccess) e = cudaGraphConditionalHandleCreate(&cond, g, 1, cudaGraphCondAssignDefault);
  if (!rc && e == cudaSuccess) {
    cp.type = cudaGraphNodeTypeConditional;
    cp.conditional.handle = cond;
    cp.conditional.type = cudaGraphCondTypeWhile;
    cp.conditional.size = 1;
    e = cudaGraphAddNode(&cnode, g, deps, ndeps, &cp);
  }
  if (!rc && e == cudaSuccess)
    e = cudaStreamUpdateCaptureDependencies(Bt.st, &cnode, 1, cudaStreamSetCaptureDependencies);
  if (!rc && e == cudaSuccess) {
    e = cudaStreamBeginCaptureToGraph(sg->side, cp.conditional.phGraph_out[0], nullptr, nullptr,
                                      0, cudaStreamCaptureModeThreadLocal);
    if (e == cudaSuccess) {
      Batch side = Bt;
      side.st = sg->side;
      rc = step_trial(side, sc, Q, Y, lse, Vc, Kc, s, true, w, &cond);
      cudaGraph_t body = nullptr;
      const cudaError_t e2 = cudaStreamEndCapture(sg->side, &body);
      if (e2 != cudaSuccess) e = e2;
    }
  }
  if (!rc && e == cudaSuccess) rc = step_tail(Bt, sc, Vc, Kc, s, status, nullptr, w);
  cudaGraph_t graph = nullptr;
  const cudaError_t e3 = cudaStreamEndCapture(Bt.st, &graph);
  sg->graph = graph;
  if (rc) return rc;
  if (e != cudaSuccess) {
    set_cuda_error(e, "building the L-BFGS step graph");
    (void)cudaGetLastError();
    return KVS_ECUDA;
  }
  KVS_CUDA_TRY(e3);
  KVS_CUDA_TRY(cudaGraphInstantiate(&sg->exec, sg->graph, 0));
  sg->kernels = g_launches.load(std::memory_order_relaxed) - n0;
  g_launches.fetch_sub(sg->kernels, std::memory_order_relaxed);  // captured, not yet run
  return KVS_OK;
}

// ------------------------------------------------------------ sub-batches
// kvs_compress_batch runs a large batch as independent sub-batches of
// contiguous problems, each on its own stream, so that the latency-bound parts
// of one (the Cholesky panels, the single-CTA L-BFGS control kernels) overlap
// the tensor-core work of the other.  Each sub-batch is a batch in its own
// right: offsets rebased to zero (on the device, in the caller's workspace),
// data pointers moved to its first rows, its own workspace and state carved
// from the caller's buffers, its own step graph and internal streams.

struct Partition {
  int n = 1;
  int cut[KVS_MAX_PARTS + 1] = {0};
};

// Sub-batches: four once the batch has at least 16 problems, two from 8 (each
// part still fills the GPU in the attention kernels), cut where the estimated
// work n_q k (d + k) of the problems reaches 1/n, 2/n, .. of the total.
static Partition partition_of(const kvs_batch *b, const HostGeom &g) {
  Partition P;
  P.cut[1] = g.B;
  if (g.B < 8 || !b->c_off_h) return P;
  const int n = g.B >= 16 ? 4 : 2;
  static_assert(KVS_MAX_PARTS >= 4, "parts");
  std::vector<double> acc(g.B + 1, 0.0);
  for (int i = 0; i < g.B; ++i) {
    const double nq = (double)(b->q_off_h[i + 1] - b->q_off_h[i]);
    const double k = (double)(b->c_off_h[i + 1] - b->c_off_h[i]);
    acc[i + 1] = acc[i] + nq * k * (g.d + k);
  }
  P.n = n;
  for (int p = 1; p < n; ++p) {
    // the cut nearest to the target that leaves at least one problem per part
    const double target = acc[g.B] * p / n;
    int best = P.cut[p - 1] + 1;
    for (int c = best; c <= g.B - (n - p); ++c)
      if (std::fabs(acc[c] - target) < std::fabs(acc[best] - target)) best = c;
    P.cut[p] = best;
  }
  P.cut[n] = g.B;
  return P;
}

// Placeholder for device offset pointers while sizing (never dereferenced).
static const int64_t *const kSizingOnly = reinterpret_cast<const int64_t *>(uintptr_t{256});

struct Part {
  int b0 = 0, b1 = 0;
  std::vector<int64_t> q_h, z_h, c_h;  // rebased host offsets
  kvs_batch kb{};
  HostGeom g;
  size_t ws_off = 0, st_off = 0;       // this part's pieces of the caller's buffers
};

// Host geometry of every part and where its workspace, state and rebased device
// offsets sit; returns false for an invalid batch.  *ws_need / *st_need: bytes.
static bool plan_parts(const kvs_batch *b, const HostGeom &g, int history, const Partition &P,
                       Part *parts, size_t *ws_need, size_t *st_need, size_t *off_at) {
  size_t ws = 0, st = 0;
  for (int p = 0; p < P.n; ++p) {
    Part &pt = parts[p];
    pt.b0 = P.cut[p];
    pt.b1 = P.cut[p + 1];
    const int n = pt.b1 - pt.b0;
    pt.q_h.resize(n + 1);
    pt.z_h.resize(n + 1);
    pt.c_h.resize(n + 1);
    for (int i = 0; i <= n; ++i) {
      pt.q_h[i] = b->q_off_h[pt.b0 + i] - b->q_off_h[pt.b0];
      pt.z_h[i] = b->z_off_h[pt.b0 + i] - b->z_off_h[pt.b0];
      pt.c_h[i] = b->c_off_h[pt.b0 + i] - b->c_off_h[pt.b0];
    }
    pt.kb = kvs_batch{n, b->d, kSizingOnly, kSizingOnly, kSizingOnly,
                      pt.q_h.data(), pt.z_h.data(), pt.c_h.data()};
    if (geom_from_batch(&pt.kb, &pt.g, true)) return false;
    Work w;
    State s;
    pt.ws_off = ws = (size_t)align_up((int64_t)ws, 256);
    ws += carve_work(pt.g, nullptr, &w);
    pt.st_off = st = (size_t)align_up((int64_t)st, 256);
    st += carve_state(pt.g, history, nullptr, &s);
  }
  *off_at = ws = (size_t)align_up((int64_t)ws, 256);
  ws += sizeof(int64_t) * 3 * (size_t)(g.B + P.n);  // rebased q, z, c offsets of every part
  *ws_need = (size_t)align_up((int64_t)ws, 256);
  *st_need = (size_t)align_up((int64_t)st, 256);
  return true;
}

// dst receives, part after part, the rebased offsets q, z and c of each part
// (3 arrays of n_p + 1 entries).
__global__ void k_rebase(const int64_t *q_off, const int64_t *z_off, const int64_t *c_off,
                         Partition P, int64_t *dst) {
  int64_t *o = dst;
  for (int p = 0; p < P.n; ++p) {
    const int b0 = P.cut[p], n = P.cut[p + 1] - b0;
    for (int i = threadIdx.x; i <= n; i += blockDim.x) {
      o[i] = q_off[b0 + i] - q_off[b0];
      o[n + 1 + i] = z_off[b0 + i] - z_off[b0];
      o[2 * (n + 1) + i] = c_off[b0 + i] - c_off[b0];
    }
    o += 3 * (n + 1);
  }
}

// The stream of sub-batch `slot` >= 1 and the events that fork it from and join it
// to the caller's stream (per host thread and device, created on first use).
struct PartStreams {
  cudaStream_t st[KVS_MAX_PARTS] = {nullptr};
  cudaEvent_t fork = nullptr, join[KVS_MAX_PARTS] = {nullptr};
};

static cudaError_t part_streams(PartStreams **out) {
  constexpr int kMaxDev = 64;
  static thread_local PartStreams ps[kMaxDev];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  PartStreams &p = ps[dev];
  if (!p.fork) {
    if ((e = cudaEventCreateWithFlags(&p.fork, cudaEventDisableTiming)) != cudaSuccess) return e;
    for (int i = 1; i < KVS_MAX_PARTS; ++i)
      if ((e = cudaStreamCreateWithFlags(&p.st[i], cudaStreamNonBlocking)) != cudaSuccess ||
          (e = cudaEventCreateWithFlags(&p.join[i], cudaEventDisableTiming)) != cudaSuccess)
        return e;
  }
  *out = &p;
  return cudaSuccess;
}

// One sub-batch's solve: its batch view, buffers and step graph.
struct Solve {
  Batch Bt;
  Work w;
  State s;
  const float *Q, *Kz, *Vz;
  float *Kc, *Vc, *trace, *parts;
  int32_t *idx, *status;
  StepGraph sg;
  bool have_graph = false;
};

}  // namespace kvs

using namespace kvs;

extern "C" {

const char *kvs_version(void) { return "kvsculpt-b200 0.1 (sm_100a)"; }

const char *kvs_last_cuda_error(void) { return g_err; }

uint64_t kvs_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int kvs_set_wait_limit(int64_t cycles) {
  if (cycles < 0) return KVS_EINVAL;
  g_wait_limit.store((long long)cycles, std::memory_order_relaxed);
  return KVS_OK;
}

size_t kvs_workspace_bytes(const kvs_batch *batch, const kvs_schedule *) {
  HostGeom g;
  if (geom_from_batch(batch, &g, false)) return 0;
  Work w;
  size_t need = carve_work(g, nullptr, &w);
  const Partition P = partition_of(batch, g);
  if (P.n > 1) {  // the sub-batches of kvs_compress_batch
    Part parts[KVS_MAX_PARTS];
    size_t ws = 0, st = 0, off = 0;
    if (!plan_parts(batch, g, 1, P, parts, &ws, &st, &off)) return 0;
    need = std::max(need, ws);
  }
  return need;
}

size_t kvs_lbfgs_state_bytes(const kvs_batch *batch, int32_t history) {
  HostGeom g;
  if (history < 1 || history > 15 || geom_from_batch(batch, &g, true)) return 0;
  State s;
  size_t need = carve_state(g, history, nullptr, &s);
  const Partition P = partition_of(batch, g);
  if (P.n > 1) {
    Part parts[KVS_MAX_PARTS];
    size_t ws = 0, st = 0, off = 0;
    if (!plan_parts(batch, g, history, P, parts, &ws, &st, &off)) return 0;
    need = std::max(need, st);
  }
  return need;
}

int kvs_lbfgs_state_layout(const kvs_batch *batch, int32_t history, kvs_lbfgs_layout *out) {
  HostGeom g;
  if (!out || history < 1 || history > 15 || geom_from_batch(batch, &g, true)) return KVS_EINVAL;
  State s;
  carve_state(g, history, reinterpret_cast<void *>(uintptr_t{1} << 40), &s);
  const char *base = reinterpret_cast<const char *>(uintptr_t{1} << 40);
  auto at = [&](const void *p) { return (uint64_t)(static_cast<const char *>(p) - base); };
  *out = kvs_lbfgs_layout{};
  out->scalars = at(s.sc);
  out->scalar_bytes = sizeof(LbfgsScal);
  out->off_f = offsetof(LbfgsScal, f);
  out->off_count = offsetof(LbfgsScal, count);
  out->off_head = offsetof(LbfgsScal, head);
  out->x = at(s.x);
  out->g = at(s.g);
  out->dir = at(s.dir);
  out->ring_s = at(s.ring_s);
  out->ring_y = at(s.ring_y);
  out->ring_stride = (uint64_t)(g.sum_c * g.d) * sizeof(float);
  out->slots = history + 1;
  return KVS_OK;
}

int kvs_build_queries(const kvs_query_spec *sp, const float *q_retain, const float *q_ctx,
                      const int32_t *pos, float *Q, void *stream) {
  if (!sp || sp->B < 1 || sp->g < 1 || sp->m_q < 0 || sp->n_syn < 0 || sp->N < 1 ||
      !(sp->rope_base > 1.f))
    return KVS_EINVAL;
  if (sp->d != 64 && sp->d != 128) return KVS_ENOTSUP;
  if (!ok_ptr(Q) || (sp->m_q > 0 && !ok_ptr(q_retain)) ||
      (sp->n_syn > 0 && (!ok_ptr(q_ctx) || !ok_ptr(pos))))
    return KVS_EINVAL;
  return launch_build_queries(sp, q_retain, q_ctx, pos, Q, static_cast<cudaStream_t>(stream));
}

int kvs_targets(const kvs_batch *batch, const float *Q, const float *Kz, const float *Vz,
                float *Y, float *lse, float *importance, void *ws, size_t ws_bytes,
                void *stream) {
  Batch Bt;
  Work w;
  int rc = prep(batch, false, ws, ws_bytes, stream, &Bt, &w);
  if (rc) return rc;
  if (!ok_ptr(Q) || !ok_ptr(Kz) || !ok_ptr(Vz) || !ok_ptr(Y) || !ok_ptr(lse) ||
      (importance && !ok_ptr(importance)))
    return KVS_EINVAL;
  if ((rc = begin(Bt, w))) return rc;
  if ((rc = launch_targets(Bt, Q, Kz, Vz, Y, lse, importance, w))) return rc;
  const HostGeom &g = Bt.g;
  return nan_if_err(Bt, w, Y, g.sum_q * g.d, lse, g.sum_q, importance, g.sum_z);
}

int kvs_init_topk(const kvs_batch *batch, const float *importance, const float *Kz,
                  int32_t *idx, float *Kc, void *stream) {
  HostGeom g;
  int rc = geom_from_batch(batch, &g, true);
  if (rc) return rc;
  if (!ok_ptr(importance) || !ok_ptr(Kz) || !ok_ptr(idx) || !ok_ptr(Kc)) return KVS_EINVAL;
  if (g.max_z > 16384) return KVS_ENOTSUP;
  for (int b = 0; b < g.B; ++b)
    if (batch->c_off_h[b + 1] - batch->c_off_h[b] > batch->z_off_h[b + 1] - batch->z_off_h[b])
      return KVS_EINVAL;
  Batch Bt{g, batch, static_cast<cudaStream_t>(stream)};
  return launch_topk(Bt, importance, Kz, idx, Kc);
}

int kvs_loss_grad(const kvs_batch *batch, const float *Q, const float *Kc, const float *Vc,
                  const float *Y, const float *lse, float w_out, float w_lse, float *loss,
                  float *parts, float *dKc, void *ws, size_t ws_bytes, void *stream) {
  Batch Bt;
  Work w;
  int rc = prep(batch, true, ws, ws_bytes, stream, &Bt, &w);
  if (rc) return rc;
  if (!ok_ptr(Q) || !ok_ptr(Kc) || !ok_ptr(Vc) || !ok_ptr(Y) || !ok_ptr(lse) || !ok_ptr(loss) ||
      (parts && !ok_ptr(parts)) || (dKc && !ok_ptr(dKc)))
    return KVS_EINVAL;
  if ((rc = begin(Bt, w))) return rc;
  if ((rc = launch_forward(Bt, Q, Kc, Vc, Y, lse, w_out, w_lse, loss, parts, ALL, false, w)))
    return rc;
  if (dKc && (rc = launch_backward(Bt, Vc, w_out, dKc, ALL, w))) return rc;
  const HostGeom &g = Bt.g;
  return nan_if_err(Bt, w, loss, g.B, parts, 2 * (int64_t)g.B, dKc, g.sum_c * g.d);
}

int kvs_fit_values(const kvs_batch *batch, const float *Q, const float *Kc, const float *Y,
                   float lambda, float *Vc, int32_t *status, void *ws, size_t ws_bytes,
                   void *stream) {
  Batch Bt;
  Work w;
  int rc = prep(batch, true, ws, ws_bytes, stream, &Bt, &w);
  if (rc) return rc;
  if (!ok_ptr(Q) || !ok_ptr(Kc) || !ok_ptr(Y) || !ok_ptr(Vc) || !ok_ptr(status) ||
      !isfinite(lambda))
    return KVS_EINVAL;
  if ((rc = begin(Bt, w))) return rc;
  if ((rc = launch_fit(Bt, Q, Kc, Y, lambda, Vc, status, false, false, w))) return rc;
  return fold_err(Bt, w, status);
}

static int prep_state(const Batch &Bt, const kvs_schedule *sched, void *state,
                      size_t state_bytes, State *s) {
  if (!ok_sched(sched) || !state || !aligned(state, 256)) return KVS_EINVAL;
  if (carve_state(Bt.g, sched->history, nullptr, s) > state_bytes) return KVS_EWORKSPACE;
  carve_state(Bt.g, sched->history, state, s);
  return KVS_OK;
}

int kvs_lbfgs_reset(const kvs_batch *batch, const kvs_schedule *sched, const float *Q,
                    const float *Y, const float *lse, const float *Vc, const float *Kc,
                    void *state, size_t state_bytes, int32_t clear_history, void *ws,
                    size_t ws_bytes, void *stream) {
  Batch Bt;
  Work w;
  State s;
  int rc = prep(batch, true, ws, ws_bytes, stream, &Bt, &w);
  if (rc) return rc;
  if ((rc = prep_state(Bt, sched, state, state_bytes, &s))) return rc;
  if (!ok_ptr(Q) || !ok_ptr(Y) || !ok_ptr(lse) || !ok_ptr(Vc) || !ok_ptr(Kc)) return KVS_EINVAL;
  if ((rc = begin(Bt, w))) return rc;
  return lbfgs_restart(Bt, *sched, Q, Y, lse, Vc, Kc, s, clear_history != 0, false, w);
}

int kvs_lbfgs_step(const kvs_batch *batch, const kvs_schedule *sched, const float *Q,
                   const float *Y, const float *lse, const float *Vc, float *Kc, void *state,
                   size_t state_bytes, int32_t *status, float *f_out, void *ws, size_t ws_bytes,
                   void *stream) {
  Batch Bt;
  Work w;
  State s;
  int rc = prep(batch, true, ws, ws_bytes, stream, &Bt, &w);
  if (rc) return rc;
  if ((rc = prep_state(Bt, sched, state, state_bytes, &s))) return rc;
  if (!ok_ptr(Q) || !ok_ptr(Y) || !ok_ptr(lse) || !ok_ptr(Vc) || !ok_ptr(Kc) ||
      (status && !ok_ptr(status)) || (f_out && !ok_ptr(f_out)))
    return KVS_EINVAL;
  if ((rc = begin(Bt, w))) return rc;
  if ((rc = lbfgs_one_step(Bt, *sched, Q, Y, lse, Vc, Kc, s, status, f_out, false, w))) return rc;
  return fold_err(Bt, w, status);
}

int kvs_adam_step(const kvs_batch *batch, float *Kc, const float *dKc, float *m, float *v,
                  int32_t t, float lr, float beta1, float beta2, float eps, void *stream) {
  HostGeom g;
  int rc = geom_from_batch(batch, &g, true);
  if (rc) return rc;
  if (!ok_ptr(Kc) || !ok_ptr(dKc) || !ok_ptr(m) || !ok_ptr(v)) return KVS_EINVAL;
  if (t < 1 || !(lr > 0.f) || !isfinite(lr) || !(beta1 >= 0.f && beta1 < 1.f) ||
      !(beta2 >= 0.f && beta2 < 1.f) || !(eps > 0.f) || !isfinite(eps))
    return KVS_EINVAL;
  const double bc1 = 1.0 - pow((double)beta1, (double)t);
  const double bc2 = 1.0 - pow((double)beta2, (double)t);
  return launch_adam(Kc, dKc, m, v, g.sum_c * g.d, lr, beta1, beta2, eps, (float)bc1, (float)bc2,
                     static_cast<cudaStream_t>(stream));
}

int kvs_compress_batch(const kvs_batch *batch, const kvs_schedule *sched, const float *Q,
                       const float *Kz, const float *Vz, float *Kc, float *Vc, int32_t *idx,
                       float *loss_trace, float *parts, int32_t *status, void *state,
                       size_t state_bytes, void *ws, size_t ws_bytes, void *stream) {
  Batch Bt;
  Work w;
  State s;
  int rc = prep(batch, true, ws, ws_bytes, stream, &Bt, &w);
  if (rc) return rc;
  if ((rc = prep_state(Bt, sched, state, state_bytes, &s))) return rc;
  if (!ok_ptr(Q) || !ok_ptr(Kz) || !ok_ptr(Vz) || !ok_ptr(Kc) || !ok_ptr(Vc) ||
      !ok_ptr(status) || (idx && !ok_ptr(idx)) || (loss_trace && !ok_ptr(loss_trace)) ||
      (parts && !ok_ptr(parts)))
    return KVS_EINVAL;
  if (Bt.g.max_z > 16384) return KVS_ENOTSUP;
  for (int b = 0; b < Bt.g.B; ++b)
    if (batch->c_off_h[b + 1] - batch->c_off_h[b] > batch->z_off_h[b + 1] - batch->z_off_h[b])
      return KVS_EINVAL;
  const kvs_schedule &sc = *sched;
  const int64_t tstride = sc.outer + 1;
  const int d = Bt.g.d;

  // the sub-batches: one (the whole batch, as given) or several
  const Partition P = partition_of(batch, Bt.g);
  Part pt[KVS_MAX_PARTS];
  Solve sv[KVS_MAX_PARTS];
  PartStreams *ps = nullptr;
  if (P.n == 1) {
    sv[0].Bt = Bt;
    sv[0].w = w;
    sv[0].s = s;
  } else {
    size_t ws_need = 0, st_need = 0, off_at = 0;
    if (!plan_parts(batch, Bt.g, sc.history, P, pt, &ws_need, &st_need, &off_at))
      return KVS_EINVAL;
    if (ws_need > ws_bytes || st_need > state_bytes) return KVS_EWORKSPACE;
    KVS_CUDA_TRY(part_streams(&ps));
    int64_t *dev_off = reinterpret_cast<int64_t *>(static_cast<char *>(ws) + off_at);
    k_rebase<<<1, 256, 0, Bt.st>>>(batch->q_off, batch->z_off, batch->c_off, P, dev_off);
    KVS_LAUNCH_CHECK("k_rebase");
    KVS_CUDA_TRY(cudaEventRecord(ps->fork, Bt.st));
    for (int p = 0; p < P.n; ++p) {
      const int n = pt[p].b1 - pt[p].b0;
      pt[p].kb.q_off = dev_off;
      pt[p].kb.z_off = dev_off + (n + 1);
      pt[p].kb.c_off = dev_off + 2 * (n + 1);
      dev_off += 3 * (n + 1);
      Solve &v = sv[p];
      v.Bt.g = pt[p].g;
      v.Bt.b = &pt[p].kb;
      v.Bt.slot = p;
      v.Bt.share = P.n;
      v.Bt.st = p == 0 ? Bt.st : ps->st[p];
      if (p > 0) KVS_CUDA_TRY(cudaStreamWaitEvent(v.Bt.st, ps->fork, 0));
      carve_work(v.Bt.g, static_cast<char *>(ws) + pt[p].ws_off, &v.w);
      carve_state(v.Bt.g, sc.history, static_cast<char *>(state) + pt[p].st_off, &v.s);
    }
  }
  for (int p = 0; p < P.n; ++p) {
    Solve &v = sv[p];
    const int b0 = P.cut[p];
    const int64_t q0 = batch->q_off_h[b0], z0 = batch->z_off_h[b0], c0 = batch->c_off_h[b0];
    v.Q = Q + q0 * d;
    v.Kz = Kz + z0 * d;
    v.Vz = Vz + z0 * d;
    v.Kc = Kc + c0 * d;
    v.Vc = Vc + c0 * d;
    v.idx = idx ? idx + c0 : v.w.idx;
    v.status = status + b0;
    v.trace = loss_trace ? loss_trace + b0 * tstride : nullptr;
    v.parts = parts ? parts + 2 * b0 : nullptr;
  }

  // initial state of every sub-batch: targets, top-k keys, Select+Fit, L-BFGS reset
  for (int p = 0; p < P.n; ++p) {
    Solve &v = sv[p];
    const Batch &B = v.Bt;
    if ((rc = begin(B, v.w))) return rc;
    KVS_CUDA_TRY(cudaMemsetAsync(v.status, 0, sizeof(int32_t) * B.g.B, B.st));
    if ((rc = launch_targets(B, v.Q, v.Kz, v.Vz, v.w.Yt, v.w.lset, v.w.imp, v.w))) return rc;
    if ((rc = launch_topk(B, v.w.imp, v.Kz, v.idx, v.Kc))) return rc;
    // from here on the bf16 splits of Q and of the targets Y stay in the workspace
    if ((rc = launch_fit(B, v.Q, v.Kc, v.w.Yt, sc.lambda, v.Vc, v.status, true, true, v.w)))
      return rc;
    if ((rc = lbfgs_restart(B, sc, v.Q, v.w.Yt, v.w.lset, v.Vc, v.Kc, v.s, 1, true, v.w)))
      return rc;
    if (v.trace && (rc = launch_copy_f(B, v.s, v.trace, tstride, 0))) return rc;
  }
  // KVS_STEP_GRAPHS=0 launches every kernel of a step individually (the same
  // arithmetic; kernel profilers do not look inside graphs with conditional nodes)
  static const bool use_graphs = [] {
    const char *e = getenv("KVS_STEP_GRAPHS");
    return !(e && e[0] == '0');
  }();
  for (int o = 0; o < sc.outer; ++o) {
    for (int t = 0; t < sc.steps; ++t) {
      for (int p = 0; p < P.n; ++p) {
        Solve &v = sv[p];
        if (use_graphs && !v.have_graph && o + t > 0) {
          // every kernel has been launched once outside capture: record the step now
          if ((rc = build_step_graph(v.Bt, sc, v.Q, v.w.Yt, v.w.lset, v.Vc, v.Kc, v.s,
                                     v.status, v.w, &v.sg)))
            return rc;
          v.have_graph = true;
        }
        if (v.have_graph) {
          KVS_CUDA_TRY(cudaGraphLaunch(v.sg.exec, v.Bt.st));
          g_launches.fetch_add(v.sg.kernels, std::memory_order_relaxed);
        } else if ((rc = lbfgs_one_step(v.Bt, sc, v.Q, v.w.Yt, v.w.lset, v.Vc, v.Kc, v.s,
                                        v.status, nullptr, true, v.w))) {
          return rc;
        }
      }
    }
    for (int p = 0; p < P.n; ++p) {
      Solve &v = sv[p];
      // every problem's l_hat at Kc is in the workspace from its accepted trial's
      // loss forward, except after a failed search
      if ((rc = launch_fit(v.Bt, v.Q, v.Kc, v.w.Yt, sc.lambda, v.Vc, v.status, true, true, v.w,
                           sc.steps > 0 ? stale_filter(v.s) : ALL)))
        return rc;
      if ((rc = lbfgs_restart(v.Bt, sc, v.Q, v.w.Yt, v.w.lset, v.Vc, v.Kc, v.s,
                              sc.persist_history ? 0 : 1, true, v.w)))
        return rc;
      if (v.trace && (rc = launch_copy_f(v.Bt, v.s, v.trace, tstride, o + 1))) return rc;
    }
  }
  for (int p = 0; p < P.n; ++p) {
    Solve &v = sv[p];
    if (v.parts && (rc = launch_forward(v.Bt, v.Q, v.Kc, v.Vc, v.w.Yt, v.w.lset, sc.w_out,
                                        sc.w_lse, v.w.fbuf, v.parts, ALL, true, v.w)))
      return rc;
    if ((rc = fold_err(v.Bt, v.w, v.status))) return rc;
    if (p > 0) {
      KVS_CUDA_TRY(cudaEventRecord(ps->join[p], v.Bt.st));
      KVS_CUDA_TRY(cudaStreamWaitEvent(Bt.st, ps->join[p], 0));
    }
  }
  return KVS_OK;
}

// Host-only budget allocation.  The real shares x_b(c) = clip(c w_b, k_min,
// k_max_b) are non-decreasing in c; c is found by bisection to the resolution
// of double precision, then the integers are floors plus largest remainders.
int kvs_pilot_allocate(int32_t B, const float *pilot_mse, int64_t total, int32_t k_min,
                       const int32_t *k_max, float alpha, int32_t *k_out) {
  if (B < 1 || !pilot_mse || !k_max || !k_out || k_min < 1 || !(alpha >= 0.f)) return KVS_EINVAL;
  int64_t lo_sum = 0, hi_sum = 0;
  for (int b = 0; b < B; ++b) {
    if (k_max[b] < k_min) return KVS_EINVAL;
    lo_sum += k_min;
    hi_sum += k_max[b];
  }
  if (total < lo_sum || total > hi_sum) return KVS_EINVAL;
  std::vector<double> w(B), x(B);
  double wsum = 0.0;
  for (int b = 0; b < B; ++b) {
    const double m = pilot_mse[b];
    w[b] = (isfinite(m) && m > 0.0) ? pow(m, (double)alpha) : 0.0;
    wsum += w[b];
  }
  if (!(wsum > 0.0)) std::fill(w.begin(), w.end(), 1.0);
  // When the problems with a positive signal cannot absorb the budget even at
  // k_max, they take k_max and the zero-signal problems share the rest evenly.
  int64_t cap_pos = 0, floor_zero = 0;
  for (int b = 0; b < B; ++b) {
    if (w[b] > 0.0) cap_pos += k_max[b];
    else floor_zero += k_min;
  }
  std::vector<double> lo(B, (double)k_min), hi(B);
  for (int b = 0; b < B; ++b) hi[b] = k_max[b];
  if (cap_pos + floor_zero < total) {
    for (int b = 0; b < B; ++b) {
      if (w[b] > 0.0) lo[b] = hi[b];   // pinned at k_max
      else w[b] = 1.0;
    }
  }
  auto shares = [&](double c) {
    double s = 0.0;
    for (int b = 0; b < B; ++b) {
      x[b] = std::min(hi[b], std::max(lo[b], c * w[b]));
      s += x[b];
    }
    return s;
  };
  double clo = 0.0, chi = 1.0;
  while (shares(chi) < (double)total && chi < 1e300) chi *= 2.0;
  for (int it = 0; it < 2000; ++it) {
    const double mid = 0.5 * (clo + chi);
    if (mid <= clo || mid >= chi) break;
    if (shares(mid) < (double)total) clo = mid;
    else chi = mid;
  }
  // Between clo and chi the total is crossed; interpolate on the linear piece.
  const double slo = shares(clo);
  std::vector<double> xlo(x);
  const double shi = shares(chi);
  std::vector<double> ideal(B);
  const double f = (shi > slo) ? ((double)total - slo) / (shi - slo) : 1.0;
  for (int b = 0; b < B; ++b) ideal[b] = xlo[b] + f * (x[b] - xlo[b]);
  std::vector<int64_t> k(B);
  std::vector<double> frac(B);
  int64_t sum = 0;
  for (int b = 0; b < B; ++b) {
    k[b] = (int64_t)floor(ideal[b]);
    k[b] = std::min<int64_t>(std::max<int64_t>(k[b], k_min), k_max[b]);
    frac[b] = ideal[b] - (double)k[b];
    sum += k[b];
  }
  std::vector<int> order(B);
  for (int b = 0; b < B; ++b) order[b] = b;
  std::stable_sort(order.begin(), order.end(), [&](int a, int c) { return frac[a] > frac[c]; });
  int64_t left = total - sum;
  for (int i = 0; left > 0 && i < B; ++i) {
    const int b = order[i];
    if (k[b] < k_max[b]) {
      ++k[b];
      --left;
    }
  }
  if (left != 0) return KVS_EINVAL;
  for (int b = 0; b < B; ++b) k_out[b] = (int32_t)k[b];
  return KVS_OK;
}

}  // extern "C"
