// Device-resident batched L-BFGS on the compressed keys.
//
// "KVSculpt: KV Cache Compression as Distillation", section 2 "Key
// Optimization": keys are optimised by L-BFGS (a quasi-Newton method).  The
// pages name the method only; the constants (history h, H0 = gamma I from
// the newest pair, curvature test s.y > 1e-10 y.y, Armijo backtracking with a
// deterministic halving schedule, first trial min(1, 1/|g|) on an empty
// history) are the reading stated in the library header.
//
// Every problem owns a segment of n_b = k_b * d floats in each vector, cut
// into chunks of LBFGS_CHUNK elements, one CTA per chunk over the whole GPU.
// The two-loop recursion d = -H g is evaluated in its inner-product form: with
// the scalars s_i . g, y_i . g, s_i . y_j (s older than y) and y_i . y_j, every
// alpha_i and beta_i of the two loops follows from a few hundred scalar
// operations, and d is one linear combination of g and the stored pairs.
// The arithmetic is the same recursion reassociated; each vector is read once
// per pass instead of once per pair and loop.
//   k_pairs (update)  stores the accepted pair, moves x and g, and reads the
//                     history once for y_new . s_j, y_new . y_j (new Gram row)
//                     and g . s_j, g . y_j (next direction)
//   k_pairs (reset)   restarts at the current keys; the same inner products
//   the last CTA of a problem sums the per-CTA partials in a fixed order (in
//   double) and runs the scalar recursion; k_direction forms d.
// A run is bit-reproducible.
#include <math.h>

#include "kvs_internal.cuh"

namespace kvs {
namespace {

constexpr int CH = LBFGS_CHUNK;
constexpr int PT = 256;             // threads of the chunked passes
constexpr int V4 = CH / 4 / PT;     // float4 per thread and vector
constexpr int NW = PT / 32;
constexpr int NDOT = LBFGS_NDOT;    // 5 + 4 per stored pair
constexpr int MODE_RESET = 0, MODE_UPDATE = 1;
static_assert(CH % (4 * PT) == 0 && NDOT >= 5 + 4 * 15, "chunk layout");

__device__ __forceinline__ int64_t seg0(const int64_t *c_off, int b, int d) {
  return c_off[b] * (int64_t)d;
}
__device__ __forceinline__ int ring_slot(int head, int p, int slots) {
  return (head - 1 - p + 2 * slots) % slots;  // p = 0 newest
}
__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ void st4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
__device__ __forceinline__ float4 sub4(float4 a, float4 b) {
  return make_float4(a.x - b.x, a.y - b.y, a.z - b.z, a.w - b.w);
}
__device__ __forceinline__ float dot4(float4 a, float4 b, float acc) {
  acc = fmaf(a.x, b.x, acc);
  acc = fmaf(a.y, b.y, acc);
  acc = fmaf(a.z, b.z, acc);
  return fmaf(a.w, b.w, acc);
}

struct PairArgs {
  LbfgsScal *sc;
  LbfgsGram *gram;
  DirCoef *dc;
  float *part;
  int *ticket;
  float *x, *g;
  const float *gsrc;  // update: gradient at the accepted point; reset: gradient at Kc
  float *Kc;
  const float *f;     // reset: loss at Kc
  float *ring_s, *ring_y;
  int64_t rstride;
  int h, d, cmax, clear;
  const int64_t *c_off;
  int32_t *status;
  float *f_out;
};

// Scalar part of the recursion for the cnt newest pairs: slots sl[], s_p . g,
// y_p . g, |g|^2 and the Gram store give alpha_p, beta_p and the combination.
__device__ void direction_coefs(const LbfgsGram &G, int cnt, const int *sl, const double *sg,
                                const double *yg, double gg, DirCoef &c) {
  double al[16], be[16];
  const double gamma = cnt > 0 ? G.sy[sl[0]][sl[0]] / G.yy[sl[0]][sl[0]] : 1.0;
  // loop 1, newest first: alpha_p = rho_p s_p . (g - sum_{q newer} alpha_q y_q)
  for (int p = 0; p < cnt; ++p) {
    double v = sg[p];
    for (int q = 0; q < p; ++q) v -= al[q] * G.sy[sl[p]][sl[q]];
    al[p] = v / G.sy[sl[p]][sl[p]];
  }
  // loop 2, oldest first: beta_p = rho_p y_p . r, with
  // r = gamma (g - sum_q alpha_q y_q) + sum_{q older} (alpha_q - beta_q) s_q
  for (int p = cnt - 1; p >= 0; --p) {
    double v = yg[p];
    for (int q = 0; q < cnt; ++q) v -= al[q] * G.yy[sl[p]][sl[q]];
    v *= gamma;
    for (int q = p + 1; q < cnt; ++q) v += (al[q] - be[q]) * G.sy[sl[q]][sl[p]];
    be[p] = v / G.sy[sl[p]][sl[p]];
  }
  // d = -r = -gamma g + sum_q (gamma alpha_q y_q + (beta_q - alpha_q) s_q)
  double gd = -gamma * gg;
  for (int p = 0; p < cnt; ++p) {
    c.cy[p] = (float)(gamma * al[p]);
    c.cs[p] = (float)(be[p] - al[p]);
    gd += gamma * al[p] * yg[p] + (be[p] - al[p]) * sg[p];
  }
  c.cg = (float)-gamma;
  c.cnt = cnt;
  if (!(gd < 0.0)) {  // not a descent direction: steepest descent
    c.cg = -1.f;
    c.cnt = 0;
    gd = -gg;
  }
  c.gtd = (float)gd;
  const double gn = sqrt(gg);
  c.t0 = cnt > 0 ? 1.f : (gn > 0.0 ? (float)fmin(1.0, 1.0 / gn) : 1.f);
}

// Reset: x = Kc, g = gradient at Kc, f; clear the history on request.
// Update: accepted problems store (s, y) = (Kc - x, g_new - g) in the scratch
// slot, keep it when s.y > 1e-10 y.y, move x, g, f; failed problems restore
// Kc = x, clear the history and flag LS_FAIL.
// Both then prepare the next direction's coefficients.
template <int MODE>
__global__ void __launch_bounds__(PT) k_pairs(PairArgs a) {
  __shared__ float wsum[NW][NDOT];
  __shared__ double tot[NDOT];
  __shared__ int last;
  const int b = blockIdx.y, cb = blockIdx.x;
  const int64_t o = a.c_off[b] * (int64_t)a.d, n = a.c_off[b + 1] * (int64_t)a.d - o;
  const int nch = (int)((n + CH - 1) / CH);
  if (cb >= nch) return;
  LbfgsScal &s = a.sc[b];
  const int slots = a.h + 1;
  const int count0 = min(max(s.count, 0), a.h), head0 = min(max(s.head, 0), a.h);
  const int phase = MODE == MODE_UPDATE ? s.phase : PH_IDLE;
  const bool newpair = MODE == MODE_UPDATE && phase == PH_ACCEPT;
  const int nvalid = (MODE == MODE_UPDATE ? phase == PH_FAIL : a.clear) ? 0 : count0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t base = o + (int64_t)cb * CH;
  const int lim = (int)(n - (int64_t)cb * CH < CH ? n - (int64_t)cb * CH : CH);  // multiple of 4
  const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 gv[V4], sv[V4], yv[V4];
  float acc[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int u = 0; u < V4; ++u) {
    const int e = (u * PT + threadIdx.x) * 4;
    gv[u] = sv[u] = yv[u] = z4;
    if (e >= lim) continue;
    const int64_t i = base + e;
    if (MODE == MODE_RESET) {
      st4(a.x + i, ld4(a.Kc + i));
      gv[u] = ld4(a.gsrc + i);
      st4(a.g + i, gv[u]);
    } else if (newpair) {
      const float4 xn = ld4(a.Kc + i), gn = ld4(a.gsrc + i);
      sv[u] = sub4(xn, ld4(a.x + i));
      yv[u] = sub4(gn, ld4(a.g + i));
      gv[u] = gn;
      st4(a.ring_s + head0 * a.rstride + i, sv[u]);
      st4(a.ring_y + head0 * a.rstride + i, yv[u]);
      st4(a.x + i, xn);
      st4(a.g + i, gn);
    } else {
      if (phase == PH_FAIL) st4(a.Kc + i, ld4(a.x + i));
      gv[u] = ld4(a.g + i);
    }
    acc[0] = dot4(sv[u], yv[u], acc[0]);
    acc[1] = dot4(yv[u], yv[u], acc[1]);
    acc[2] = dot4(gv[u], sv[u], acc[2]);
    acc[3] = dot4(gv[u], yv[u], acc[3]);
    acc[4] = dot4(gv[u], gv[u], acc[4]);
  }
#pragma unroll
  for (int k = 0; k < 5; ++k) {
    const float v = warp_sum(acc[k]);
    if (lane == 0) wsum[warp][k] = v;
  }
  // one read of each stored pair: y_new . s_j, y_new . y_j, g . s_j, g . y_j; the
  // next pair's loads are issued before this pair's warp sums
  float4 sj[V4], yj[V4];
  auto fetch = [&](int p, float4 *sd, float4 *yd) {
    const int sl = ring_slot(head0, p, slots);
    const float *rs = a.ring_s + sl * a.rstride, *ry = a.ring_y + sl * a.rstride;
#pragma unroll
    for (int u = 0; u < V4; ++u) {
      const int e = (u * PT + threadIdx.x) * 4;
      sd[u] = yd[u] = z4;
      if (e < lim) {
        sd[u] = ld4(rs + base + e);
        yd[u] = ld4(ry + base + e);
      }
    }
  };
  if (nvalid > 0) fetch(0, sj, yj);
  for (int p = 0; p < nvalid; ++p) {
    float4 sn[V4], yn[V4];
    if (p + 1 < nvalid) fetch(p + 1, sn, yn);
    float c4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < V4; ++u) {
      c4[0] = dot4(yv[u], sj[u], c4[0]);
      c4[1] = dot4(yv[u], yj[u], c4[1]);
      c4[2] = dot4(gv[u], sj[u], c4[2]);
      c4[3] = dot4(gv[u], yj[u], c4[3]);
    }
#pragma unroll
    for (int u = 0; u < V4; ++u) {
      sj[u] = sn[u];
      yj[u] = yn[u];
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float v = warp_sum(c4[k]);
      if (lane == 0) wsum[warp][5 + 4 * p + k] = v;
    }
  }
  __syncthreads();
  const int nd = 5 + 4 * nvalid;
  float *pp = a.part + ((int64_t)b * a.cmax + cb) * NDOT;
  for (int k = threadIdx.x; k < nd; k += PT) {
    float v = 0.f;
    for (int w = 0; w < NW; ++w) v += wsum[w][k];
    pp[k] = v;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(&a.ticket[b], 1) == nch - 1;
  __syncthreads();
  if (!last) return;
  // the last CTA of the problem: fixed-order sums, then the scalar work
  __threadfence();
  for (int k = threadIdx.x; k < nd; k += PT) {
    double v = 0.0;
    for (int c = 0; c < nch; ++c) v += (double)__ldcg(a.part + ((int64_t)b * a.cmax + c) * NDOT + k);
    tot[k] = v;
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  a.ticket[b] = 0;
  LbfgsGram &G = a.gram[b];
  int count = count0, head = head0;
  bool kept = false;
  if (MODE == MODE_UPDATE) {
    if (phase == PH_ACCEPT) {
      const double sy = tot[0], yy = tot[1];
      if (sy > 1e-10 * yy) {
        kept = true;
        G.sy[head0][head0] = sy;
        G.yy[head0][head0] = yy;
        for (int p = 0; p < count0; ++p) {
          const int j = ring_slot(head0, p, slots);
          G.sy[j][head0] = tot[5 + 4 * p];
          G.yy[head0][j] = G.yy[j][head0] = tot[5 + 4 * p + 1];
        }
        s.rho[head0] = (float)(1.0 / sy);
        s.gamma = (float)(sy / yy);
        head = (head0 + 1) % slots;
        count = min(count0 + 1, a.h);
      }
      s.f = s.ft;
      if (!isfinite(s.f) || !isfinite(tot[4])) s.nonfinite = 1;
    } else if (phase == PH_FAIL) {
      count = 0;
      head = 0;
      if (a.status) a.status[b] |= KVS_ST_LS_FAIL;
    }
    s.phase = PH_IDLE;
    s.lse_stale = phase == PH_FAIL;  // the last loss forward ran at a rejected trial
    if (s.nonfinite && a.status) a.status[b] |= KVS_ST_NONFINITE;
    s.nonfinite = 0;
    if (a.f_out) a.f_out[b] = s.f;
  } else {
    s.f = a.f[b];
    s.phase = PH_IDLE;
    s.trials = 0;
    s.lse_stale = 0;
    // reported by the next step (the reset itself has no status array)
    s.nonfinite = !isfinite(s.f) || !isfinite(tot[4]);
    if (a.clear) {
      count = 0;
      head = 0;
      s.gamma = 1.f;
    }
  }
  s.count = count;
  s.head = head;
  int sl[16];
  double sg[16], yg[16];
  for (int p = 0; p < count; ++p) {
    const int q = kept ? p - 1 : p;  // index among the pairs read by this pass
    sl[p] = ring_slot(head, p, slots);
    sg[p] = q < 0 ? tot[2] : tot[5 + 4 * q + 2];
    yg[p] = q < 0 ? tot[3] : tot[5 + 4 * q + 3];
  }
  direction_coefs(G, count, sl, sg, yg, tot[4], a.dc[b]);
}

// d = cg g + sum_p (cy[p] y_p + cs[p] s_p); arms the Armijo search.
__global__ void __launch_bounds__(PT) k_direction(LbfgsScal *sc, const DirCoef *dc,
                                                  const float *__restrict__ g,
                                                  float *__restrict__ dir, const float *ring_s,
                                                  const float *ring_y, int64_t rstride, int h,
                                                  const int64_t *c_off, int d) {
  const int b = blockIdx.y, cb = blockIdx.x;
  const int64_t o = c_off[b] * (int64_t)d, n = c_off[b + 1] * (int64_t)d - o;
  if ((int64_t)cb * CH >= n) return;
  LbfgsScal &s = sc[b];
  const DirCoef &c = dc[b];
  const int slots = h + 1;
  const int cnt = min(max(c.cnt, 0), h), head = min(max(s.head, 0), h);
  const int64_t base = o + (int64_t)cb * CH;
  const int lim = (int)(n - (int64_t)cb * CH < CH ? n - (int64_t)cb * CH : CH);
  float4 r[V4];
#pragma unroll
  for (int u = 0; u < V4; ++u) {
    const int e = (u * PT + threadIdx.x) * 4;
    r[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (e < lim) {
      const float4 gv = ld4(g + base + e);
      r[u] = make_float4(c.cg * gv.x, c.cg * gv.y, c.cg * gv.z, c.cg * gv.w);
    }
  }
  for (int p = 0; p < cnt; ++p) {
    const int sl = ring_slot(head, p, slots);
    const float cy = c.cy[p], cs = c.cs[p];
    const float *rs = ring_s + sl * rstride + base, *ry = ring_y + sl * rstride + base;
#pragma unroll
    for (int u = 0; u < V4; ++u) {
      const int e = (u * PT + threadIdx.x) * 4;
      if (e >= lim) continue;
      const float4 sv = ld4(rs + e), yv = ld4(ry + e);
      r[u].x = fmaf(cs, sv.x, fmaf(cy, yv.x, r[u].x));
      r[u].y = fmaf(cs, sv.y, fmaf(cy, yv.y, r[u].y));
      r[u].z = fmaf(cs, sv.z, fmaf(cy, yv.z, r[u].z));
      r[u].w = fmaf(cs, sv.w, fmaf(cy, yv.w, r[u].w));
    }
  }
#pragma unroll
  for (int u = 0; u < V4; ++u) {
    const int e = (u * PT + threadIdx.x) * 4;
    if (e < lim) st4(dir + base + e, r[u]);
  }
  if (cb == 0 && threadIdx.x == 0) {
    s.gtd = c.gtd;
    s.t = c.t0;
    s.trials = 0;
    s.phase = PH_SEARCH;
  }
}

// Kc = x + t d for problems still searching, with the bf16 hi/lo split of the
// trial keys that the loss forward reads (pairs of elements: n is even).
__global__ void k_trial(const LbfgsScal *sc, const float *__restrict__ x,
                        const float *__restrict__ dir, float *__restrict__ Kc,
                        __nv_bfloat16 *__restrict__ kh, __nv_bfloat16 *__restrict__ kl,
                        const int64_t *c_off, const int64_t *c_pad, int d) {
  const int b = blockIdx.y;
  if (sc[b].phase != PH_SEARCH) return;
  const int64_t o = seg0(c_off, b, d), n = c_off[b + 1] * (int64_t)d - o;
  const int64_t op = c_pad[b] * (int64_t)d;  // the split at the padded pair rows
  const float t = sc[b].t;
  for (int64_t i = 2 * (blockIdx.x * (int64_t)blockDim.x + threadIdx.x); i < n;
       i += 2 * (int64_t)gridDim.x * blockDim.x) {
    const float2 xv = *reinterpret_cast<const float2 *>(x + o + i);
    const float2 dv = *reinterpret_cast<const float2 *>(dir + o + i);
    const float k0 = fmaf(t, dv.x, xv.x), k1 = fmaf(t, dv.y, xv.y);
    *reinterpret_cast<float2 *>(Kc + o + i) = make_float2(k0, k1);
    const __nv_bfloat162 h = __floats2bfloat162_rn(k0, k1);
    const float2 hf = __bfloat1622float2(h);
    *reinterpret_cast<__nv_bfloat162 *>(kh + op + i) = h;
    *reinterpret_cast<__nv_bfloat162 *>(kl + op + i) = __floats2bfloat162_rn(k0 - hf.x, k1 - hf.y);
  }
}

// Armijo test of the trial loss: accept, or halve t, or give up after max_bt
// trials.  The loss is summed (fixed order, double) from the loss forward's
// per-CTA partials of the output and LSE terms.  One CTA walks all problems;
// inside a CUDA graph it also sets the trial loop's condition to "some
// problem is still searching".
__global__ void __launch_bounds__(256) k_armijo(LbfgsScal *sc, int B, const float *partials,
                                                int tiles, const int64_t *q_off, int d,
                                                float w_out, float w_lse, float c1,
                                                float backtrack, int max_bt, int use_cond,
                                                cudaGraphConditionalHandle cond) {
  int still = 0;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    LbfgsScal &s = sc[b];
    if (s.phase != PH_SEARCH) continue;
    const int nq = (int)(q_off[b + 1] - q_off[b]);
    double so = 0.0, sl = 0.0;
    for (int t = 0; t < (nq + 127) / 128; ++t) {
      so += partials[((int64_t)b * tiles + t) * 2];
      sl += partials[((int64_t)b * tiles + t) * 2 + 1];
    }
    const float f = (float)(w_out * (so / ((double)nq * d)) + w_lse * (sl / (double)nq));
    s.trials += 1;
    if (!isfinite(f)) s.nonfinite = 1;
    if (isfinite(f) && f <= s.f + c1 * s.t * s.gtd) {
      s.ft = f;
      s.phase = PH_ACCEPT;
    } else if (s.trials >= max_bt) {
      s.phase = PH_FAIL;
    } else {
      s.t *= backtrack;
      still = 1;
    }
  }
  still = __syncthreads_or(still);
  if (use_cond && threadIdx.x == 0) cudaGraphSetConditional(cond, still ? 1u : 0u);
}

__global__ void k_copy_f(const LbfgsScal *sc, int B, float *dst, int64_t stride, int64_t col) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) dst[b * stride + col] = sc[b].f;
}

PairArgs pair_args(const Batch &Bt, const State &s) {
  PairArgs a{};
  a.sc = s.sc;
  a.gram = s.gram;
  a.dc = s.dc;
  a.part = s.part;
  a.ticket = s.ticket;
  a.x = s.x;
  a.g = s.g;
  a.ring_s = s.ring_s;
  a.ring_y = s.ring_y;
  a.rstride = Bt.g.sum_c * Bt.g.d;
  a.h = s.h;
  a.d = Bt.g.d;
  a.cmax = s.cmax;
  a.c_off = Bt.b->c_off;
  return a;
}

}  // namespace

int launch_lbfgs_reset(const Batch &Bt, const State &s, const float *Kc, const float *f,
                       const float *g, int clear) {
  if (clear) KVS_CUDA_TRY(cudaMemsetAsync(s.ticket, 0, sizeof(int) * Bt.g.B, Bt.st));
  PairArgs a = pair_args(Bt, s);
  a.Kc = const_cast<float *>(Kc);  // read only when resetting
  a.f = f;
  a.gsrc = g;
  a.clear = clear;
  k_pairs<MODE_RESET><<<dim3(s.cmax, Bt.g.B), PT, 0, Bt.st>>>(a);
  KVS_LAUNCH_CHECK("k_pairs");
  return KVS_OK;
}

int launch_lbfgs_direction(const Batch &Bt, const State &s, const kvs_schedule &) {
  k_direction<<<dim3(s.cmax, Bt.g.B), PT, 0, Bt.st>>>(s.sc, s.dc, s.g, s.dir, s.ring_s, s.ring_y,
                                                      Bt.g.sum_c * Bt.g.d, s.h, Bt.b->c_off,
                                                      Bt.g.d);
  KVS_LAUNCH_CHECK("k_direction");
  return KVS_OK;
}

int launch_lbfgs_trial(const Batch &Bt, const State &s, float *Kc, const Work &w) {
  const int64_t n = (int64_t)Bt.g.max_c * Bt.g.d / 2;
  const int blocks = (int)std::min<int64_t>((n + 255) / 256, 64);
  k_trial<<<dim3(blocks, Bt.g.B), 256, 0, Bt.st>>>(s.sc, s.x, s.dir, Kc, w.kh, w.kl,
                                                   Bt.b->c_off, w.c_pad, Bt.g.d);
  KVS_LAUNCH_CHECK("k_trial");
  return KVS_OK;
}

int launch_lbfgs_armijo(const Batch &Bt, const State &s, const kvs_schedule &sc, const Work &w,
                        const cudaGraphConditionalHandle *cond) {
  k_armijo<<<1, 256, 0, Bt.st>>>(s.sc, Bt.g.B, w.partials, (Bt.g.max_q + 127) / 128,
                                 Bt.b->q_off, Bt.g.d, sc.w_out, sc.w_lse, sc.c1, sc.backtrack,
                                 sc.max_bt, cond ? 1 : 0,
                                 cond ? *cond : cudaGraphConditionalHandle{});
  KVS_LAUNCH_CHECK("k_armijo");
  return KVS_OK;
}

int launch_lbfgs_update(const Batch &Bt, const State &s, float *Kc, int32_t *status,
                        float *f_out) {
  PairArgs a = pair_args(Bt, s);
  a.Kc = Kc;
  a.gsrc = s.gn;
  a.status = status;
  a.f_out = f_out;
  k_pairs<MODE_UPDATE><<<dim3(s.cmax, Bt.g.B), PT, 0, Bt.st>>>(a);
  KVS_LAUNCH_CHECK("k_pairs");
  return KVS_OK;
}

int launch_copy_f(const Batch &Bt, const State &s, float *dst, int64_t stride, int64_t col) {
  k_copy_f<<<(Bt.g.B + 127) / 128, 128, 0, Bt.st>>>(s.sc, Bt.g.B, dst, stride, col);
  KVS_LAUNCH_CHECK("k_copy_f");
  return KVS_OK;
}

}  // namespace kvs
