// Device-resident batched L-BFGS on the compressed keys.
//
// "KVSculpt: KV Cache Compression as Distillation", section 2 "Key
// Optimization": keys are optimised by L-BFGS (a quasi-Newton method).  The
// pages name the method only; the constants (history h, H0 = gamma I from
// the newest pair, curvature test s.y > 1e-10 y.y, Armijo backtracking with a
// deterministic halving schedule, first trial min(1, 1/|g|) on an empty
// history) are the reading stated in the library header.
//
// Every problem owns a segment of n_b = k_b * d floats in each vector.  The
// two-loop recursion runs one CTA per problem with fixed-order block
// reductions, so a run is bit-reproducible.  Each pass over the vectors fuses
// the axpy of one pair with the dot product of the next one: every history
// vector is read once per loop (4 h n floats per direction).
#include <math.h>

#include "kvs_internal.cuh"

namespace kvs {
namespace {

constexpr int NT = 1024;

__device__ __forceinline__ int64_t seg0(const int64_t *c_off, int b, int d) {
  return c_off[b] * (int64_t)d;
}

__global__ void __launch_bounds__(NT) k_reset(LbfgsScal *sc, float *x, float *g,
                                              const float *Kc, const float *f,
                                              const float *gsrc, const int64_t *c_off, int d,
                                              int clear) {
  const int b = blockIdx.x;
  const int64_t o = seg0(c_off, b, d), n = c_off[b + 1] * (int64_t)d - o;
  for (int64_t i = threadIdx.x; i < n; i += NT) {
    x[o + i] = Kc[o + i];
    g[o + i] = gsrc[o + i];
  }
  if (threadIdx.x == 0) {
    LbfgsScal &s = sc[b];
    s.f = f[b];
    s.phase = PH_IDLE;
    s.trials = 0;
    if (clear) {
      s.count = 0;
      s.head = 0;
      s.gamma = 1.f;
    }
  }
}

// Two-loop recursion d = -H g (H0 = gamma I), then the first trial step.
__global__ void __launch_bounds__(NT) k_direction(LbfgsScal *sc, const float *__restrict__ g,
                                                  float *__restrict__ q, const float *ring_s,
                                                  const float *ring_y, int64_t rstride, int h,
                                                  const int64_t *c_off, int d) {
  __shared__ float red[32];
  __shared__ float alpha[16];
  const int b = blockIdx.x;
  LbfgsScal &s = sc[b];
  const int64_t o = seg0(c_off, b, d), n = c_off[b + 1] * (int64_t)d - o;
  const int slots = h + 1;
  const int count = min(max(s.count, 0), h), head = min(max(s.head, 0), h);
  const float gamma = count > 0 ? s.gamma : 1.f;
  // loop 1, newest pair first: q <- q - alpha_j y_j ; alpha_j = rho_j s_j . q
  for (int p = 0; p <= count; ++p) {
    const int sl_prev = p > 0 ? (head - p + slots) % slots : 0;  // pair j = p - 1
    const int sl = (head - 1 - p + 2 * slots) % slots;           // pair j = p
    const float *yp = ring_y + sl_prev * rstride + o;
    const float *sp = ring_s + sl * rstride + o;
    const float ap = p > 0 ? alpha[p - 1] : 0.f;
    float acc = 0.f;
    for (int64_t i = threadIdx.x; i < n; i += NT) {
      float qi = p == 0 ? g[o + i] : q[o + i];
      if (p > 0) qi = fmaf(-ap, yp[i], qi);
      if (p < count) acc = fmaf(sp[i], qi, acc);
      else qi *= gamma;
      q[o + i] = qi;
    }
    if (p < count) {
      const float dot = block_sum(acc, red);
      if (threadIdx.x == 0) alpha[p] = s.rho[sl] * dot;
      __syncthreads();
    }
  }
  // loop 2, oldest pair first: r <- r + (alpha_j - beta_j) s_j ; beta_j = rho_j y_j . r
  float beta_prev = 0.f;
  for (int p = 0; p <= count; ++p) {
    const int jj = count - 1 - p;                                    // pair handled now
    const int jprev = count - p;                                     // pair finished last pass
    const int sl = (head - 1 - jj + 2 * slots) % slots;
    const int slp = (head - 1 - jprev + 2 * slots) % slots;
    const float *yc = ring_y + sl * rstride + o;
    const float *spv = ring_s + slp * rstride + o;
    const float coef = p > 0 ? alpha[jprev] - beta_prev : 0.f;
    float acc = 0.f;
    for (int64_t i = threadIdx.x; i < n; i += NT) {
      float ri = q[o + i];
      if (p > 0) ri = fmaf(coef, spv[i], ri);
      if (p < count) acc = fmaf(yc[i], ri, acc);
      q[o + i] = ri;
    }
    if (p < count) {
      const float dot = block_sum(acc, red);
      beta_prev = s.rho[sl] * dot;
    }
  }
  // d = -r ; g.d and |g|^2
  float gd = 0.f, gg = 0.f;
  for (int64_t i = threadIdx.x; i < n; i += NT) {
    const float di = -q[o + i];
    const float gi = g[o + i];
    q[o + i] = di;
    gd = fmaf(gi, di, gd);
    gg = fmaf(gi, gi, gg);
  }
  gd = block_sum(gd, red);
  gg = block_sum(gg, red);
  if (!(gd < 0.f)) {
    for (int64_t i = threadIdx.x; i < n; i += NT) q[o + i] = -g[o + i];
    gd = -gg;
  }
  if (threadIdx.x == 0) {
    s.gtd = gd;
    const float gn = sqrtf(gg);
    s.t = count > 0 ? 1.f : (gn > 0.f ? fminf(1.f, 1.f / gn) : 1.f);
    s.trials = 0;
    s.phase = PH_SEARCH;
  }
}

// Kc = x + t d for problems still searching, with the bf16 hi/lo split of the
// trial keys that the loss forward reads (pairs of elements: n is even).
__global__ void k_trial(const LbfgsScal *sc, const float *__restrict__ x,
                        const float *__restrict__ dir, float *__restrict__ Kc,
                        __nv_bfloat16 *__restrict__ kh, __nv_bfloat16 *__restrict__ kl,
                        const int64_t *c_off, int d) {
  const int b = blockIdx.y;
  if (sc[b].phase != PH_SEARCH) return;
  const int64_t o = seg0(c_off, b, d), n = c_off[b + 1] * (int64_t)d - o;
  const float t = sc[b].t;
  for (int64_t i = 2 * (blockIdx.x * (int64_t)blockDim.x + threadIdx.x); i < n;
       i += 2 * (int64_t)gridDim.x * blockDim.x) {
    const float2 xv = *reinterpret_cast<const float2 *>(x + o + i);
    const float2 dv = *reinterpret_cast<const float2 *>(dir + o + i);
    const float k0 = fmaf(t, dv.x, xv.x), k1 = fmaf(t, dv.y, xv.y);
    *reinterpret_cast<float2 *>(Kc + o + i) = make_float2(k0, k1);
    const __nv_bfloat162 h = __floats2bfloat162_rn(k0, k1);
    const float2 hf = __bfloat1622float2(h);
    *reinterpret_cast<__nv_bfloat162 *>(kh + o + i) = h;
    *reinterpret_cast<__nv_bfloat162 *>(kl + o + i) = __floats2bfloat162_rn(k0 - hf.x, k1 - hf.y);
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

// Accepted: store (s, y) in the scratch slot, keep it when s.y > 1e-10 y.y,
// move x, g, f.  Failed: restore Kc = x, clear the history, flag LS_FAIL.
__global__ void __launch_bounds__(NT) k_update(LbfgsScal *sc, float *__restrict__ x,
                                               float *__restrict__ g,
                                               const float *__restrict__ gn,
                                               float *__restrict__ Kc, float *ring_s,
                                               float *ring_y, int64_t rstride, int h,
                                               const int64_t *c_off, int d, int32_t *status,
                                               float *f_out) {
  __shared__ float red[32];
  const int b = blockIdx.x;
  LbfgsScal &s = sc[b];
  const int phase = s.phase;
  const int64_t o = seg0(c_off, b, d), n = c_off[b + 1] * (int64_t)d - o;
  if (phase == PH_ACCEPT) {
    const int slot = min(max(s.head, 0), h);
    float *rs = ring_s + slot * rstride + o;
    float *ry = ring_y + slot * rstride + o;
    float sy = 0.f, yy = 0.f;
    for (int64_t i = threadIdx.x; i < n; i += NT) {
      const float xn = Kc[o + i], gv = gn[o + i];
      const float si = xn - x[o + i], yi = gv - g[o + i];
      rs[i] = si;
      ry[i] = yi;
      x[o + i] = xn;
      g[o + i] = gv;
      sy = fmaf(si, yi, sy);
      yy = fmaf(yi, yi, yy);
    }
    sy = block_sum(sy, red);
    yy = block_sum(yy, red);
    if (threadIdx.x == 0) {
      if (sy > 1e-10f * yy) {
        s.rho[slot] = 1.f / sy;
        s.gamma = sy / yy;
        s.head = (slot + 1) % (h + 1);
        s.count = min(max(s.count, 0) + 1, h);
      }
      s.f = s.ft;
      if (!isfinite(s.f) && status) status[b] |= KVS_ST_NONFINITE;
    }
  } else if (phase == PH_FAIL) {
    for (int64_t i = threadIdx.x; i < n; i += NT) Kc[o + i] = x[o + i];
    if (threadIdx.x == 0) {
      s.count = 0;
      s.head = 0;
      if (status) status[b] |= KVS_ST_LS_FAIL;
    }
  }
  if (threadIdx.x == 0) {
    s.phase = PH_IDLE;
    if (f_out) f_out[b] = s.f;
  }
}

__global__ void k_copy_f(const LbfgsScal *sc, int B, float *dst, int64_t stride, int64_t col) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) dst[b * stride + col] = sc[b].f;
}

}  // namespace

int launch_lbfgs_reset(const Batch &Bt, const State &s, const float *Kc, const float *f,
                       const float *g, int clear) {
  k_reset<<<Bt.g.B, NT, 0, Bt.st>>>(s.sc, s.x, s.g, Kc, f, g, Bt.b->c_off, Bt.g.d, clear);
  KVS_LAUNCH_CHECK("k_reset");
  return KVS_OK;
}

int launch_lbfgs_direction(const Batch &Bt, const State &s, const kvs_schedule &) {
  k_direction<<<Bt.g.B, NT, 0, Bt.st>>>(s.sc, s.g, s.dir, s.ring_s, s.ring_y,
                                        Bt.g.sum_c * Bt.g.d, s.h, Bt.b->c_off, Bt.g.d);
  KVS_LAUNCH_CHECK("k_direction");
  return KVS_OK;
}

int launch_lbfgs_trial(const Batch &Bt, const State &s, float *Kc, const Work &w) {
  const int64_t n = (int64_t)Bt.g.max_c * Bt.g.d / 2;
  const int blocks = (int)std::min<int64_t>((n + 255) / 256, 64);
  k_trial<<<dim3(blocks, Bt.g.B), 256, 0, Bt.st>>>(s.sc, s.x, s.dir, Kc, w.kh, w.kl,
                                                   Bt.b->c_off, Bt.g.d);
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
  k_update<<<Bt.g.B, NT, 0, Bt.st>>>(s.sc, s.x, s.g, s.gn, Kc, s.ring_s, s.ring_y,
                                     Bt.g.sum_c * Bt.g.d, s.h, Bt.b->c_off, Bt.g.d, status,
                                     f_out);
  KVS_LAUNCH_CHECK("k_update");
  return KVS_OK;
}

int launch_copy_f(const Batch &Bt, const State &s, float *dst, int64_t stride, int64_t col) {
  k_copy_f<<<(Bt.g.B + 127) / 128, 128, 0, Bt.st>>>(s.sc, Bt.g.B, dst, stride, col);
  KVS_LAUNCH_CHECK("k_copy_f");
  return KVS_OK;
}

}  // namespace kvs
