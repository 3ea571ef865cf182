// Batched Cholesky factorisation and triangular solves of the ridge normal
// equations (A^T A + lam I) V_c = A^T Y ("KVSculpt: KV Cache Compression as
// Distillation", section 2 "Value Optimization": values in closed form by
// ridge regression).
//
// One CTA per problem; factor and solves run in float64 on the CUDA cores
// (the Gram matrix of softmax weights reaches condition numbers of ~3e4 on
// the synthetic Qwen-shaped workloads).  A pivot <= 0 (or non-finite) marks
// the problem KVS_ST_NOT_PD and leaves its V_c untouched.
#include <math.h>

#include "kvs_internal.cuh"

namespace kvs {
namespace {

constexpr int NB = 32;

__global__ void __launch_bounds__(1024) k_chol_solve(const float *__restrict__ gram,
                                                     double *__restrict__ L,
                                                     const float *__restrict__ R,
                                                     double *__restrict__ X, float *Vc,
                                                     int32_t *status, const int64_t *c_off,
                                                     int64_t ld, int d) {
  const int b = blockIdx.x;
  const int64_t r0 = c_off[b];
  const int k = (int)(c_off[b + 1] - r0);
  if (k <= 0) return;
  const int tid = threadIdx.x, nt = blockDim.x;
  const float *G = gram + r0 * ld;
  double *Lb = L + r0 * ld;
  __shared__ double D[NB][NB + 1];
  __shared__ double Pi[NB][NB + 1];
  __shared__ double Pj[NB][NB + 1];
  __shared__ int bad;
  if (tid == 0) bad = 0;
  for (int64_t e = tid; e < (int64_t)k * k; e += nt) {
    const int i = (int)(e / k), j = (int)(e % k);
    if (j <= i) Lb[(int64_t)i * ld + j] = (double)G[(int64_t)i * ld + j];
  }
  __syncthreads();
  for (int j0 = 0; j0 < k; j0 += NB) {
    const int jb = min(NB, k - j0);
    // (1) diagonal block, unblocked, in shared memory by warp 0
    for (int e = tid; e < NB * NB; e += nt) {
      const int r = e / NB, c = e % NB;
      D[r][c] = (r < jb && c <= r) ? Lb[(int64_t)(j0 + r) * ld + j0 + c] : 0.0;
    }
    __syncthreads();
    if (tid < 32) {
      const int r = tid;
      for (int c = 0; c < jb; ++c) {
        if (r == c) {
          const double piv = D[c][c];
          if (!(piv > 0.0) || !isfinite(piv)) bad = 1;
          D[c][c] = sqrt(fmax(piv, 1e-300));
        }
        __syncwarp();
        if (r > c && r < jb) D[r][c] /= D[c][c];
        __syncwarp();
        if (r > c && r < jb)
          for (int cc = c + 1; cc <= r; ++cc) D[r][cc] -= D[r][c] * D[cc][c];
        __syncwarp();
      }
    }
    __syncthreads();
    if (bad) {
      if (tid == 0) status[b] |= KVS_ST_NOT_PD;
      return;
    }
    for (int e = tid; e < NB * NB; e += nt) {
      const int r = e / NB, c = e % NB;
      if (r < jb && c <= r) Lb[(int64_t)(j0 + r) * ld + j0 + c] = D[r][c];
    }
    // (2) panel below the diagonal block: L21 = A21 L11^-T, one row per thread
    for (int i = j0 + jb + tid; i < k; i += nt) {
      double *row = Lb + (int64_t)i * ld + j0;
      double x[NB];
#pragma unroll
      for (int c = 0; c < NB; ++c) {
        if (c < jb) {
          double a = row[c];
          for (int t = 0; t < c; ++t) a -= x[t] * D[c][t];
          x[c] = a / D[c][c];
          row[c] = x[c];
        }
      }
    }
    __syncthreads();
    // (3) trailing update of the lower triangle: A22 -= L21 L21^T
    const int s0 = j0 + jb;
    const int n2 = k - s0;
    const int nt2 = (n2 + NB - 1) / NB;
    for (int ti = 0; ti < nt2; ++ti) {
      for (int e = tid; e < NB * NB; e += nt) {
        const int r = e / NB, c = e % NB;
        const int i = s0 + ti * NB + r;
        Pi[r][c] = (i < k && c < jb) ? Lb[(int64_t)i * ld + j0 + c] : 0.0;
      }
      for (int tj = 0; tj <= ti; ++tj) {
        for (int e = tid; e < NB * NB; e += nt) {
          const int r = e / NB, c = e % NB;
          const int j = s0 + tj * NB + r;
          Pj[r][c] = (j < k && c < jb) ? Lb[(int64_t)j * ld + j0 + c] : 0.0;
        }
        __syncthreads();
        {
          const int r = tid / NB, c = tid % NB;
          const int i = s0 + ti * NB + r, j = s0 + tj * NB + c;
          if (tid < NB * NB && i < k && j <= i) {
            double acc = 0.0;
#pragma unroll 8
            for (int t = 0; t < NB; ++t) acc += Pi[r][t] * Pj[c][t];
            Lb[(int64_t)i * ld + j] -= acc;
          }
        }
        __syncthreads();
      }
    }
    __syncthreads();
  }
  // Solves: forward L y = R, backward L^T x = y; X holds the d right-hand sides.
  double *Xb = X + r0 * d;
  const float *Rb = R + r0 * d;
  for (int64_t e = tid; e < (int64_t)k * d; e += nt) Xb[e] = (double)Rb[e];
  __syncthreads();
  for (int i0 = 0; i0 < k; i0 += NB) {
    const int ib = min(NB, k - i0);
    for (int e = tid; e < ib * d; e += nt) {
      const int r = e / d, c = e % d;
      const double *lr = Lb + (int64_t)(i0 + r) * ld;
      double acc = 0.0;
      for (int t = 0; t < i0; ++t) acc += lr[t] * Xb[(int64_t)t * d + c];
      Xb[(int64_t)(i0 + r) * d + c] -= acc;
    }
    __syncthreads();
    for (int c = tid; c < d; c += nt) {
      for (int r = 0; r < ib; ++r) {
        const double *lr = Lb + (int64_t)(i0 + r) * ld + i0;
        double a = Xb[(int64_t)(i0 + r) * d + c];
        for (int t = 0; t < r; ++t) a -= lr[t] * Xb[(int64_t)(i0 + t) * d + c];
        Xb[(int64_t)(i0 + r) * d + c] = a / lr[r];
      }
    }
    __syncthreads();
  }
  const int nblk = (k + NB - 1) / NB;
  for (int bi = nblk - 1; bi >= 0; --bi) {
    const int i0 = bi * NB;
    const int ib = min(NB, k - i0);
    for (int e = tid; e < ib * d; e += nt) {
      const int r = e / d, c = e % d;
      const int i = i0 + r;
      double acc = 0.0;
      for (int t = i0 + ib; t < k; ++t) acc += Lb[(int64_t)t * ld + i] * Xb[(int64_t)t * d + c];
      Xb[(int64_t)i * d + c] -= acc;
    }
    __syncthreads();
    for (int c = tid; c < d; c += nt) {
      for (int r = ib - 1; r >= 0; --r) {
        const int i = i0 + r;
        double a = Xb[(int64_t)i * d + c];
        for (int t = r + 1; t < ib; ++t) a -= Lb[(int64_t)(i0 + t) * ld + i] * Xb[(int64_t)(i0 + t) * d + c];
        Xb[(int64_t)i * d + c] = a / Lb[(int64_t)i * ld + i];
      }
    }
    __syncthreads();
  }
  bool finite = true;
  for (int64_t e = tid; e < (int64_t)k * d; e += nt) finite &= isfinite(Xb[e]);
  finite = __syncthreads_and(finite);
  if (!finite) {
    if (tid == 0) status[b] |= KVS_ST_NONFINITE;
    return;
  }
  float *V = Vc + r0 * d;
  for (int64_t e = tid; e < (int64_t)k * d; e += nt) V[e] = (float)Xb[e];
}

}  // namespace

int launch_chol_solve(const Batch &Bt, float *Vc, int32_t *status, const Work &w) {
  k_chol_solve<<<Bt.g.B, 1024, 0, Bt.st>>>(w.gram, w.chol, w.R, w.xs, Vc, status, Bt.b->c_off,
                                           Bt.g.max_c, Bt.g.d);
  KVS_LAUNCH_CHECK("k_chol_solve");
  return KVS_OK;
}

}  // namespace kvs
