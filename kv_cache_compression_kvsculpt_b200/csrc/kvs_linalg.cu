// Batched Cholesky factorisation and triangular solves of the ridge normal
// equations (A^T A + lam I) V_c = A^T Y ("KVSculpt: KV Cache Compression as
// Distillation", section 2 "Value Optimization": values in closed form by
// ridge regression).
//
// Right-looking blocked algorithm over panels of NB = 64 columns, float32,
// every problem of the batch advancing together so that all SMs share the work:
//   per panel j:
//     diag    factor the diagonal block G_jj = L_jj L_jj^T in shared memory and
//             keep T_j = L_jj^-1
//     tmul    forward-solved rows y_j = T_j r_j
//     panel   L_ij = G_ij T_j^T for the rows below
//     update  G_ik -= L_ij L_kj^T on the trailing lower triangle and
//             r_i -= L_ij y_j on the right-hand sides (64 x 64 register tiles)
//   then per panel from the last one: x_j = T_j^T y_j and y_i -= L_ji^T x_j.
// The factor overwrites the Gram matrix, the solution the right-hand sides.
// A pivot <= 0 (or non-finite) marks the problem KVS_ST_NOT_PD; its V_c is
// left untouched and its remaining steps are skipped.
#include <math.h>

#include "kvs_internal.cuh"

namespace kvs {
namespace {

constexpr int NB = 64;

struct CholArgs {
  float *G;              // [sum_c, ld] Gram matrix -> factor (lower triangle)
  float *R;              // [sum_c, d] right-hand sides -> solution
  float *T;              // [B, npanel, NB, NB] inverses of the diagonal blocks
  int npanel;
  int *dead;             // [B] set once a problem's factorisation failed
  int32_t *status;
  const int64_t *c_off;
  int64_t ld;
  int d;
};

__device__ __forceinline__ int kdim(const CholArgs &a, int b) {
  return (int)(a.c_off[b + 1] - a.c_off[b]);
}

// Diagonal block of panel j0: factor in shared memory and keep its inverse T_j.
__global__ void __launch_bounds__(256) k_chol_diag(CholArgs a, int j0) {
  const int b = blockIdx.x;
  const int k = kdim(a, b);
  if (j0 >= k || a.dead[b]) return;
  const int jb = min(NB, k - j0);
  __shared__ float L[NB][NB + 1];
  __shared__ float Ti[NB][NB + 1];
  __shared__ int bad;
  float *G = a.G + (a.c_off[b] + j0) * a.ld + j0;
  const int tid = threadIdx.x;
  if (tid == 0) bad = 0;
  for (int e = tid; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    L[r][c] = (r < jb && c <= r) ? G[(int64_t)r * a.ld + c] : 0.f;
    Ti[r][c] = 0.f;
  }
  __syncthreads();
  for (int c = 0; c < jb; ++c) {
    if (tid == 0) {
      const float piv = L[c][c];
      if (!(piv > 0.f) || !isfinite(piv)) bad = 1;
      L[c][c] = sqrtf(fmaxf(piv, 1e-30f));
    }
    __syncthreads();
    const float inv = 1.f / L[c][c];
    for (int i = c + 1 + tid; i < jb; i += blockDim.x) L[i][c] *= inv;
    __syncthreads();
    const int n = jb - c - 1;
    for (int e = tid; e < n * n; e += blockDim.x) {
      const int i = c + 1 + e / n, j = c + 1 + e % n;
      if (j <= i) L[i][j] -= L[i][c] * L[j][c];
    }
    __syncthreads();
  }
  if (bad) {
    if (tid == 0) {
      a.status[b] |= KVS_ST_NOT_PD;
      a.dead[b] = 1;
    }
    return;
  }
  // T = L^-1 (lower triangular), one column per thread
  if (tid < jb) {
    const int c = tid;
    Ti[c][c] = 1.f / L[c][c];
    for (int i = c + 1; i < jb; ++i) {
      float s = 0.f;
      for (int t = c; t < i; ++t) s = fmaf(L[i][t], Ti[t][c], s);
      Ti[i][c] = -s / L[i][i];
    }
  }
  __syncthreads();
  float *Tg = a.T + ((int64_t)b * a.npanel + j0 / NB) * NB * NB;
  for (int e = tid; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    if (r < jb && c <= r) G[(int64_t)r * a.ld + c] = L[r][c];
    Tg[e] = Ti[r][c];
  }
}

// Rows j0 .. j0+63 of the right-hand sides times T_j (forward sweep) or T_j^T
// (backward sweep), in place; 64 columns of R per CTA, 4 x 4 register tiles.
__global__ void __launch_bounds__(256) k_chol_tmul(CholArgs a, int j0, int transpose) {
  const int b = blockIdx.y;
  const int k = kdim(a, b);
  if (j0 >= k || a.dead[b]) return;
  const int jb = min(NB, k - j0);
  const int c0 = blockIdx.x * NB;
  if (c0 >= a.d) return;
  __shared__ float Ts[NB][NB + 4];  // Ts[r][t] = M[r][t]
  __shared__ float Xs[NB][NB + 4];  // Xs[col][t] = R[j0 + t][c0 + col]
  const float *Tg = a.T + ((int64_t)b * a.npanel + j0 / NB) * NB * NB;
  float *R = a.R + (a.c_off[b] + j0) * a.d + c0;
  const int tid = threadIdx.x;
  for (int e = tid; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, t = e % NB;
    Ts[r][t] = transpose ? Tg[t * NB + r] : Tg[e];
    Xs[t][r] = (r < jb && c0 + t < a.d) ? R[(int64_t)r * a.d + t] : 0.f;
  }
  __syncthreads();
  const int tx = tid & 15, ty = tid >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
  for (int t = 0; t < NB; ++t) {
    float av[4], bv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) av[i] = Ts[ty + 16 * i][t];
#pragma unroll
    for (int j = 0; j < 4; ++j) bv[j] = Xs[tx + 16 * j][t];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty + 16 * i;
    if (r >= jb) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = tx + 16 * j;
      if (c0 + col < a.d) R[(int64_t)r * a.d + col] = acc[i][j];
    }
  }
}

// L_ij = G_ij T^T for 64 rows of the panel below the diagonal block.
__global__ void __launch_bounds__(256) k_chol_panel(CholArgs a, int j0) {
  const int b = blockIdx.y;
  const int k = kdim(a, b);
  if (j0 >= k || a.dead[b]) return;
  const int jb = min(NB, k - j0);
  const int i0 = j0 + jb + blockIdx.x * NB;
  if (i0 >= k) return;
  const int ib = min(NB, k - i0);
  __shared__ float Ti[NB][NB + 1];
  __shared__ float Ar[NB][NB + 1];
  const int tid = threadIdx.x;
  float *P = a.G + (a.c_off[b] + i0) * a.ld + j0;
  for (int e = tid; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    Ti[r][c] = a.T[((int64_t)b * a.npanel + j0 / NB) * NB * NB + e];
    Ar[r][c] = (r < ib && c < jb) ? P[(int64_t)r * a.ld + c] : 0.f;
  }
  __syncthreads();
  for (int e = tid; e < ib * jb; e += blockDim.x) {
    const int r = e / jb, c = e % jb;
    float s = 0.f;
    for (int t = 0; t <= c; ++t) s = fmaf(Ar[r][t], Ti[c][t], s);
    P[(int64_t)r * a.ld + c] = s;
  }
}

// Trailing update: tiles (ti >= tj) of G_ik -= L_i L_k^T, and tiles of
// r_i -= L_i y_j (columns of R in chunks of 64), 64 x 64 outputs per CTA.
__global__ void __launch_bounds__(256) k_chol_update(CholArgs a, int j0, int ntile_max) {
  const int b = blockIdx.y;
  const int k = kdim(a, b);
  if (j0 >= k || a.dead[b]) return;
  const int jb = min(NB, k - j0);
  const int s0 = j0 + jb;
  const int n2 = k - s0;
  if (n2 <= 0) return;
  const int nt = (n2 + NB - 1) / NB;
  const int ntri = nt * (nt + 1) / 2;
  const int ndc = (a.d + NB - 1) / NB;
  int t = blockIdx.x;
  bool rhs = false;
  int ti, tj;
  if (t < ntri) {
    ti = (int)((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
    while (ti * (ti + 1) / 2 > t) --ti;
    while ((ti + 1) * (ti + 2) / 2 <= t) ++ti;
    tj = t - ti * (ti + 1) / 2;
  } else {
    t -= ntri;
    if (t >= nt * ndc) return;
    rhs = true;
    ti = t / ndc;
    tj = t % ndc;
  }
  __shared__ float As[NB][NB + 4];  // L_i panel rows, [row][c]
  __shared__ float Bs[NB][NB + 4];  // L_k panel rows or y_j, [row or col][c]
  const int tid = threadIdx.x;
  const int64_t row0 = a.c_off[b];
  const int ri = s0 + ti * NB;
  for (int e = tid; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    As[r][c] = (ri + r < k && c < jb) ? a.G[(row0 + ri + r) * a.ld + j0 + c] : 0.f;
    if (!rhs) {
      const int rk = s0 + tj * NB + r;
      Bs[r][c] = (rk < k && c < jb) ? a.G[(row0 + rk) * a.ld + j0 + c] : 0.f;
    } else {
      // Bs[col][c] = y_j[c][col]
      const int col = tj * NB + r;
      Bs[r][c] = (col < a.d && c < jb) ? a.R[(row0 + j0 + c) * a.d + col] : 0.f;
    }
  }
  __syncthreads();
  const int tx = tid & 15, ty = tid >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
  for (int c = 0; c < NB; ++c) {
    float av[4], bv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) av[i] = As[ty + 16 * i][c];
#pragma unroll
    for (int j = 0; j < 4; ++j) bv[j] = Bs[tx + 16 * j][c];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ri + ty + 16 * i;
    if (r >= k) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (!rhs) {
        const int cc = s0 + tj * NB + tx + 16 * j;
        if (cc < k && cc <= r) a.G[(row0 + r) * a.ld + cc] -= acc[i][j];
      } else {
        const int col = tj * NB + tx + 16 * j;
        if (col < a.d) a.R[(row0 + r) * a.d + col] -= acc[i][j];
      }
    }
  }
}

// Backward sweep update: y_i -= L_ji^T x_j for the rows i < j0 (64 x 64 tiles).
__global__ void __launch_bounds__(256) k_chol_bupdate(CholArgs a, int j0) {
  const int b = blockIdx.z;
  const int k = kdim(a, b);
  if (j0 >= k || a.dead[b]) return;
  const int jb = min(NB, k - j0);
  const int i0 = blockIdx.y * NB;
  if (i0 >= j0) return;
  const int c0 = blockIdx.x * NB;
  if (c0 >= a.d) return;
  __shared__ float As[NB][NB + 4];  // As[i][t] = L[j0 + t][i0 + i]
  __shared__ float Bs[NB][NB + 4];  // Bs[col][t] = x[t][c0 + col]
  const int tid = threadIdx.x;
  const int64_t row0 = a.c_off[b];
  for (int e = tid; e < NB * NB; e += blockDim.x) {
    const int t = e / NB, u = e % NB;
    As[u][t] = (t < jb && i0 + u < j0) ? a.G[(row0 + j0 + t) * a.ld + i0 + u] : 0.f;
    Bs[u][t] = (t < jb && c0 + u < a.d) ? a.R[(row0 + j0 + t) * a.d + c0 + u] : 0.f;
  }
  __syncthreads();
  const int tx = tid & 15, ty = tid >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
  for (int t = 0; t < NB; ++t) {
    float av[4], bv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) av[i] = As[ty + 16 * i][t];
#pragma unroll
    for (int j = 0; j < 4; ++j) bv[j] = Bs[tx + 16 * j][t];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = i0 + ty + 16 * i;
    if (r >= j0) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = c0 + tx + 16 * j;
      if (col < a.d) a.R[(row0 + r) * a.d + col] -= acc[i][j];
    }
  }
}

// V_c <- solution for the problems whose factorisation succeeded and is finite.
__global__ void __launch_bounds__(256) k_chol_store(CholArgs a, float *Vc) {
  const int b = blockIdx.x;
  if (a.dead[b]) return;
  const int64_t n = (int64_t)kdim(a, b) * a.d;
  const float *X = a.R + a.c_off[b] * a.d;
  bool finite = true;
  for (int64_t e = threadIdx.x; e < n; e += blockDim.x) finite &= isfinite(X[e]);
  finite = __syncthreads_and(finite);
  if (!finite) {
    if (threadIdx.x == 0) a.status[b] |= KVS_ST_NONFINITE;
    return;
  }
  float *V = Vc + a.c_off[b] * a.d;
  for (int64_t e = threadIdx.x; e < n; e += blockDim.x) V[e] = X[e];
}

}  // namespace

int launch_chol_solve(const Batch &Bt, float *Vc, int32_t *status, const Work &w) {
  const HostGeom &g = Bt.g;
  const int npanel = (g.max_c + NB - 1) / NB;
  CholArgs a{w.gram, w.R, w.chol_t, npanel, w.dead, status, Bt.b->c_off, (int64_t)g.max_c, g.d};
  KVS_CUDA_TRY(cudaMemsetAsync(w.dead, 0, sizeof(int) * g.B, Bt.st));
  const int ndc = (g.d + NB - 1) / NB;
  for (int p = 0; p < npanel; ++p) {
    const int j0 = p * NB;
    k_chol_diag<<<g.B, 256, 0, Bt.st>>>(a, j0);
    KVS_LAUNCH_CHECK("k_chol_diag");
    k_chol_tmul<<<dim3(ndc, g.B), 256, 0, Bt.st>>>(a, j0, 0);
    KVS_LAUNCH_CHECK("k_chol_tmul");
    const int n2 = g.max_c - j0 - NB;
    if (n2 <= 0) continue;
    const int nt = (n2 + NB - 1) / NB;
    k_chol_panel<<<dim3(nt, g.B), 256, 0, Bt.st>>>(a, j0);
    KVS_LAUNCH_CHECK("k_chol_panel");
    k_chol_update<<<dim3(nt * (nt + 1) / 2 + nt * ndc, g.B), 256, 0, Bt.st>>>(a, j0, nt);
    KVS_LAUNCH_CHECK("k_chol_update");
  }
  for (int p = npanel - 1; p >= 0; --p) {
    const int j0 = p * NB;
    k_chol_tmul<<<dim3(ndc, g.B), 256, 0, Bt.st>>>(a, j0, 1);
    KVS_LAUNCH_CHECK("k_chol_tmul");
    if (j0 == 0) continue;
    k_chol_bupdate<<<dim3(ndc, (j0 + NB - 1) / NB, g.B), 256, 0, Bt.st>>>(a, j0);
    KVS_LAUNCH_CHECK("k_chol_bupdate");
  }
  k_chol_store<<<g.B, 256, 0, Bt.st>>>(a, Vc);
  KVS_LAUNCH_CHECK("k_chol_store");
  return KVS_OK;
}

}  // namespace kvs
