// Batched Cholesky factorisation and triangular solves of the ridge normal
// equations (A^T A + lam I) V_c = A^T Y ("KVSculpt: KV Cache Compression as
// Distillation", section 2 "Value Optimization": values in closed form by
// ridge regression).
//
// Right-looking blocked algorithm over panels of NB = 64 columns, float32,
// every problem of the batch advancing together so that all SMs share the work:
//   per panel j:
//     diag    factor the diagonal block G_jj = L_jj L_jj^T in shared memory,
//             keep T_j = L_jj^-1 and forward-solve its rows y_j = T_j r_j
//     panel   L_ij = G_ij T_j^T for the rows below
//     update  G_ik -= L_ij L_kj^T on the trailing lower triangle and
//             r_i -= L_ij y_j on the right-hand sides
//   then one kernel sweeps the panels from the last one: x_j = T_j^T y_j,
//   y_i -= L_ji^T x_j.
// Every 64 x 64 product runs from shared memory with 4 x 4 register tiles and
// 128-bit shared loads.  The factor overwrites the Gram matrix, the forward
// sweep the right-hand sides; the solution goes to a separate buffer and is
// copied to V_c only when finite.  A pivot <= 0 (or non-finite) marks the
// problem KVS_ST_NOT_PD; its V_c is left untouched and its remaining steps
// are skipped.
#include <math.h>

#include "kvs_internal.cuh"

namespace kvs {
namespace {

constexpr int NB = 64;
constexpr int SP = NB + 4;  // shared row stride (floats): 16-byte rows, conflict-free columns
constexpr int DEAD_NOT_PD = 1, DEAD_NONFINITE = 2;

struct CholArgs {
  float *G;              // [sum_c, ld] Gram matrix -> factor (lower triangle)
  float *R;              // [sum_c, d] right-hand sides -> forward-solved rows
  float *X;              // [sum_c, d] solution
  float *T;              // [B, npanel, NB, NB] inverses of the diagonal blocks
  int npanel;
  int *dead;             // [B] DEAD_* bits
  int32_t *status;
  const int64_t *c_off;
  int64_t ld;            // multiple of 4
  int d;                 // 64 or 128
};

__device__ __forceinline__ int kdim(const CholArgs &a, int b) {
  return (int)(a.c_off[b + 1] - a.c_off[b]);
}

__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }

// S[r][c] = M[r0 + r][c0 + c] for r0 + r < rmax, c0 + c < cmax, else 0
// (M row-major with ld a multiple of 4 and c0 a multiple of 4).
__device__ __forceinline__ void load_tile(float (*S)[SP], const float *M, int64_t ld, int r0,
                                          int rmax, int c0, int cmax) {
  for (int e = threadIdx.x; e < NB * NB / 4; e += blockDim.x) {
    const int r = e >> 4, c = (e & 15) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + r < rmax && c0 + c < cmax) {
      v = ld4(M + (int64_t)(r0 + r) * ld + c0 + c);
      const int m = cmax - c0 - c;  // valid lanes of the vector
      if (m < 4) {
        v.w = 0.f;
        if (m < 3) v.z = 0.f;
        if (m < 2) v.y = 0.f;
      }
    }
    *reinterpret_cast<float4 *>(&S[r][c]) = v;
  }
}

// Transposed: S[c][r] = M[r0 + r][c0 + c], same bounds.
__device__ __forceinline__ void load_tile_t(float (*S)[SP], const float *M, int64_t ld, int r0,
                                            int rmax, int c0, int cmax) {
  for (int e = threadIdx.x; e < NB * NB / 4; e += blockDim.x) {
    const int r = e >> 4, c = (e & 15) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + r < rmax && c0 + c < cmax) v = ld4(M + (int64_t)(r0 + r) * ld + c0 + c);
    const int m = cmax - c0 - c;
    S[c][r] = m > 0 ? v.x : 0.f;
    S[c + 1][r] = m > 1 ? v.y : 0.f;
    S[c + 2][r] = m > 2 ? v.z : 0.f;
    S[c + 3][r] = m > 3 ? v.w : 0.f;
  }
}

// acc[i][j] += sum_t A[ty + 16 i][t] * B[tx + 16 j][t], t ascending
__device__ __forceinline__ void mm64(const float (*A)[SP], const float (*B)[SP], float acc[4][4],
                                     int tx, int ty) {
#pragma unroll 2
  for (int t = 0; t < NB; t += 4) {
    float4 av[4], bv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) av[i] = *reinterpret_cast<const float4 *>(&A[ty + 16 * i][t]);
#pragma unroll
    for (int j = 0; j < 4; ++j) bv[j] = *reinterpret_cast<const float4 *>(&B[tx + 16 * j][t]);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float s = acc[i][j];
        s = fmaf(av[i].x, bv[j].x, s);
        s = fmaf(av[i].y, bv[j].y, s);
        s = fmaf(av[i].z, bv[j].z, s);
        acc[i][j] = fmaf(av[i].w, bv[j].w, s);
      }
  }
}

__device__ __forceinline__ void zero_acc(float acc[4][4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
}

// Diagonal block of panel j0: factor in shared memory, keep T_j = L_jj^-1 and
// forward-solve the block's rows of the right-hand sides, y_j = T_j r_j.
__global__ void __launch_bounds__(256) k_chol_diag(CholArgs a, int j0) {
  const int b = blockIdx.x;
  const int k = kdim(a, b);
  if (j0 >= k || a.dead[b]) return;
  const int jb = min(NB, k - j0);
  __shared__ __align__(16) float L[NB][SP];   // the block; later the right-hand side tile
  __shared__ __align__(16) float Ts[NB][SP];  // T_j
  __shared__ float dsq[NB];
  __shared__ int bad;
  float *G = a.G + (a.c_off[b] + j0) * a.ld + j0;
  const int tid = threadIdx.x;
  if (tid == 0) bad = 0;
  load_tile(L, G, a.ld, 0, jb, 0, jb);
  for (int e = tid; e < NB * SP; e += blockDim.x) (&Ts[0][0])[e] = 0.f;
  __syncthreads();
  // Unnormalised elimination: after step c, column c holds l_ic * sqrt(p_c) and
  // L[c][c] = p_c, the pivot; the trailing block loses l_i l_j^T = L_ic L_jc / p_c.
  // Thread (i, q) owns row i = tid / 4 at the columns j = q + 4 m.
  {
    const int i = tid >> 2, q = tid & 3;
    for (int c = 0; c < jb - 1; ++c) {
      if (i > c && i < jb) {
        const float lic = L[i][c] / L[c][c];
        const int m0 = (c + 1 - q + 3) >> 2;  // first m with q + 4 m > c
#pragma unroll 4
        for (int m = m0; m < 16; ++m) {
          const int j = q + 4 * m;
          if (j > i) break;
          L[i][j] = fmaf(-lic, L[j][c], L[i][j]);
        }
      }
      __syncthreads();
    }
  }
  if (tid < jb) {
    const float p = L[tid][tid];
    if (!(p > 0.f) || !isfinite(p)) atomicOr(&bad, 1);
    dsq[tid] = sqrtf(fmaxf(p, 1e-30f));
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) {
      a.status[b] |= KVS_ST_NOT_PD;
      a.dead[b] = DEAD_NOT_PD;
    }
    return;
  }
  for (int e = tid; e < jb * jb; e += blockDim.x) {
    const int r = e / jb, c = e % jb;
    if (c < r) L[r][c] /= dsq[c];
    else if (c == r) L[r][c] = dsq[c];
  }
  __syncthreads();
  // T = L^-1 column by column: warp w owns columns 8w .. 8w+7, four lanes per
  // column split each row's dot product; T[i][cc] = -(sum_t L[i][t] T[t][cc]) / L[i][i].
  if (tid < jb) Ts[tid][tid] = 1.f / L[tid][tid];
  __syncthreads();
  {
    const int warp = tid >> 5, lane = tid & 31;
    const int cc = warp * 8 + (lane >> 2), q = lane & 3;
    for (int i = 1; i < jb; ++i) {
      float s = 0.f;
      if (i > cc)
        for (int t = cc + q; t < i; t += 4) s = fmaf(L[i][t], Ts[t][cc], s);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (i > cc && q == 0) Ts[i][cc] = -s * Ts[i][i];
      __syncwarp();
    }
  }
  __syncthreads();
  float *Tg = a.T + ((int64_t)b * a.npanel + j0 / NB) * NB * NB;
  for (int e = tid; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    if (r < jb && c <= r) G[(int64_t)r * a.ld + c] = L[r][c];
    Tg[e] = Ts[r][c];
  }
  __syncthreads();
  // y_j = T_j r_j, 64 right-hand-side columns at a time (the tile reuses L)
  const int tx = tid & 15, ty = tid >> 4;
  float *R = a.R + (a.c_off[b] + j0) * a.d;
  for (int c0 = 0; c0 < a.d; c0 += NB) {
    load_tile_t(L, R, a.d, 0, jb, c0, a.d);  // L[col][t] = r[t][c0 + col]
    __syncthreads();
    float acc[4][4];
    zero_acc(acc);
    mm64(Ts, L, acc, tx, ty);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty + 16 * i;
      if (r >= jb) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) R[(int64_t)r * a.d + c0 + tx + 16 * j] = acc[i][j];
    }
    __syncthreads();
  }
}

// L_ij = G_ij T_j^T for 64 rows of the panel below the diagonal block.
__global__ void __launch_bounds__(256) k_chol_panel(CholArgs a, int j0) {
  const int b = blockIdx.y;
  const int k = kdim(a, b);
  if (j0 >= k || a.dead[b]) return;
  const int jb = min(NB, k - j0);
  const int i0 = j0 + jb + blockIdx.x * NB;
  if (i0 >= k) return;
  __shared__ __align__(16) float Ar[NB][SP];
  __shared__ __align__(16) float Ts[NB][SP];
  const int tid = threadIdx.x;
  const int64_t row0 = a.c_off[b];
  load_tile(Ar, a.G + row0 * a.ld, a.ld, i0, k, j0, j0 + jb);
  const float *Tg = a.T + ((int64_t)b * a.npanel + j0 / NB) * NB * NB;
  for (int e = tid; e < NB * NB / 4; e += blockDim.x) {
    const int r = e >> 4, c = (e & 15) * 4;
    *reinterpret_cast<float4 *>(&Ts[r][c]) = ld4(Tg + r * NB + c);
  }
  __syncthreads();
  const int tx = tid & 15, ty = tid >> 4;
  float acc[4][4];
  zero_acc(acc);
  mm64(Ar, Ts, acc, tx, ty);  // sum_t G[r][t] T[col][t]
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = i0 + ty + 16 * i;
    if (r >= k) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = tx + 16 * j;
      if (c < jb) a.G[(row0 + r) * a.ld + j0 + c] = acc[i][j];
    }
  }
}

// Trailing update: tiles (ti >= tj) of G_ik -= L_i L_k^T, and tiles of
// r_i -= L_i y_j (columns of R in chunks of 64), 64 x 64 outputs per CTA.
__global__ void __launch_bounds__(256) k_chol_update(CholArgs a, int j0) {
  const int b = blockIdx.y;
  const int k = kdim(a, b);
  if (j0 >= k || a.dead[b]) return;
  const int jb = min(NB, k - j0);
  const int s0 = j0 + jb;
  const int n2 = k - s0;
  if (n2 <= 0) return;
  const int nt = (n2 + NB - 1) / NB;
  const int ntri = nt * (nt + 1) / 2;
  const int ndc = a.d / NB;
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
  __shared__ __align__(16) float As[NB][SP];  // L_i panel rows, [row][c]
  __shared__ __align__(16) float Bs[NB][SP];  // L_k panel rows [row][c], or y_j as [col][c]
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int64_t row0 = a.c_off[b];
  const int ri = s0 + ti * NB;
  // the outputs' current values first: their loads overlap the tile loads
  float cur[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ri + ty + 16 * i;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      cur[i][j] = 0.f;
      if (r >= k) continue;
      if (!rhs) {
        const int cc = s0 + tj * NB + tx + 16 * j;
        if (cc <= r) cur[i][j] = a.G[(row0 + r) * a.ld + cc];
      } else {
        cur[i][j] = a.R[(row0 + r) * a.d + tj * NB + tx + 16 * j];
      }
    }
  }
  load_tile(As, a.G + row0 * a.ld, a.ld, ri, k, j0, j0 + jb);
  if (!rhs)
    load_tile(Bs, a.G + row0 * a.ld, a.ld, s0 + tj * NB, k, j0, j0 + jb);
  else
    load_tile_t(Bs, a.R + row0 * a.d, a.d, j0, j0 + jb, tj * NB, a.d);
  __syncthreads();
  float acc[4][4];
  zero_acc(acc);
  mm64(As, Bs, acc, tx, ty);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ri + ty + 16 * i;
    if (r >= k) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (!rhs) {
        const int cc = s0 + tj * NB + tx + 16 * j;
        if (cc <= r) a.G[(row0 + r) * a.ld + cc] = cur[i][j] - acc[i][j];
      } else {
        a.R[(row0 + r) * a.d + tj * NB + tx + 16 * j] = cur[i][j] - acc[i][j];
      }
    }
  }
}

// The whole backward sweep for 64 right-hand-side columns of one problem, from
// the last panel to the first: x_j = T_j^T y_j (stored, checked finite), then
// y_i -= L_ji^T x_j for every i < j.  The next L_ji tile is fetched into
// registers while the current one is multiplied (two shared tiles in turn).
constexpr int BWD_SMEM = 3 * NB * SP * 4;

__global__ void __launch_bounds__(256) k_chol_backward(CholArgs a) {
  extern __shared__ __align__(16) float bsm[];
  float (*Xs)[SP] = reinterpret_cast<float (*)[SP]>(bsm);
  float (*At[2])[SP] = {reinterpret_cast<float (*)[SP]>(bsm + NB * SP),
                        reinterpret_cast<float (*)[SP]>(bsm + 2 * NB * SP)};
  const int b = blockIdx.y;
  const int k = kdim(a, b);
  if (a.dead[b]) return;
  const int c0 = blockIdx.x * NB;
  const int np = (k + NB - 1) / NB;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int64_t row0 = a.c_off[b];
  const float *G = a.G + row0 * a.ld;
  float *R = a.R + row0 * a.d;
  for (int p = np - 1; p >= 0; --p) {
    const int j0 = p * NB, jb = min(NB, k - j0);
    const float *Tg = a.T + ((int64_t)b * a.npanel + p) * NB * NB;
    load_tile_t(At[0], Tg, NB, 0, NB, 0, NB);           // At[r][t] = T[t][r]
    load_tile_t(Xs, R, a.d, j0, j0 + jb, c0, a.d);      // Xs[col][t] = y[j0 + t][c0 + col]
    __syncthreads();
    float acc[4][4];
    zero_acc(acc);
    mm64(At[0], Xs, acc, tx, ty);                       // x[r][col]
    __syncthreads();
    bool fin = true;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty + 16 * i;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        Xs[tx + 16 * j][r] = acc[i][j];  // as the B operand of the updates
        if (r < jb) {
          a.X[(row0 + j0 + r) * a.d + c0 + tx + 16 * j] = acc[i][j];
          fin &= isfinite(acc[i][j]);
        }
      }
    }
    if (!fin) atomicOr(&a.dead[b], DEAD_NONFINITE);
    if (p == 0) break;
    // y_i -= L_ji^T x_j, with At[r][t] = L[j0 + t][64 i + r]
    float4 pf[4];
    auto fetch = [&](int i) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = tid + 256 * u, r = e >> 4, c = (e & 15) * 4;
        pf[u] = r < jb ? ld4(G + (int64_t)(j0 + r) * a.ld + NB * i + c)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    };
    auto place = [&](float (*S)[SP]) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = tid + 256 * u, r = e >> 4, c = (e & 15) * 4;
        S[c][r] = pf[u].x;
        S[c + 1][r] = pf[u].y;
        S[c + 2][r] = pf[u].z;
        S[c + 3][r] = pf[u].w;
      }
    };
    fetch(0);
    place(At[0]);
    __syncthreads();
    for (int i = 0; i < p; ++i) {
      float cur[4][4];
#pragma unroll
      for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
          cur[ii][jj] = R[(int64_t)(NB * i + ty + 16 * ii) * a.d + c0 + tx + 16 * jj];
      if (i + 1 < p) fetch(i + 1);
      zero_acc(acc);
      mm64(At[i & 1], Xs, acc, tx, ty);
#pragma unroll
      for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
          R[(int64_t)(NB * i + ty + 16 * ii) * a.d + c0 + tx + 16 * jj] = cur[ii][jj] - acc[ii][jj];
      if (i + 1 < p) place(At[(i + 1) & 1]);
      __syncthreads();
    }
  }
}

// V_c <- solution for the problems whose factorisation succeeded and whose
// solution is finite; the others keep V_c and get their status bit.
__global__ void __launch_bounds__(256) k_chol_store(CholArgs a, float *Vc) {
  const int b = blockIdx.y;
  const int dead = a.dead[b];
  if (dead) {
    if (blockIdx.x == 0 && threadIdx.x == 0 && (dead & DEAD_NONFINITE))
      a.status[b] |= KVS_ST_NONFINITE;
    return;
  }
  const int64_t n4 = (int64_t)kdim(a, b) * a.d / 4;
  const float4 *X = reinterpret_cast<const float4 *>(a.X + a.c_off[b] * a.d);
  float4 *V = reinterpret_cast<float4 *>(Vc + a.c_off[b] * a.d);
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n4;
       e += (int64_t)gridDim.x * blockDim.x)
    V[e] = X[e];
}

}  // namespace

int launch_chol_solve(const Batch &Bt, float *Vc, int32_t *status, const Work &w) {
  const HostGeom &g = Bt.g;
  const int npanel = (g.max_c + NB - 1) / NB;
  CholArgs a{w.gram, w.R, w.X, w.chol_t, npanel, w.dead, status, Bt.b->c_off, g.ld_g, g.d};
  KVS_CUDA_TRY(set_smem_once(k_chol_backward, BWD_SMEM));
  KVS_CUDA_TRY(cudaMemsetAsync(w.dead, 0, sizeof(int) * g.B, Bt.st));
  const int ndc = g.d / NB;
  for (int p = 0; p < npanel; ++p) {
    const int j0 = p * NB;
    k_chol_diag<<<g.B, 256, 0, Bt.st>>>(a, j0);
    KVS_LAUNCH_CHECK("k_chol_diag");
    const int n2 = g.max_c - j0 - NB;
    if (n2 <= 0) continue;
    const int nt = (n2 + NB - 1) / NB;
    k_chol_panel<<<dim3(nt, g.B), 256, 0, Bt.st>>>(a, j0);
    KVS_LAUNCH_CHECK("k_chol_panel");
    k_chol_update<<<dim3(nt * (nt + 1) / 2 + nt * ndc, g.B), 256, 0, Bt.st>>>(a, j0);
    KVS_LAUNCH_CHECK("k_chol_update");
  }
  k_chol_backward<<<dim3(ndc, g.B), 256, BWD_SMEM, Bt.st>>>(a);
  KVS_LAUNCH_CHECK("k_chol_backward");
  const int64_t n4 = (int64_t)g.max_c * g.d / 4;
  const int blocks = (int)std::min<int64_t>((n4 + 255) / 256, 64);
  k_chol_store<<<dim3(blocks, g.B), 256, 0, Bt.st>>>(a, Vc);
  KVS_LAUNCH_CHECK("k_chol_store");
  return KVS_OK;
}

}  // namespace kvs
