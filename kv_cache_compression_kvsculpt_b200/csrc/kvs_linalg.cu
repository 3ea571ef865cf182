// Batched Cholesky factorisation and triangular solves of the ridge normal
// equations (A^T A + lam I) V_c = A^T Y ("KVSculpt: KV Cache Compression as
// Distillation", section 2 "Value Optimization": values in closed form by
// ridge regression).
//
// Right-looking blocked algorithm over panels of NB = 64 columns, float32,
// every problem of the batch advancing together so that all SMs share the work:
//   per panel j:
//     diag    apply panel j-1's update to the diagonal block and its
//             right-hand-side rows, factor G_jj = L_jj L_jj^T in shared memory,
//             keep T_j = L_jj^-1 and forward-solve its rows y_j = T_j r_j
//     panel   apply panel j-1's update to the column below, L_ij = G_ij T_j^T
//     update  G_ik -= L_ij L_kj^T on the trailing lower triangle from column
//             block j+2 on and r_i -= L_ij y_j on those right-hand-side rows,
//             on tensor cores (kvs_chol_tc.cu) from tf32 hi / lo splits of L_ij
//             and y_j that the panel and diagonal-block kernels write beside
//             their results
//   then one kernel sweeps the panels from the last one: x_j = T_j^T y_j,
//   y_i -= L_ji^T x_j.
// Look-ahead: diag and panel run on a second stream, and the update of panel j
// on the caller's stream beside diag and panel of j+1, which need only the
// update of panel j-1 (the splits alternate between two buffers by panel parity,
// so the next panel never overwrites the operands of the running update).
// The 64 x 64 x 64 products of the diagonal block, the panel and the backward
// sweep run from shared memory with both operands stored
// contraction-index-major (S[t][row]): each thread owns a 4 x 4 output block
// and forms a rank-1 update from two 128-bit loads per t.  The diagonal block
// is factored 16 columns at a time: one warp factors and inverts the 16 x 16
// pivot block in registers, then all threads apply it to the rows below and to
// the trailing block, and T_j is assembled from the four 16 x 16 inverses.  The
// factor overwrites the Gram matrix (lower triangle; the upper one is scratch),
// the forward sweep the right-hand sides; the solution goes to a separate
// buffer and is copied to V_c only when finite.  A pivot <= 0 (or non-finite)
// marks the problem KVS_ST_NOT_PD; its V_c is left untouched and its remaining
// steps are skipped.
#include <math.h>

#include "kvs_attn_tc.cuh"

namespace kvs {
namespace {

constexpr int NB = 64;
constexpr int SP = NB + 4;  // shared row stride (floats): 16-byte rows, offset banks
constexpr int DEAD_NOT_PD = 1, DEAD_NONFINITE = 2;
constexpr unsigned FULL = 0xffffffffu;

struct CholArgs {
  float *G;              // [sum_c, ld] Gram matrix -> factor (lower triangle)
  float *R;              // [sum_c, d] right-hand sides -> forward-solved rows
  float *X;              // [sum_c, d] solution
  float *Tt;             // [B, npanel, NB, NB] transposes of the diagonal-block inverses
  float *P;              // [2, 2, sum_c, NB] tf32 hi / lo of the panel's factor rows
  float *Y;              // [2, 2, B d, NB] tf32 hi / lo of the forward-solved rows, transposed
  int64_t sum_c;
  int B;
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

// x = hi + lo with hi = x rounded toward zero to tf32 (low 13 mantissa bits
// cleared); lo is exact in fp32.
__device__ __forceinline__ void split_tf32(float x, float &hi, float &lo) {
  hi = __uint_as_float(__float_as_uint(x) & 0xffffe000u);
  lo = x - hi;
}

__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ void st4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }

// M[r][c0 + c .. c0 + c + 3] with the lanes at or past cmax zeroed (c0 + c < cmax;
// M row-major with ld a multiple of 4 and c0 + c a multiple of 4).
__device__ __forceinline__ float4 ld4m(const float *M, int64_t ld, int r, int c, int cmax) {
  float4 v = ld4(M + (int64_t)r * ld + c);
  const int m = cmax - c;
  if (m < 4) {
    v.w = 0.f;
    if (m < 3) v.z = 0.f;
    if (m < 2) v.y = 0.f;
  }
  return v;
}

// S[r][c] = M[r0 + r][c0 + c] for r0 + r < rmax, c0 + c < cmax, else 0.
__device__ __forceinline__ void load_d(float (*S)[SP], const float *M, int64_t ld, int r0,
                                       int rmax, int c0, int cmax) {
  for (int e = threadIdx.x; e < NB * NB / 4; e += blockDim.x) {
    const int r = e >> 4, c = (e & 15) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + r < rmax && c0 + c < cmax) v = ld4m(M, ld, r0 + r, c0 + c, cmax);
    st4(&S[r][c], v);
  }
}

// Transposed: S[c][r] = M[r0 + r][c0 + c], same bounds.  Lanes take consecutive
// rows, so the shared-memory stores of a warp hit 32 consecutive words.
__device__ __forceinline__ void load_t(float (*S)[SP], const float *M, int64_t ld, int r0,
                                       int rmax, int c0, int cmax) {
  for (int e = threadIdx.x; e < NB * NB / 4; e += blockDim.x) {
    const int r = e & (NB - 1), c = (e >> 6) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + r < rmax && c0 + c < cmax) v = ld4m(M, ld, r0 + r, c0 + c, cmax);
    S[c][r] = v.x;
    S[c + 1][r] = v.y;
    S[c + 2][r] = v.z;
    S[c + 3][r] = v.w;
  }
}

// acc[i][j] += sum_t A[t][4 ty + i] * B[t][4 tx + j], t ascending
__device__ __forceinline__ void mmk(const float (*A)[SP], const float (*B)[SP], float acc[4][4],
                                    int tx, int ty) {
#pragma unroll 8
  for (int t = 0; t < NB; ++t) {
    const float4 av = ld4(&A[t][4 * ty]);
    const float4 bv = ld4(&B[t][4 * tx]);
    const float ai[4] = {av.x, av.y, av.z, av.w};
    const float bj[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(ai[i], bj[j], acc[i][j]);
  }
}

__device__ __forceinline__ void zero_acc(float acc[4][4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
}

// Warp step of the diagonal-block factorisation: lane r (and its mirror r + 16)
// holds row r of the 16 x 16 pivot block at (c0, c0) (rows of the padding past jb
// read as identity rows), factors it, inverts the factor and writes both back.
// Returns true when a pivot was not positive and finite.
__device__ __forceinline__ bool factor16(float (*L)[SP], float (*Ts)[SP], int c0, int jb,
                                         int lane) {
  const int r = lane & 15, gr = c0 + r;
  float av[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    float v = j <= r ? L[gr][c0 + j] : 0.f;
    if (gr >= jb) v = j == r ? 1.f : 0.f;
    av[j] = v;
  }
  // unblocked Cholesky, column c: pivot from lane c, scale, rank-1 update
  bool bad = false;
  float invd = 1.f;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const float p = __shfl_sync(FULL, av[c], c);
    bad |= !(p > 0.f) || !isfinite(p);
    const float dc = sqrtf(fmaxf(p, 1e-30f));
    const float inv = 1.f / dc;
    const float l = r == c ? dc : av[c] * inv;
    if (r == c) invd = inv;
    av[c] = l;
#pragma unroll
    for (int j = c + 1; j < 16; ++j) av[j] = fmaf(-l, __shfl_sync(FULL, l, j), av[j]);
  }
  // T = L^-1 row by row: lane r accumulates -sum_u L[r][u] T[u][j] over the rows
  // u < r as lane u finalises them, then scales by 1 / L[r][r]
  float tv[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) tv[j] = 0.f;
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    if (r == u) {
#pragma unroll
      for (int j = 0; j < u; ++j) tv[j] *= invd;
      tv[u] = invd;
    }
#pragma unroll
    for (int j = 0; j <= u; ++j) {
      const float tu = __shfl_sync(FULL, tv[j], u);
      if (r > u) tv[j] = fmaf(-av[u], tu, tv[j]);
    }
  }
  if (lane < 16) {
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j <= r) {
        L[gr][c0 + j] = av[j];
        Ts[gr][c0 + j] = tv[j];
      }
  }
  return bad;
}

// Diagonal block of panel j0: factor in shared memory, keep T_j = L_jj^-1 (stored
// transposed) and forward-solve the block's rows of the right-hand sides, y_j = T_j r_j.
// Rows past jb (the last panel of a problem whose k is not a multiple of 64) are
// factored as identity rows, so T_j is the identity there.
// The previous panel's update of this block and of its right-hand-side rows
// (G_jj -= L_j,j-1 L_j,j-1^T, r_j -= L_j,j-1 y_j-1) is applied here first, in
// fp32; the trailing update leaves those to this kernel, so that it is not on
// the path from one panel to the next.
// Every input tile is requested at entry (asynchronous copies for the row-major
// ones), and the block's right-hand-side rows stay in shared memory from the
// update through the forward solve.
constexpr int DIAG_SMEM = 7 * NB * SP * 4;

// 16-byte asynchronous copy global -> shared; bytes past src_bytes are zero.
__device__ __forceinline__ void cp16(void *dst, const void *src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src), "r"(src_bytes)
               : "memory");
}

// S[r][c] = M[r0 + r][c0 + c] by asynchronous copies, zero for r0 + r >= rmax or
// c0 + c >= cmax (M row-major, ld and c0 multiples of 4).
__device__ __forceinline__ void cp_tile(float (*S)[SP], const float *M, int64_t ld, int r0,
                                        int rmax, int c0, int cmax) {
  for (int e = threadIdx.x; e < NB * NB / 4; e += blockDim.x) {
    const int r = e >> 4, c = (e & 15) * 4;
    const int n = (r0 + r < rmax) ? max(0, min(4, cmax - (c0 + c))) : 0;
    cp16(&S[r][c], M + (int64_t)(n > 0 ? r0 + r : 0) * ld + (n > 0 ? c0 + c : 0), 4 * n);
  }
}

__global__ void __launch_bounds__(256) k_chol_diag(CholArgs a, int j0) {
  const int b = blockIdx.x;
  const int k = kdim(a, b);
  if (j0 >= k || a.dead[b]) return;
  const int jb = min(NB, k - j0);
  extern __shared__ __align__(16) float dsm[];
  float (*L)[SP] = reinterpret_cast<float (*)[SP]>(dsm);             // the block; then T_j^T
  float (*Ts)[SP] = reinterpret_cast<float (*)[SP]>(dsm + NB * SP);  // T_j
  float (*Xs)[SP] = reinterpret_cast<float (*)[SP]>(dsm + 2 * NB * SP);
  // right-hand-side rows of this block (r_j, then y_j) and of the previous one
  // (y_j-1), 64 columns per tile
  float (*Rb[2])[SP] = {reinterpret_cast<float (*)[SP]>(dsm + 3 * NB * SP),
                        reinterpret_cast<float (*)[SP]>(dsm + 4 * NB * SP)};
  float (*Yp[2])[SP] = {reinterpret_cast<float (*)[SP]>(dsm + 5 * NB * SP),
                        reinterpret_cast<float (*)[SP]>(dsm + 6 * NB * SP)};
  __shared__ int bad;
  const int64_t row0 = a.c_off[b];
  float *G = a.G + (row0 + j0) * a.ld + j0;
  const float *R = a.R + row0 * a.d;
  const int ndc = a.d / NB;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tx = tid & 15, ty = tid >> 4;
  if (tid == 0) bad = 0;
  cp_tile(L, G, a.ld, 0, jb, 0, jb);
  for (int ch = 0; ch < ndc; ++ch) {
    cp_tile(Rb[ch], R, a.d, j0, k, ch * NB, a.d);
    if (j0 > 0) cp_tile(Yp[ch], R, a.d, j0 - NB, j0, ch * NB, a.d);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  // Xs[t][r] = L_j,j-1[r][t]: the previous panel's factor rows of this block
  if (j0 > 0) load_t(Xs, a.G + row0 * a.ld, a.ld, j0, k, j0 - NB, j0);
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  if (j0 > 0) {
    // the previous panel's update: G_jj -= L_j,j-1 L_j,j-1^T, r_j -= L_j,j-1 y_j-1
    float acc[4][4];
    zero_acc(acc);
    mmk(Xs, Xs, acc, tx, ty);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) L[4 * ty + i][4 * tx + j] -= acc[i][j];
    for (int ch = 0; ch < ndc; ++ch) {
      zero_acc(acc);
      mmk(Xs, Yp[ch], acc, tx, ty);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) Rb[ch][4 * ty + i][4 * tx + j] -= acc[i][j];
    }
  }
  for (int e = tid; e < NB * SP; e += blockDim.x) (&Ts[0][0])[e] = 0.f;
  __syncthreads();
#pragma unroll 1
  for (int c0 = 0; c0 < NB; c0 += 16) {
    if (warp == 0 && factor16(L, Ts, c0, jb, lane) && lane == 0) bad = 1;
    __syncthreads();
    const int m = NB - c0 - 16;  // rows below the pivot block
    if (m == 0) break;
    // L[i][c0 ..] = A[i][c0 ..] T_kk^T for the rows below: four threads per row
    // (one warp holds all four), four columns each
    {
      const int i = c0 + 16 + (tid >> 2), q = tid & 3;
      const bool act = (tid >> 2) < m;
      float4 ar[4];
      if (act)
#pragma unroll
        for (int u = 0; u < 4; ++u) ar[u] = ld4(&L[i][c0 + 4 * u]);
      __syncwarp();
      if (act) {
        float o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float *tr = &Ts[c0 + 4 * q + e][c0];  // row of T_kk (zero past the diagonal)
          float s = 0.f;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float4 t4 = ld4(tr + 4 * u);
            s = fmaf(ar[u].x, t4.x, s);
            s = fmaf(ar[u].y, t4.y, s);
            s = fmaf(ar[u].z, t4.z, s);
            s = fmaf(ar[u].w, t4.w, s);
          }
          o[e] = s;
        }
        st4(&L[i][c0 + 4 * q], make_float4(o[0], o[1], o[2], o[3]));
      }
    }
    __syncthreads();
    // trailing block: A[i][j] -= sum_t L[i][c0 + t] L[j][c0 + t], c0 + 16 <= j <= i,
    // in groups of four columns
    {
      const int ng = m / 4, s0 = c0 + 16;
      for (int e = tid; e < m * ng; e += blockDim.x) {
        const int i = s0 + e / ng, j4 = s0 + (e % ng) * 4;
        if (j4 > i) continue;
        float4 li[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) li[u] = ld4(&L[i][c0 + 4 * u]);
        float acc[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          float s = 0.f;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float4 lj = ld4(&L[j4 + jj][c0 + 4 * u]);
            s = fmaf(li[u].x, lj.x, s);
            s = fmaf(li[u].y, lj.y, s);
            s = fmaf(li[u].z, lj.z, s);
            s = fmaf(li[u].w, lj.w, s);
          }
          acc[jj] = s;
        }
        float4 v = ld4(&L[i][j4]);
        v.x -= acc[0];
        v.y -= acc[1];
        v.z -= acc[2];
        v.w -= acc[3];
        st4(&L[i][j4], v);
      }
    }
    __syncthreads();
  }
  if (bad) {
    if (tid == 0) {
      a.status[b] |= KVS_ST_NOT_PD;
      a.dead[b] = DEAD_NOT_PD;
    }
    return;
  }
  // T_j from the four 16 x 16 inverses T_k on its diagonal, by 2 x 2 blocks:
  // [[T1, 0], [L21, L22]]^-1 has lower-left block -T2 L21 T1.  Products go
  // through the upper-right quadrant of Ts (zero in T_j) as scratch.
  {
    // 16 x 16 level, both 32 x 32 halves q: W_q = L[32q+16 ..][32q ..] T_2q
    const int q = tid >> 7, i = (tid >> 3) & 15, j2 = (tid & 7) * 2;
    const int o = 32 * q;
    float *W = &Ts[16 * q][32 + 16 * q];  // 16 x 16 scratch, row stride SP
    {
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        const float l = L[o + 16 + i][o + t];
        s0 = fmaf(l, Ts[o + t][o + j2], s0);
        s1 = fmaf(l, Ts[o + t][o + j2 + 1], s1);
      }
      W[i * SP + j2] = s0;
      W[i * SP + j2 + 1] = s1;
    }
    __syncthreads();
    {
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        const float tt = Ts[o + 16 + i][o + 16 + t];
        s0 = fmaf(tt, W[t * SP + j2], s0);
        s1 = fmaf(tt, W[t * SP + j2 + 1], s1);
      }
      Ts[o + 16 + i][o + j2] = -s0;
      Ts[o + 16 + i][o + j2 + 1] = -s1;
    }
    __syncthreads();
    // 32 x 32 level: W = L[32 ..][0 .. 32) T1 into the upper-right quadrant, then
    // the lower-left quadrant = -T2 W
    const int i2 = tid >> 3, j4 = (tid & 7) * 4;
    {
      float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
      for (int t = 0; t < 32; ++t) {
        const float l = L[32 + i2][t];
        const float4 tt = ld4(&Ts[t][j4]);
        s[0] = fmaf(l, tt.x, s[0]);
        s[1] = fmaf(l, tt.y, s[1]);
        s[2] = fmaf(l, tt.z, s[2]);
        s[3] = fmaf(l, tt.w, s[3]);
      }
      st4(&Ts[i2][32 + j4], make_float4(s[0], s[1], s[2], s[3]));
    }
    __syncthreads();
    {
      float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
      for (int t = 0; t < 32; ++t) {
        const float tt = Ts[32 + i2][32 + t];
        const float4 w = ld4(&Ts[t][32 + j4]);
        s[0] = fmaf(tt, w.x, s[0]);
        s[1] = fmaf(tt, w.y, s[1]);
        s[2] = fmaf(tt, w.z, s[2]);
        s[3] = fmaf(tt, w.w, s[3]);
      }
      st4(&Ts[32 + i2][j4], make_float4(-s[0], -s[1], -s[2], -s[3]));
    }
    __syncthreads();
    st4(&Ts[i2][32 + j4], make_float4(0.f, 0.f, 0.f, 0.f));
  }
  // the factor's lower triangle back to G
  for (int e = tid; e < NB * NB; e += blockDim.x) {
    const int r = e >> 6, c = e & (NB - 1);
    if (r < jb && c <= r) G[(int64_t)r * a.ld + c] = L[r][c];
  }
  __syncthreads();
  // T_j^T to global and into L (the A operand of the forward solve)
  float *Tg = a.Tt + ((int64_t)b * a.npanel + j0 / NB) * NB * NB;
  for (int e = tid; e < NB * NB; e += blockDim.x) {
    const int c = e >> 6, r = e & (NB - 1);
    const float v = Ts[r][c];
    Tg[e] = v;
    L[c][r] = v;
  }
  __syncthreads();
  // y_j = T_j r_j, 64 right-hand-side columns at a time
  float *Rj = a.R + (row0 + j0) * a.d;
  const int par = (j0 / NB) & 1;
  float *Yh = a.Y + ((int64_t)(par * 2) * a.B * a.d + (int64_t)b * a.d) * NB;
  float *Yl = Yh + (int64_t)a.B * a.d * NB;
  for (int ch = 0; ch < ndc; ++ch) {
    const int c0 = ch * NB;
    float acc[4][4];
    zero_acc(acc);
    mmk(L, Rb[ch], acc, tx, ty);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 4 * ty + i;
      if (r < jb)
        st4(Rj + (int64_t)r * a.d + c0 + 4 * tx, make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]));
    }
    // the trailing update's B operand: Y[par][h][b d + c][t] = split of y[t][c]
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float h[4], l[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) split_tf32(acc[i][j], h[i], l[i]);
      const int64_t o = (int64_t)(c0 + 4 * tx + j) * NB + 4 * ty;
      st4(Yh + o, make_float4(h[0], h[1], h[2], h[3]));
      st4(Yl + o, make_float4(l[0], l[1], l[2], l[3]));
    }
  }
}

// L_ij = G_ij T_j^T for 64 rows of the panel below the diagonal block.
// The previous panel's update of these rows of the column block,
// G_ij -= L_i,j-1 L_j,j-1^T, is applied here first (fp32), as in the diagonal block.
__global__ void __launch_bounds__(256) k_chol_panel(CholArgs a, int j0) {
  const int b = blockIdx.y;
  const int k = kdim(a, b);
  if (j0 + NB >= k || a.dead[b]) return;  // rows below exist only after a full block
  const int i0 = j0 + NB + blockIdx.x * NB;
  if (i0 >= k) return;
  __shared__ __align__(16) float As[NB][SP];  // As[t][r] = G[i0 + r][j0 + t]
  __shared__ __align__(16) float Bs[NB][SP];  // Bs[t][c] = T[c][t]
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int64_t row0 = a.c_off[b];
  float acc[4][4];
  if (j0 > 0) {
    // acc[r][t] = sum_u L[i0 + r][j0 - 64 + u] L[j0 + t][j0 - 64 + u]
    load_t(As, a.G + row0 * a.ld, a.ld, i0, k, j0 - NB, j0);
    load_t(Bs, a.G + row0 * a.ld, a.ld, j0, k, j0 - NB, j0);
    __syncthreads();
    zero_acc(acc);
    mmk(As, Bs, acc, tx, ty);
    __syncthreads();
  }
  load_t(As, a.G + row0 * a.ld, a.ld, i0, k, j0, j0 + NB);
  load_d(Bs, a.Tt + ((int64_t)b * a.npanel + j0 / NB) * NB * NB, NB, 0, NB, 0, NB);
  __syncthreads();
  if (j0 > 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) As[4 * tx + j][4 * ty + i] -= acc[i][j];
    __syncthreads();
  }
  zero_acc(acc);
  mmk(As, Bs, acc, tx, ty);
  const int par = (j0 / NB) & 1;
  float *Ph = a.P + ((int64_t)(par * 2) * a.sum_c + row0) * NB;
  float *Pl = Ph + a.sum_c * NB;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = i0 + 4 * ty + i;
    if (r < k) {
      st4(a.G + (row0 + r) * a.ld + j0 + 4 * tx,
          make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]));
      float h[4], l[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) split_tf32(acc[i][j], h[j], l[j]);
      st4(Ph + (int64_t)r * NB + 4 * tx, make_float4(h[0], h[1], h[2], h[3]));
      st4(Pl + (int64_t)r * NB + 4 * tx, make_float4(l[0], l[1], l[2], l[3]));
    }
  }
}

// The whole backward sweep for 64 right-hand-side columns of one problem, from
// the last panel to the first: x_j = T_j^T y_j (stored, checked finite), then
// y_i -= L_ji^T x_j for every i < j.  Two groups of 256 threads take the
// independent products of a step in turn (group g the rows i = g (mod 2)), so
// that sixteen warps hide the shared-memory latency of the 64 x 64 x 64
// products; each group fetches its next L_ji tile into registers while it
// multiplies the current one (two shared tiles per group in turn).
constexpr int BWD_SMEM = 5 * NB * SP * 4;

__global__ void __launch_bounds__(512, 1) k_chol_backward(CholArgs a) {
  extern __shared__ __align__(16) float bsm[];
  const int tid = threadIdx.x, grp = tid >> 8, tl = tid & 255;
  float (*Xs)[SP] = reinterpret_cast<float (*)[SP]>(bsm);
  float (*At[2])[SP] = {reinterpret_cast<float (*)[SP]>(bsm + (1 + 2 * grp) * NB * SP),
                        reinterpret_cast<float (*)[SP]>(bsm + (2 + 2 * grp) * NB * SP)};
  float (*Ts)[SP] = reinterpret_cast<float (*)[SP]>(bsm + NB * SP);  // group 0's first tile
  const int b = blockIdx.y;
  const int k = kdim(a, b);
  if (a.dead[b]) return;
  const int c0 = blockIdx.x * NB;
  const int np = (k + NB - 1) / NB;
  const int tx = tl & 15, ty = tl >> 4;
  const int64_t row0 = a.c_off[b];
  const float *G = a.G + row0 * a.ld;
  float *R = a.R + row0 * a.d;
  for (int p = np - 1; p >= 0; --p) {
    const int j0 = p * NB, jb = min(NB, k - j0);
    const float *Tg = a.Tt + ((int64_t)b * a.npanel + p) * NB * NB;
    load_t(Ts, Tg, NB, 0, NB, 0, NB);             // Ts[t][r] = T[t][r]
    load_d(Xs, R, a.d, j0, j0 + jb, c0, a.d);     // Xs[t][col] = y[j0 + t][c0 + col]
    __syncthreads();
    float acc[4][4];
    if (grp == 0) {
      zero_acc(acc);
      mmk(Ts, Xs, acc, tx, ty);                   // x[r][col]
    }
    __syncthreads();
    if (grp == 0) {
      bool fin = true;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = 4 * ty + i;
        const float4 v = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        st4(&Xs[r][4 * tx], v);  // as the B operand of the updates
        if (r < jb) {
          st4(a.X + (row0 + j0 + r) * a.d + c0 + 4 * tx, v);
          fin &= isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w);
        }
      }
      if (!fin) atomicOr(&a.dead[b], DEAD_NONFINITE);
    }
    if (p == 0) break;
    // y_i -= L_ji^T x_j, with At[t][r] = L[j0 + t][64 i + r]
    float4 pf[4];
    auto fetch = [&](int i) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = tl + 256 * u, r = e >> 4, c = (e & 15) * 4;
        pf[u] = r < jb ? ld4(G + (int64_t)(j0 + r) * a.ld + NB * i + c)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    };
    auto place = [&](float (*S)[SP]) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = tl + 256 * u, r = e >> 4, c = (e & 15) * 4;
        st4(&S[r][c], pf[u]);
      }
    };
    // both groups take the same number of rounds (and barriers); group 1 has no
    // product in the last round when p is odd
    const int rounds = (p + 1) / 2;
    if (grp < p) {
      fetch(grp);
      place(At[0]);
    }
    __syncthreads();
    for (int q = 0; q < rounds; ++q) {
      const int i = 2 * q + grp;
      const bool act = i < p, more = i + 2 < p;
      float4 cur[4];
      if (act)
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
          cur[ii] = ld4(R + (int64_t)(NB * i + 4 * ty + ii) * a.d + c0 + 4 * tx);
      if (more) fetch(i + 2);
      if (act) {
        zero_acc(acc);
        mmk(At[q & 1], Xs, acc, tx, ty);
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
          st4(R + (int64_t)(NB * i + 4 * ty + ii) * a.d + c0 + 4 * tx,
              make_float4(cur[ii].x - acc[ii][0], cur[ii].y - acc[ii][1], cur[ii].z - acc[ii][2],
                          cur[ii].w - acc[ii][3]));
      }
      if (more) place(At[(q + 1) & 1]);
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

// A side stream (highest priority) and two events per host thread, device and
// sub-batch slot: the next panel's diagonal block and panel run on the side stream
// while the caller's stream finishes the current trailing update (disjoint tiles).
// Per-thread objects keep concurrent callers from sharing events, and per-slot ones
// the concurrent sub-batches of one solve; they are created on first use and kept
// for the life of the process (three handles per thread, device and slot).
struct Lookahead {
  cudaStream_t side = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  cudaEvent_t updated[2] = {nullptr, nullptr};  // trailing update of panel p done, [p % 2]
};

static cudaError_t lookahead(int slot, Lookahead **out) {
  constexpr int kMaxDev = 64;
  static thread_local Lookahead la[kMaxDev][KVS_MAX_PARTS];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev || slot < 0 || slot >= KVS_MAX_PARTS)
    return cudaErrorInvalidDevice;
  Lookahead &l = la[dev][slot];
  if (!l.side) {
    // the highest priority: the next panel's few CTAs take SMs as soon as update
    // CTAs retire instead of queueing behind all of them
    int least = 0, greatest = 0;
    if ((e = cudaDeviceGetStreamPriorityRange(&least, &greatest)) != cudaSuccess ||
        (e = cudaStreamCreateWithPriority(&l.side, cudaStreamNonBlocking, greatest)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&l.fork, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&l.join, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&l.updated[0], cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&l.updated[1], cudaEventDisableTiming)) != cudaSuccess)
      return e;
  }
  *out = &l;
  return cudaSuccess;
}

int launch_chol_solve(const Batch &Bt, float *Vc, int32_t *status, const Work &w) {
  const HostGeom &g = Bt.g;
  if (!w.gram || !w.R || !w.X || !w.chol_t || !w.chol_p || !w.chol_y || !w.dead) return KVS_EINVAL;
  const int npanel = (g.max_c + NB - 1) / NB;
  CholArgs a{w.gram, w.R, w.X, w.chol_t, w.chol_p, w.chol_y, g.sum_c, g.B, npanel,
             w.dead, status, Bt.b->c_off, g.ld_g, g.d};
  CholTcArgs ta{w.gram, w.R, Bt.b->c_off, w.dead, g.ld_g, g.sum_c, g.B, g.d, w.err, wait_limit()};
  CholTcMaps tm;
  int rc;
  if ((rc = make_map_f32(&tm.p, w.chol_p, 4 * (uint64_t)g.sum_c, NB, 128)) ||
      (rc = make_map_f32(&tm.y, w.chol_y, 4 * (uint64_t)g.B * g.d, NB, (uint32_t)g.d)))
    return rc;
  KVS_CUDA_TRY(set_smem_once(k_chol_backward, BWD_SMEM));
  KVS_CUDA_TRY(set_smem_once(k_chol_diag, DIAG_SMEM));
  Lookahead *la = nullptr;
  KVS_CUDA_TRY(lookahead(Bt.slot, &la));
  KVS_CUDA_TRY(cudaMemsetAsync(w.dead, 0, sizeof(int) * g.B, Bt.st));
  const int ndc = g.d / NB;
  // Panel p on the side stream: its diagonal block (with the update by panel p - 1),
  // then its column below (likewise).  The trailing update of panel p runs on the
  // caller's stream beside panel p + 1, which waits only for the update of panel
  // p - 1 (it covers column blocks from p + 2 on).
  KVS_CUDA_TRY(cudaEventRecord(la->fork, Bt.st));
  KVS_CUDA_TRY(cudaStreamWaitEvent(la->side, la->fork, 0));
  for (int p = 0; p < npanel; ++p) {
    const int j0 = p * NB;
    if (p >= 2) KVS_CUDA_TRY(cudaStreamWaitEvent(la->side, la->updated[p & 1], 0));
    k_chol_diag<<<g.B, 256, DIAG_SMEM, la->side>>>(a, j0);
    KVS_LAUNCH_CHECK("k_chol_diag");
    const int n2 = g.max_c - j0 - NB;
    if (n2 > 0) {
      k_chol_panel<<<dim3((n2 + NB - 1) / NB, g.B), 256, 0, la->side>>>(a, j0);
      KVS_LAUNCH_CHECK("k_chol_panel");
    }
    KVS_CUDA_TRY(cudaEventRecord(la->join, la->side));
    KVS_CUDA_TRY(cudaStreamWaitEvent(Bt.st, la->join, 0));
    if (p + 1 < npanel) {
      if ((rc = launch_chol_update_tc(tm, ta, j0, g.max_c, Bt.st))) return rc;
      KVS_CUDA_TRY(cudaEventRecord(la->updated[p & 1], Bt.st));
    }
  }
  k_chol_backward<<<dim3(ndc, g.B), 512, BWD_SMEM, Bt.st>>>(a);
  KVS_LAUNCH_CHECK("k_chol_backward");
  const int64_t n4 = (int64_t)g.max_c * g.d / 4;
  const int blocks = (int)std::min<int64_t>((n4 + 255) / 256, 64);
  k_chol_store<<<dim3(blocks, g.B), 256, 0, Bt.st>>>(a, Vc);
  KVS_LAUNCH_CHECK("k_chol_store");
  return KVS_OK;
}

}  // namespace kvs
