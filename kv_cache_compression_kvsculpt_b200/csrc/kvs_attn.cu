// Attention contractions of the distillation solve: targets, loss forward,
// dK_c backward and the ridge normal equations.
//
// "KVSculpt: KV Cache Compression as Distillation", section 2 "Loss Function"
// (output MSE + LSE matching), "Value Optimization" (ridge regression given
// the attention weights) and "Initialization" (attention importance).
//
// This file holds the straightforward batched formulation on CUDA cores: the
// score matrix of every problem is materialised in the workspace and each
// contraction is a tiled fp32 GEMM with a small fused epilogue.
#include <math.h>

#include "kvs_internal.cuh"

namespace kvs {
namespace {

enum { EPI_STORE = 0, EPI_GRAM = 1, EPI_DS = 2 };

struct GemmArgs {
  Mat A, B, C;          // C is written through a const_cast
  Dim M, N, K;
  float alpha, lam;
  Mat rowvec;           // EPI_DS: delta per row (ld = 1)
  Filter flt;
};

constexpr int TM = 64, TN = 64, TK = 16;

// C = alpha * op(A) op(B) with op(A) = A (row-major M x K) or A^T (A stored K x M),
// op(B) = B^T (B stored N x K) or B (stored K x N).  One 64 x 64 tile per CTA.
template <bool TA, bool TB, int EPI>
__global__ void __launch_bounds__(256) k_gemm(GemmArgs a) {
  const int b = blockIdx.z;
  if (a.flt.skip(b)) return;
  const int M = a.M.of(b), N = a.N.of(b), K = a.K.of(b);
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  if (m0 >= M || n0 >= N) return;
  const float *A = a.A.at(b);
  const float *Bm = a.B.at(b);
  float *C = const_cast<float *>(a.C.at(b));
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
  for (int k0 = 0; k0 < K; k0 += TK) {
#pragma unroll
    for (int e = t; e < TM * TK; e += 256) {
      int m, kk;
      if (!TA) { m = e >> 4; kk = e & 15; } else { kk = e >> 6; m = e & 63; }
      const int gm = m0 + m, gk = k0 + kk;
      float v = 0.f;
      if (gm < M && gk < K)
        v = TA ? A[(int64_t)gk * a.A.ld + gm] : A[(int64_t)gm * a.A.ld + gk];
      As[kk][m] = v;
    }
#pragma unroll
    for (int e = t; e < TN * TK; e += 256) {
      int n, kk;
      if (TB) { n = e >> 4; kk = e & 15; } else { kk = e >> 6; n = e & 63; }
      const int gn = n0 + n, gk = k0 + kk;
      float v = 0.f;
      if (gn < N && gk < K)
        v = TB ? Bm[(int64_t)gn * a.B.ld + gk] : Bm[(int64_t)gk * a.B.ld + gn];
      Bs[kk][n] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  const float *dl = (EPI == EPI_DS) ? a.rowvec.at(b) : nullptr;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn >= N) continue;
      float v = a.alpha * acc[i][j];
      float *c = C + (int64_t)gm * a.C.ld + gn;
      if (EPI == EPI_STORE) *c = v;
      else if (EPI == EPI_GRAM) *c = v + (gm == gn ? a.lam : 0.f);
      else *c = *c * (v - dl[gm]);
    }
  }
}

template <bool TA, bool TB, int EPI>
int gemm(const Batch &Bt, const GemmArgs &a, int max_m, int max_n) {
  if (max_m <= 0 || max_n <= 0) return KVS_OK;
  dim3 grid((max_n + TN - 1) / TN, (max_m + TM - 1) / TM, Bt.g.B);
  k_gemm<TA, TB, EPI><<<grid, 256, 0, Bt.st>>>(a);
  KVS_LAUNCH_CHECK("k_gemm");
  return KVS_OK;
}

// Row softmax in place: S[i, :n] <- exp(S - lse_i); lse_i = log sum_j exp(S_ij).
__global__ void __launch_bounds__(256) k_softmax_rows(Mat S, Dim rows, Dim cols, Mat lse,
                                                      Filter flt) {
  const int b = blockIdx.y;
  if (flt.skip(b)) return;
  const int r = blockIdx.x;
  if (r >= rows.of(b)) return;
  const int n = cols.of(b);
  float *s = const_cast<float *>(S.at(b)) + (int64_t)r * S.ld;
  __shared__ float red[32];
  float mx = -INFINITY;
  for (int j = threadIdx.x; j < n; j += blockDim.x) mx = fmaxf(mx, s[j]);
  mx = block_max(mx, red);
  float sum = 0.f;
  for (int j = threadIdx.x; j < n; j += blockDim.x) sum += expf(s[j] - mx);
  sum = block_sum(sum, red);
  const float l = mx + logf(sum);
  for (int j = threadIdx.x; j < n; j += blockDim.x) s[j] = expf(s[j] - l);
  if (threadIdx.x == 0) const_cast<float *>(lse.at(b))[r] = l;
}

// Per-row residual of the loss: one warp per training query.
//   Go = c_o (Yh - Y), delta = Go . Yh - c_l (lh - l), row_out = |Yh - Y|^2,
//   row_ls = (lh - l)^2, with c_o = 2 w_out / (n_q d) and c_l = 2 w_lse / n_q.
__global__ void __launch_bounds__(256) k_residual(Mat Yh, Mat Y, Mat lh, Mat l, Mat Go,
                                                  Mat delta, Mat row_out, Mat row_ls, Dim rows,
                                                  int d, float w_out, float w_lse,
                                                  Filter flt) {
  const int b = blockIdx.y;
  if (flt.skip(b)) return;
  const int nq = rows.of(b);
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= nq) return;
  const float co = 2.f * w_out / ((float)nq * (float)d);
  const float cl = 2.f * w_lse / (float)nq;
  const float *yh = Yh.at(b) + (int64_t)r * d;
  const float *y = Y.at(b) + (int64_t)r * d;
  float *go = const_cast<float *>(Go.at(b)) + (int64_t)r * d;
  float se = 0.f, gy = 0.f;
  for (int c = lane; c < d; c += 32) {
    const float e = yh[c] - y[c];
    se = fmaf(e, e, se);
    const float gv = co * e;
    go[c] = gv;
    gy = fmaf(gv, yh[c], gy);
  }
  se = warp_sum(se);
  gy = warp_sum(gy);
  if (lane == 0) {
    const float el = lh.at(b)[r] - l.at(b)[r];
    const_cast<float *>(delta.at(b))[r] = gy - cl * el;
    const_cast<float *>(row_out.at(b))[r] = se;
    const_cast<float *>(row_ls.at(b))[r] = el * el;
  }
}

// loss[b] = w_out/(n_q d) sum row_out + w_lse/n_q sum row_ls (fixed-order block sums).
__global__ void __launch_bounds__(256) k_loss_reduce(Mat row_out, Mat row_ls, Dim rows, int d,
                                                     float w_out, float w_lse, float *loss,
                                                     float *parts, Filter flt) {
  const int b = blockIdx.x;
  if (flt.skip(b)) return;
  const int nq = rows.of(b);
  __shared__ double red[32];
  const float *ro = row_out.at(b), *rl = row_ls.at(b);
  double so = 0.0, sl = 0.0;
  for (int i = threadIdx.x; i < nq; i += blockDim.x) {
    so += ro[i];
    sl += rl[i];
  }
  so = block_sum_d(so, red);
  sl = block_sum_d(sl, red);
  if (threadIdx.x == 0) {
    const double out = so / ((double)nq * d), ls = sl / (double)nq;
    loss[b] = (float)(w_out * out + w_lse * ls);
    if (parts) {
      parts[2 * b] = (float)out;
      parts[2 * b + 1] = (float)ls;
    }
  }
}

// importance[j] = sum_i A[i, j] over the problem's training queries.
__global__ void __launch_bounds__(256) k_colsum(Mat A, Dim rows, Dim cols, Mat imp) {
  const int b = blockIdx.y;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= cols.of(b)) return;
  const int nq = rows.of(b);
  const float *a = A.at(b) + j;
  float s = 0.f;
  for (int i = 0; i < nq; ++i) s += a[(int64_t)i * A.ld];
  const_cast<float *>(imp.at(b))[j] = s;
}

Mat mat(const float *p, const int64_t *off, int64_t ld) { return Mat{p, off, 0, ld}; }

}  // namespace

int launch_targets(const Batch &Bt, const float *Q, const float *Kz, const float *Vz, float *Y,
                   float *lse, float *imp, const Work &w) {
  const HostGeom &g = Bt.g;
  const kvs_batch *b = Bt.b;
  const float s = 1.f / sqrtf((float)g.d);
  GemmArgs a{};
  a.A = mat(Q, b->q_off, g.d);
  a.B = mat(Kz, b->z_off, g.d);
  a.C = mat(w.S, b->q_off, g.ld_s);
  a.M = Dim{b->q_off, 0};
  a.N = Dim{b->z_off, 0};
  a.K = Dim{nullptr, g.d};
  a.alpha = s;
  int rc = gemm<false, true, EPI_STORE>(Bt, a, g.max_q, g.max_z);
  if (rc) return rc;
  k_softmax_rows<<<dim3(g.max_q, g.B), 256, 0, Bt.st>>>(mat(w.S, b->q_off, g.ld_s), Dim{b->q_off, 0},
                                                         Dim{b->z_off, 0}, mat(lse, b->q_off, 1),
                                                         Filter{nullptr, 0, 0});
  KVS_LAUNCH_CHECK("k_softmax_rows");
  GemmArgs o{};
  o.A = mat(w.S, b->q_off, g.ld_s);
  o.B = mat(Vz, b->z_off, g.d);
  o.C = mat(Y, b->q_off, g.d);
  o.M = Dim{b->q_off, 0};
  o.N = Dim{nullptr, g.d};
  o.K = Dim{b->z_off, 0};
  o.alpha = 1.f;
  rc = gemm<false, false, EPI_STORE>(Bt, o, g.max_q, g.d);
  if (rc) return rc;
  if (imp) {
    k_colsum<<<dim3((g.max_z + 255) / 256, g.B), 256, 0, Bt.st>>>(
        mat(w.S, b->q_off, g.ld_s), Dim{b->q_off, 0}, Dim{b->z_off, 0}, mat(imp, b->z_off, 1));
    KVS_LAUNCH_CHECK("k_colsum");
  }
  return KVS_OK;
}

static int scores_softmax(const Batch &Bt, const float *Q, const float *Kc, Filter flt,
                          const Work &w) {
  const HostGeom &g = Bt.g;
  const kvs_batch *b = Bt.b;
  GemmArgs a{};
  a.A = mat(Q, b->q_off, g.d);
  a.B = mat(Kc, b->c_off, g.d);
  a.C = mat(w.S, b->q_off, g.ld_s);
  a.M = Dim{b->q_off, 0};
  a.N = Dim{b->c_off, 0};
  a.K = Dim{nullptr, g.d};
  a.alpha = 1.f / sqrtf((float)g.d);
  a.flt = flt;
  int rc = gemm<false, true, EPI_STORE>(Bt, a, g.max_q, g.max_c);
  if (rc) return rc;
  k_softmax_rows<<<dim3(g.max_q, g.B), 256, 0, Bt.st>>>(mat(w.S, b->q_off, g.ld_s), Dim{b->q_off, 0},
                                                         Dim{b->c_off, 0},
                                                         mat(w.lse_h, b->q_off, 1), flt);
  KVS_LAUNCH_CHECK("k_softmax_rows");
  return KVS_OK;
}

int launch_forward(const Batch &Bt, const float *Q, const float *Kc, const float *Vc,
                   const float *Y, const float *lse, float w_out, float w_lse, float *loss,
                   float *parts, Filter flt, const Work &w) {
  const HostGeom &g = Bt.g;
  const kvs_batch *b = Bt.b;
  int rc = scores_softmax(Bt, Q, Kc, flt, w);
  if (rc) return rc;
  GemmArgs o{};
  o.A = mat(w.S, b->q_off, g.ld_s);
  o.B = mat(Vc, b->c_off, g.d);
  o.C = mat(w.Yh, b->q_off, g.d);
  o.M = Dim{b->q_off, 0};
  o.N = Dim{nullptr, g.d};
  o.K = Dim{b->c_off, 0};
  o.alpha = 1.f;
  o.flt = flt;
  rc = gemm<false, false, EPI_STORE>(Bt, o, g.max_q, g.d);
  if (rc) return rc;
  k_residual<<<dim3((g.max_q + 7) / 8, g.B), 256, 0, Bt.st>>>(
      mat(w.Yh, b->q_off, g.d), mat(Y, b->q_off, g.d), mat(w.lse_h, b->q_off, 1),
      mat(lse, b->q_off, 1), mat(w.Go, b->q_off, g.d), mat(w.delta, b->q_off, 1),
      mat(w.row_out, b->q_off, 1), mat(w.row_ls, b->q_off, 1), Dim{b->q_off, 0}, g.d, w_out,
      w_lse, flt);
  KVS_LAUNCH_CHECK("k_residual");
  k_loss_reduce<<<g.B, 256, 0, Bt.st>>>(mat(w.row_out, b->q_off, 1), mat(w.row_ls, b->q_off, 1),
                                        Dim{b->q_off, 0}, g.d, w_out, w_lse, loss, parts, flt);
  KVS_LAUNCH_CHECK("k_loss_reduce");
  return KVS_OK;
}

int launch_backward(const Batch &Bt, const float *Q, const float *Vc, float *dKc,
                    Filter flt, const Work &w) {
  const HostGeom &g = Bt.g;
  const kvs_batch *b = Bt.b;
  // dS = A * (Go Vc^T - delta), in place over A.
  GemmArgs p{};
  p.A = mat(w.Go, b->q_off, g.d);
  p.B = mat(Vc, b->c_off, g.d);
  p.C = mat(w.S, b->q_off, g.ld_s);
  p.M = Dim{b->q_off, 0};
  p.N = Dim{b->c_off, 0};
  p.K = Dim{nullptr, g.d};
  p.alpha = 1.f;
  p.rowvec = mat(w.delta, b->q_off, 1);
  p.flt = flt;
  int rc = gemm<false, true, EPI_DS>(Bt, p, g.max_q, g.max_c);
  if (rc) return rc;
  // dKc = s dS^T Q
  GemmArgs k{};
  k.A = mat(w.S, b->q_off, g.ld_s);
  k.B = mat(Q, b->q_off, g.d);
  k.C = mat(dKc, b->c_off, g.d);
  k.M = Dim{b->c_off, 0};
  k.N = Dim{nullptr, g.d};
  k.K = Dim{b->q_off, 0};
  k.alpha = 1.f / sqrtf((float)g.d);
  k.flt = flt;
  return gemm<true, false, EPI_STORE>(Bt, k, g.max_c, g.d);
}

int launch_fit(const Batch &Bt, const float *Q, const float *Kc, const float *Y, float lam,
               float *Vc, int32_t *status, const Work &w) {
  const HostGeom &g = Bt.g;
  const kvs_batch *b = Bt.b;
  int rc = scores_softmax(Bt, Q, Kc, Filter{nullptr, 0, 0}, w);
  if (rc) return rc;
  GemmArgs G{};
  G.A = mat(w.S, b->q_off, g.ld_s);
  G.B = mat(w.S, b->q_off, g.ld_s);
  G.C = mat(w.gram, b->c_off, g.max_c);
  G.M = Dim{b->c_off, 0};
  G.N = Dim{b->c_off, 0};
  G.K = Dim{b->q_off, 0};
  G.alpha = 1.f;
  G.lam = lam;
  rc = gemm<true, false, EPI_GRAM>(Bt, G, g.max_c, g.max_c);
  if (rc) return rc;
  GemmArgs R{};
  R.A = mat(w.S, b->q_off, g.ld_s);
  R.B = mat(Y, b->q_off, g.d);
  R.C = mat(w.R, b->c_off, g.d);
  R.M = Dim{b->c_off, 0};
  R.N = Dim{nullptr, g.d};
  R.K = Dim{b->q_off, 0};
  R.alpha = 1.f;
  rc = gemm<true, false, EPI_STORE>(Bt, R, g.max_c, g.d);
  if (rc) return rc;
  return launch_chol_solve(Bt, Vc, status, w);
}

}  // namespace kvs
