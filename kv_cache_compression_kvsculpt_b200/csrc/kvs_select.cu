// Training-query construction and top-k key initialisation.
//
// "KVSculpt: KV Cache Compression as Distillation", section 2
// "Training Query Construction" (retain queries; synthetic future queries by
// De-RoPE of context queries and re-embedding at future positions) and
// "Initialization" (keys start at the top-k positions by attention importance).
#include <math.h>

#include "kvs_internal.cuh"

namespace kvs {
namespace {

// One CTA per output row, one thread per rotation pair (i, i + d/2).
// Synthetic row j of a query head: the context query RoPE'd at p is rotated
// back by p and forward by N + j, i.e. by (N + j - p) theta_i; the angle is
// formed and reduced in float64, the rotation applied in float32.
__global__ void k_build_queries(kvs_query_spec sp, const float *__restrict__ q_retain,
                                const float *__restrict__ q_ctx, const int32_t *__restrict__ pos,
                                float *__restrict__ Q) {
  const int per_head = sp.m_q + sp.n_syn;
  const int64_t row = blockIdx.x;
  const int64_t bh = row / per_head;  // problem * g + head
  const int j = (int)(row % per_head);
  const int d = sp.d, half = d / 2;
  float *out = Q + row * d;
  if (j < sp.m_q) {
    const float *src = q_retain + (bh * sp.m_q + j) * d;
    for (int c = threadIdx.x; c < d; c += blockDim.x) out[c] = src[c];
    return;
  }
  const int js = j - sp.m_q;
  const int64_t srow = bh * sp.n_syn + js;
  const float *src = q_ctx + srow * d;
  const double shift = (double)sp.N + (double)js - (double)pos[srow];
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    const double theta = pow((double)sp.rope_base, -2.0 * (double)i / (double)d);
    double sn, cs;
    sincos(shift * theta, &sn, &cs);
    const float c = (float)cs, s = (float)sn;
    const float lo = src[i], hi = src[i + half];
    out[i] = lo * c - hi * s;
    out[i + half] = hi * c + lo * s;
  }
}

__device__ __forceinline__ uint32_t order_key(float f) {
  if (f == 0.f) f = 0.f;  // -0 and +0 compare equal
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exact top-k per problem: radix select of the k-th largest order key, then a
// stable compaction in position order that keeps every key above it and the
// lowest-position keys equal to it.  One CTA of 1024 threads per problem.
__global__ void __launch_bounds__(1024) k_topk(const float *__restrict__ imp,
                                               const int64_t *__restrict__ z_off,
                                               const int64_t *__restrict__ c_off,
                                               int32_t *__restrict__ idx) {
  extern __shared__ uint32_t keys[];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t wsum[32];
  __shared__ uint32_t s_sel, s_need, s_run_eq, s_run_out;
  const int b = blockIdx.x;
  const int z = (int)(z_off[b + 1] - z_off[b]);
  const int k = (int)(c_off[b + 1] - c_off[b]);
  const float *im = imp + z_off[b];
  int32_t *out = idx + c_off[b];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  for (int j = tid; j < z; j += blockDim.x) keys[j] = order_key(im[j]);
  uint32_t prefix = 0, mask = 0;
  if (tid == 0) s_need = (uint32_t)k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int e = tid; e < 256; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    for (int j = tid; j < z; j += blockDim.x) {
      const uint32_t key = keys[j];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      uint32_t need = s_need, cum = 0;
      int sel = 0;
      for (int bk = 255; bk >= 0; --bk) {
        if (cum + hist[bk] >= need) {
          sel = bk;
          need -= cum;
          break;
        }
        cum += hist[bk];
      }
      s_sel = (uint32_t)sel;
      s_need = need;
    }
    __syncthreads();
    prefix |= s_sel << shift;
    mask |= 255u << shift;
  }
  const uint32_t T = prefix;       // value of the k-th largest key
  const uint32_t take_eq = s_need; // keys equal to T to keep, lowest positions first
  if (tid == 0) {
    s_run_eq = 0;
    s_run_out = 0;
  }
  __syncthreads();
  const uint32_t lt = (1u << lane) - 1u;
  for (int base = 0; base < z; base += blockDim.x) {
    const int j = base + tid;
    const uint32_t key = (j < z) ? keys[j] : 0u;
    const bool eq = (j < z) && key == T;
    // rank of this equal key among equal keys at lower positions
    uint32_t bal = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) wsum[w] = __popc(bal);
    __syncthreads();
    if (tid == 0) {
      uint32_t run = s_run_eq;
      for (int q = 0; q < 32; ++q) {
        const uint32_t c = wsum[q];
        wsum[q] = run;
        run += c;
      }
      s_run_eq = run;
    }
    __syncthreads();
    const uint32_t eq_rank = wsum[w] + __popc(bal & lt);
    const bool sel = (j < z) && (key > T || (eq && eq_rank < take_eq));
    __syncthreads();
    bal = __ballot_sync(0xffffffffu, sel);
    if (lane == 0) wsum[w] = __popc(bal);
    __syncthreads();
    if (tid == 0) {
      uint32_t run = s_run_out;
      for (int q = 0; q < 32; ++q) {
        const uint32_t c = wsum[q];
        wsum[q] = run;
        run += c;
      }
      s_run_out = run;
    }
    __syncthreads();
    const uint32_t at = wsum[w] + __popc(bal & lt);
    if (sel && at < (uint32_t)k) out[at] = j;
    __syncthreads();
  }
}

// Kc[c_off[b] + r] = Kz[z_off[b] + idx[r]]; one warp per selected row.
__global__ void k_gather(const float *__restrict__ Kz, const int64_t *__restrict__ z_off,
                         const int64_t *__restrict__ c_off, const int32_t *__restrict__ idx,
                         float *__restrict__ Kc, int d) {
  const int b = blockIdx.y;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int64_t c0 = c_off[b];
  if (r >= c_off[b + 1] - c0) return;
  const int src_row = idx[c0 + r];
  if (src_row < 0 || src_row >= z_off[b + 1] - z_off[b]) return;
  const float *src = Kz + (z_off[b] + src_row) * d;
  float *dst = Kc + (c0 + r) * d;
  for (int c = threadIdx.x & 31; c < d; c += 32) dst[c] = src[c];
}

}  // namespace

int launch_build_queries(const kvs_query_spec *sp, const float *q_retain, const float *q_ctx,
                         const int32_t *pos, float *Q, cudaStream_t st) {
  const int64_t rows = (int64_t)sp->B * sp->g * (sp->m_q + sp->n_syn);
  if (rows == 0) return KVS_OK;
  k_build_queries<<<(unsigned)rows, sp->d / 2, 0, st>>>(*sp, q_retain, q_ctx, pos, Q);
  KVS_LAUNCH_CHECK("k_build_queries");
  return KVS_OK;
}

int launch_topk(const Batch &Bt, const float *imp, const float *Kz, int32_t *idx, float *Kc) {
  const size_t smem = (size_t)Bt.g.max_z * sizeof(uint32_t);
  KVS_CUDA_TRY(set_smem_once(k_topk, (int)smem));
  k_topk<<<Bt.g.B, 1024, smem, Bt.st>>>(imp, Bt.b->z_off, Bt.b->c_off, idx);
  KVS_LAUNCH_CHECK("k_topk");
  k_gather<<<dim3((Bt.g.max_c + 7) / 8, Bt.g.B), 256, 0, Bt.st>>>(Kz, Bt.b->z_off, Bt.b->c_off,
                                                                    idx, Kc, Bt.g.d);
  KVS_LAUNCH_CHECK("k_gather");
  return KVS_OK;
}

}  // namespace kvs
