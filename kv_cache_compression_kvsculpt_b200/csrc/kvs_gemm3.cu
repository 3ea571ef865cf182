// Normal equations of the ridge fit on tcgen05 tensor cores:
// G = A^T A + lambda I and R = A^T Y ("KVSculpt: KV Cache Compression as
// Distillation", section 2 "Value Optimization": values solved in closed form
// by ridge regression given the attention weights A of the current keys).
//
// A (softmax weights, [padded n_q, k] per problem) and Y are held as bf16
// hi/lo pairs; each product takes three bf16 MMAs (hi.hi + hi.lo + lo.hi)
// with fp32 accumulation in TMEM, which keeps about 16 significant bits of
// each operand.  Both operands are read MN-major (keys / value columns
// contiguous), the contraction runs over training queries in tiles of 64.
// One CTA owns one 128 x 128 output tile: the Gram matrix is formed on its
// lower block triangle only (the Cholesky reads the lower triangle).
#include <math.h>

#include "kvs_attn_tc.cuh"

namespace kvs {
namespace {

using namespace tc;

constexpr int TM = 128, TN = 128, TKQ = 64, NS = 3;
constexpr int OP_BYTES = TKQ * TM * 2;        // one 64-row x 128-column bf16 operand tile
constexpr int STAGE = 4 * OP_BYTES;           // A hi, A lo, B hi, B lo
constexpr int SMEM = NS * STAGE + 1024;

struct GBars {
  uint64_t full[NS], empty[NS];
  uint64_t done;
  uint32_t tmem;
  int abort;
};

__global__ void __launch_bounds__(192, 1)
    k_gemm3(const __grid_constant__ CUtensorMap mAh, const __grid_constant__ CUtensorMap mAl,
            const __grid_constant__ CUtensorMap mBh, const __grid_constant__ CUtensorMap mBl,
            GemmArgs3 a, int gram) {
  extern __shared__ unsigned char smraw[];
  unsigned char *sm = (unsigned char *)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
  __shared__ GBars bars;
  const int b = blockIdx.y;
  const int64_t m_begin = a.m_off[b];
  const int nk = (int)(a.m_off[b + 1] - m_begin);
  const int T = (nk + TM - 1) / TM;
  int ti, tj;
  const int t = blockIdx.x;
  if (gram) {
    if (t >= T * (T + 1) / 2) return;
    ti = (int)((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
    while (ti * (ti + 1) / 2 > t) --ti;
    while ((ti + 1) * (ti + 2) / 2 <= t) ++ti;
    tj = t - ti * (ti + 1) / 2;
  } else {
    if (t >= T) return;
    ti = t;
    tj = 0;
  }
  const int N = gram ? TN : a.n_fixed;          // MMA N
  const int ncols = gram ? nk : a.n_fixed;      // valid output columns
  const int64_t ka0 = a.a_pad_off[b];
  const int kq = (int)(a.a_pad_off[b + 1] - ka0);  // padded query rows (multiple of 128)
  const int64_t kb0 = a.b_row_off[b];
  const int nkt = kq / TKQ;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&bars.full[i], 1);
      mbar_init(&bars.empty[i], 1);
    }
    mbar_init(&bars.done, 1);
    bars.abort = 0;
    fence_barrier_init();
  }
  if (warp == 5) tmem_alloc(&bars.tmem, 128);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = bars.tmem;
  volatile int *abort = &bars.abort;
  const int nb_boxes = N / 64;
  const uint32_t stage_tx = 2 * OP_BYTES + 2 * (uint32_t)(nb_boxes * 64 * TKQ * 2);

  if (warp == 4) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nkt; ++i) {
        const int st = i % NS;
        if (i >= NS && !mbar_wait(&bars.empty[st], ((i / NS) - 1) & 1, abort)) {
          *abort = 1;
          break;
        }
        issued = i + 1;
        unsigned char *base = sm + st * STAGE;
        mbar_arrive_expect_tx(&bars.full[st], stage_tx);
        const int ya = (int)(ka0 + i * TKQ), yb = (int)(kb0 + i * TKQ);
        for (int r = 0; r < 2; ++r) {
          tma_load_2d(base + r * TKQ * 128, &mAh, &bars.full[st], ti * TM + 64 * r, ya);
          tma_load_2d(base + OP_BYTES + r * TKQ * 128, &mAl, &bars.full[st], ti * TM + 64 * r, ya);
        }
        for (int r = 0; r < nb_boxes; ++r) {
          tma_load_2d(base + 2 * OP_BYTES + r * TKQ * 128, &mBh, &bars.full[st], tj * TN + 64 * r, yb);
          tma_load_2d(base + 3 * OP_BYTES + r * TKQ * 128, &mBl, &bars.full[st], tj * TN + 64 * r, yb);
        }
      }
      if (*abort)
        for (int i = (issued > NS ? issued - NS : 0); i < issued; ++i)
          mbar_wait(&bars.full[i % NS], (i / NS) & 1);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      const uint32_t id = idesc_bf16(TM, N, true, true);
      bool ok = true;
      for (int i = 0; i < nkt; ++i) {
        const int st = i % NS;
        if (!mbar_wait(&bars.full[st], (i / NS) & 1, abort)) { ok = false; break; }
        fence_after_sync();
        const uint64_t d0 = sdesc(smem_u32(sm + st * STAGE), TKQ * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < TKQ / 16; ++kk) {
          const uint64_t ah = sdesc_add(d0, kk * 2048);
          const uint64_t al = sdesc_add(ah, OP_BYTES);
          const uint64_t bh = sdesc_add(ah, 2 * OP_BYTES);
          const uint64_t bl = sdesc_add(ah, 3 * OP_BYTES);
          mma_bf16(tmem, ah, bh, id, (i > 0 || kk > 0) ? 1u : 0u);
          mma_bf16(tmem, ah, bl, id, 1u);
          mma_bf16(tmem, al, bh, id, 1u);
        }
        mma_commit(&bars.empty[st]);
      }
      mma_commit(&bars.done);
      if (!ok) *abort = 1;
      mbar_wait(&bars.done, 0);
    }
  } else {
    const int row = tid;
    const int gi = ti * TM + row;
    if (!mbar_wait(&bars.done, 0, abort)) *abort = 1;
    fence_after_sync();
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float *crow = a.c + (m_begin + gi) * a.ldc;
#pragma unroll 1
    for (int c0 = 0; c0 < N; c0 += 32) {
      float v[32];
      tmem_ld32(tmem + lane_base + c0, v);
      if (gi < nk && nkt > 0) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int gc = tj * TN + c0 + e;
          if (gc < ncols) crow[gc] = v[e] + ((gram && gc == gi) ? a.diag : 0.f);
        }
      }
    }
    if (nkt == 0 && gi < nk)
      for (int gc = tj * TN; gc < min(tj * TN + N, ncols); ++gc)
        crow[gc] = (gram && gc == gi) ? a.diag : 0.f;
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    fence_after_sync();
    tmem_dealloc(tmem, 128);
  }
  if (tid == 0 && bars.abort && a.err) atomicOr(a.err, 1);
}

}  // namespace

int launch_gemm3_tc(const GemmMaps &m, const GemmArgs3 &a, int tiles_m, int gram, int B,
                    cudaStream_t st) {
  KVS_CUDA_TRY(set_smem_once(k_gemm3, SMEM));
  const int tiles = gram ? tiles_m * (tiles_m + 1) / 2 : tiles_m;
  if (tiles <= 0) return KVS_OK;
  k_gemm3<<<dim3(tiles, B), 192, SMEM, st>>>(m.ah, m.al, m.bh, m.bl, a, gram);
  KVS_LAUNCH_CHECK("k_gemm3");
  return KVS_OK;
}

}  // namespace kvs
