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
// One CTA owns one 128-row output tile, as wide as the product allows: a
// tcgen05.mma instruction costs about the same for any N up to 256, so Gram
// tiles are 128 x 256 (only those that reach the lower triangle, which the
// Cholesky reads) and A^T Y tiles are 128 x d.
#include <math.h>

#include "kvs_attn_tc.cuh"

namespace kvs {
namespace {

using namespace tc;

constexpr int TM = 128, TKQ = 64;
constexpr int A_BYTES = TKQ * TM * 2;  // one 64-row x 128-column bf16 operand tile

template <int TN>
struct G3 {
  static constexpr int B_BYTES = TKQ * TN * 2;            // one 64-row x TN-column tile
  static constexpr int STAGE = 2 * A_BYTES + 2 * B_BYTES;  // A hi, A lo, B hi, B lo
  static constexpr int NS = TN > 128 ? 2 : 3;
  static constexpr int SMEM = NS * STAGE + 1024;
  // tiles up to 128 wide take B_hi and B_lo side by side as one operand of N = 2 TN
  // for A_hi, and B_hi alone (N = TN) for A_lo: two instructions per 16-row step
  // instead of three, into two summed halves
  static constexpr bool CAT = TN <= 128;
  static constexpr int MMA_N = CAT ? 2 * TN : TN;
  static constexpr uint32_t TMEM_COLS = MMA_N < 32 ? 32 : MMA_N;
};
constexpr int NSMAX = 3;

// Gram tile t of a problem with T row tiles: the t-th (row, column) pair in
// row-major order among the 128 x TN tiles that reach the lower triangle.
template <int TN>
__device__ __forceinline__ bool gram_tile(int t, int T, int *ti, int *tj) {
  for (int i = 0; i < T; ++i) {
    const int n = (i * TM + TM - 1) / TN + 1;  // column tiles of row tile i
    if (t < n) {
      *ti = i;
      *tj = t;
      return true;
    }
    t -= n;
  }
  return false;
}

template <int TN>
__host__ __device__ constexpr int gram_tiles(int T) {
  int n = 0;
  for (int i = 0; i < T; ++i) n += (i * TM + TM - 1) / TN + 1;
  return n;
}

struct GBars {
  uint64_t full[NSMAX], empty[NSMAX];
  uint64_t done;
  uint32_t tmem;
  int abort;
};

template <int TN>
__global__ void __launch_bounds__(192, 1)
    k_gemm3(const __grid_constant__ CUtensorMap mAh, const __grid_constant__ CUtensorMap mAl,
            const __grid_constant__ CUtensorMap mBh, const __grid_constant__ CUtensorMap mBl,
            GemmArgs3 a, int gram) {
  using C = G3<TN>;
  constexpr int NS = C::NS;
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
    if (!gram_tile<TN>(t, T, &ti, &tj)) return;
  } else {
    if (t >= T) return;
    ti = t;
    tj = 0;
  }
  const int N = TN;                             // MMA N (A^T Y: TN = d)
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
  if (warp == 5) tmem_alloc(&bars.tmem, C::TMEM_COLS);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = bars.tmem;
  volatile int *abort = &bars.abort;
  const int nb_boxes = N / 64;
  const uint32_t stage_tx = C::STAGE;

  if (warp == 4) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nkt; ++i) {
        const int st = i % NS;
        if (i >= NS && !mbar_wait(&bars.empty[st], ((i / NS) - 1) & 1, abort, a.wait)) {
          *abort = 1;
          break;
        }
        issued = i + 1;
        unsigned char *base = sm + st * C::STAGE;
        mbar_arrive_expect_tx(&bars.full[st], stage_tx);
        const int ya = (int)(ka0 + i * TKQ), yb = (int)(kb0 + i * TKQ);
        for (int r = 0; r < 2; ++r) {
          tma_load_2d(base + r * TKQ * 128, &mAh, &bars.full[st], ti * TM + 64 * r, ya);
          tma_load_2d(base + A_BYTES + r * TKQ * 128, &mAl, &bars.full[st], ti * TM + 64 * r, ya);
        }
        for (int r = 0; r < nb_boxes; ++r) {
          tma_load_2d(base + 2 * A_BYTES + r * TKQ * 128, &mBh, &bars.full[st], tj * TN + 64 * r, yb);
          tma_load_2d(base + 2 * A_BYTES + C::B_BYTES + r * TKQ * 128, &mBl, &bars.full[st],
                      tj * TN + 64 * r, yb);
        }
      }
      if (*abort)
        for (int i = (issued > NS ? issued - NS : 0); i < issued; ++i)
          mbar_wait(&bars.full[i % NS], (i / NS) & 1);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      const uint32_t id = idesc_bf16(TM, C::MMA_N, true, true);
      const uint32_t id_h = idesc_bf16(TM, TN, true, true);  // CAT: B_hi alone
      bool ok = true;
      for (int i = 0; i < nkt; ++i) {
        const int st = i % NS;
        if (!mbar_wait(&bars.full[st], (i / NS) & 1, abort, a.wait)) { ok = false; break; }
        fence_after_sync();
        const uint64_t d0 = sdesc(smem_u32(sm + st * C::STAGE), TKQ * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < TKQ / 16; ++kk) {
          const uint64_t ah = sdesc_add(d0, kk * 2048);
          const uint64_t al = sdesc_add(ah, A_BYTES);
          const uint64_t bh = sdesc_add(ah, 2 * A_BYTES);
          const uint64_t bl = sdesc_add(ah, 2 * A_BYTES + C::B_BYTES);
          if (C::CAT) {  // A_hi [B_hi | B_lo] into both halves + A_lo B_hi into the first
            mma_bf16(tmem, ah, bh, id, (i > 0 || kk > 0) ? 1u : 0u);
            mma_bf16(tmem, al, bh, id_h, 1u);
          } else {
            mma_bf16(tmem, ah, bh, id, (i > 0 || kk > 0) ? 1u : 0u);
            mma_bf16(tmem, ah, bl, id, 1u);
            mma_bf16(tmem, al, bh, id, 1u);
          }
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
    if (!mbar_wait(&bars.done, 0, abort, a.wait)) *abort = 1;
    fence_after_sync();
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float *crow = a.c + (m_begin + gi) * a.ldc;
#pragma unroll 1
    for (int c0 = 0; c0 < N; c0 += 32) {
      float v[32];
      tmem_ld32(tmem + lane_base + c0, v);
      if (C::CAT) {
        float v2[32];
        tmem_ld32(tmem + lane_base + TN + c0, v2);
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] += v2[e];
      }
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
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (tid == 0 && bars.abort && a.err) atomicOr(a.err, 1);
}

}  // namespace

template <int TN>
int launch_tn(const GemmMaps &m, const GemmArgs3 &a, int tiles, int gram, int B,
              cudaStream_t st) {
  KVS_CUDA_TRY(set_smem_once(k_gemm3<TN>, G3<TN>::SMEM));
  if (tiles <= 0) return KVS_OK;
  k_gemm3<TN><<<dim3(tiles, B), 192, G3<TN>::SMEM, st>>>(m.ah, m.al, m.bh, m.bl, a, gram);
  KVS_LAUNCH_CHECK("k_gemm3");
  return KVS_OK;
}

int launch_gemm3_tc(const GemmMaps &m, const GemmArgs3 &a, int tiles_m, int gram, int B,
                    cudaStream_t st) {
  if (gram) return launch_tn<256>(m, a, gram_tiles<256>(tiles_m), 1, B, st);
  if (a.n_fixed == 128) return launch_tn<128>(m, a, tiles_m, 0, B, st);
  if (a.n_fixed == 64) return launch_tn<64>(m, a, tiles_m, 0, B, st);
  return KVS_ENOTSUP;
}

}  // namespace kvs
