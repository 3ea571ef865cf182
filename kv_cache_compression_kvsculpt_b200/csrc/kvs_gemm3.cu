// Normal equations of the ridge fit on tcgen05 tensor cores:
// G = A^T A + lambda I and R = A^T Y ("KVSculpt: KV Cache Compression as
// Distillation", section 2 "Value Optimization": values solved in closed form
// by ridge regression given the attention weights A of the current keys).
//
// A (softmax weights, [padded n_q, k] per problem) and Y are held as bf16
// hi/lo pairs; each product takes three bf16 MMAs (hi.hi + hi.lo + lo.hi)
// with fp32 accumulation in TMEM, which keeps about 16 significant bits of
// each operand.  Both operands are read MN-major (keys / value columns
// contiguous), the contraction runs over training queries.
// A^T Y (k_gemm3): one CTA per 128 x d output tile, [Y_hi | Y_lo] side by side
// as one N = 2d operand, stages of 64 queries.
// Gram (k_gram2): one CTA per 256 x 256 tile of the lower triangle (which the
// Cholesky reads), two 128-row accumulators against one 256-column block,
// stages of 32 queries.
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
  static constexpr int NS = 3;
  static constexpr int SMEM = NS * STAGE + 1024;
  // B_hi and B_lo side by side as one operand of N = 2 TN for A_hi, and B_hi alone
  // (N = TN) for A_lo: two instructions per 16-row step instead of three, into two
  // summed halves
  static constexpr int MMA_N = 2 * TN;
  static constexpr uint32_t TMEM_COLS = MMA_N < 32 ? 32 : MMA_N;
  static_assert(TN <= 128, "N = 2 TN <= 256");
};
constexpr int NSMAX = 3;

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
            GemmArgs3 a) {
  using C = G3<TN>;
  constexpr int NS = C::NS;
  extern __shared__ unsigned char smraw[];
  unsigned char *sm = (unsigned char *)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
  __shared__ GBars bars;
  const int b = blockIdx.y;
  const int64_t m_begin = a.m_off[b];
  const int nk = (int)(a.m_off[b + 1] - m_begin);
  const int T = (nk + TM - 1) / TM;
  const int ti = blockIdx.x, tj = 0;
  if (ti >= T) return;
  const int N = TN;                             // output columns (TN = d)
  const int ncols = a.n_fixed;                  // valid output columns
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
      const uint32_t id_h = idesc_bf16(TM, TN, true, true);  // B_hi alone
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
          // A_hi [B_hi | B_lo] into both halves + A_lo B_hi into the first
          mma_bf16(tmem, ah, bh, id, (i > 0 || kk > 0) ? 1u : 0u);
          mma_bf16(tmem, al, bh, id_h, 1u);
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
      {
        float v2[32];
        tmem_ld32(tmem + lane_base + TN + c0, v2);
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] += v2[e];
      }
      if (gi < nk && nkt > 0) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int gc = tj * TN + c0 + e;
          if (gc < ncols) crow[gc] = v[e];
        }
      }
    }
    if (nkt == 0 && gi < nk)
      for (int gc = tj * TN; gc < min(tj * TN + N, ncols); ++gc) crow[gc] = 0.f;
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (tid == 0 && bars.abort && a.err) atomicOr(a.err, 1);
}

// ---------------------------------------------------------------- Gram pairs
// The Gram matrix in 256 x 256 tiles: one CTA takes two 128-row blocks of keys
// (rows 256 m .. 256 m + 255, two TMEM accumulators of 256 columns, all of tensor
// memory) against one 256-column block J <= m, so each stage of 32 training
// queries brings 64 KB of operands (A hi / lo of both row blocks and of the column
// block) for 12 MMAs of N = 256: half again the products per byte of the single
// 128 x 256 tile, whose operand stream the L2 does not keep up with.
constexpr int GKQ = 32;                              // training queries per stage
constexpr int GA_BYTES = GKQ * TM * 2;               // one 32 x 128 bf16 tile
constexpr int GB_BYTES = GKQ * 256 * 2;              // one 32 x 256 bf16 tile
constexpr int GSTAGE = 4 * GA_BYTES + 2 * GB_BYTES;  // A0 hi, A0 lo, A1 hi, A1 lo, B hi, B lo
constexpr int GNS = 3;
constexpr int GSMEM = GNS * GSTAGE + 1024;
static_assert(GSMEM <= 227 * 1024, "shared memory");

// Pair tile t of a problem with P = ceil(T / 2) row pairs: the t-th (m, J <= m) in
// row-major order.
__host__ __device__ inline bool pair_tile(int t, int P, int *m, int *J) {
  for (int i = 0; i < P; ++i) {
    if (t <= i) {
      *m = i;
      *J = t;
      return true;
    }
    t -= i + 1;
  }
  return false;
}

__global__ void __launch_bounds__(192, 1)
    k_gram2(const __grid_constant__ CUtensorMap mAh, const __grid_constant__ CUtensorMap mAl,
            GemmArgs3 a) {
  extern __shared__ unsigned char smraw[];
  unsigned char *sm = (unsigned char *)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
  __shared__ GBars bars;
  const int b = blockIdx.y;
  const int64_t m_begin = a.m_off[b];
  const int nk = (int)(a.m_off[b + 1] - m_begin);
  const int T = (nk + TM - 1) / TM;
  int pm, pj;
  if (!pair_tile(blockIdx.x, (T + 1) / 2, &pm, &pj)) return;
  const int64_t ka0 = a.a_pad_off[b];
  const int kq = (int)(a.a_pad_off[b + 1] - ka0);  // padded query rows (multiple of 128)
  const int nkt = kq / GKQ;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < GNS; ++i) {
      mbar_init(&bars.full[i], 1);
      mbar_init(&bars.empty[i], 1);
    }
    mbar_init(&bars.done, 1);
    bars.abort = 0;
    fence_barrier_init();
  }
  if (warp == 5) tmem_alloc(&bars.tmem, 512);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = bars.tmem;
  volatile int *abort = &bars.abort;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nkt; ++i) {
        const int st = i % GNS;
        if (i >= GNS && !mbar_wait(&bars.empty[st], ((i / GNS) - 1) & 1, abort, a.wait)) {
          *abort = 1;
          break;
        }
        issued = i + 1;
        unsigned char *base = sm + st * GSTAGE;
        mbar_arrive_expect_tx(&bars.full[st], GSTAGE);
        const int y = (int)(ka0 + i * GKQ);
        for (int u = 0; u < 2; ++u)
          for (int r = 0; r < 2; ++r) {
            const int x = (2 * pm + u) * TM + 64 * r;
            tma_load_2d(base + (2 * u) * GA_BYTES + r * GKQ * 128, &mAh, &bars.full[st], x, y);
            tma_load_2d(base + (2 * u + 1) * GA_BYTES + r * GKQ * 128, &mAl, &bars.full[st], x, y);
          }
        for (int r = 0; r < 4; ++r) {
          const int x = pj * 256 + 64 * r;
          tma_load_2d(base + 4 * GA_BYTES + r * GKQ * 128, &mAh, &bars.full[st], x, y);
          tma_load_2d(base + 4 * GA_BYTES + GB_BYTES + r * GKQ * 128, &mAl, &bars.full[st], x, y);
        }
      }
      if (*abort)
        for (int i = (issued > GNS ? issued - GNS : 0); i < issued; ++i)
          mbar_wait(&bars.full[i % GNS], (i / GNS) & 1);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id = idesc_bf16(TM, 256, true, true);
      bool ok = true;
      for (int i = 0; i < nkt; ++i) {
        const int st = i % GNS;
        if (!mbar_wait(&bars.full[st], (i / GNS) & 1, abort, a.wait)) { ok = false; break; }
        fence_after_sync();
        const uint64_t d0 = sdesc(smem_u32(sm + st * GSTAGE), GKQ * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < GKQ / 16; ++kk) {
          const uint64_t bh = sdesc_add(d0, 4 * GA_BYTES + kk * 2048);
          const uint64_t bl = sdesc_add(bh, GB_BYTES);
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const uint64_t ah = sdesc_add(d0, 2 * u * GA_BYTES + kk * 2048);
            const uint64_t al = sdesc_add(ah, GA_BYTES);
            const uint32_t acc = tmem + 256 * u;
            mma_bf16(acc, ah, bh, id, (i > 0 || kk > 0) ? 1u : 0u);
            mma_bf16(acc, ah, bl, id, 1u);
            mma_bf16(acc, al, bh, id, 1u);
          }
        }
        mma_commit(&bars.empty[st]);
      }
      mma_commit(&bars.done);
      if (!ok) *abort = 1;
      mbar_wait(&bars.done, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // thread = row of each 128-row block (its TMEM lane)
    if (!mbar_wait(&bars.done, 0, abort, a.wait)) *abort = 1;
    fence_after_sync();
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    if (!*abort) {
#pragma unroll 1
      for (int u = 0; u < 2; ++u) {
        const int gi = (2 * pm + u) * TM + tid;
        float *crow = a.c + (m_begin + gi) * a.ldc;
#pragma unroll 1
        for (int c0 = 0; c0 < 256; c0 += 32) {
          float v[32];
          tmem_ld32(tmem + lane_base + 256 * u + c0, v);
          if (gi < nk && nkt > 0) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int gc = pj * 256 + c0 + e;
              if (gc < nk) crow[gc] = v[e] + (gc == gi ? a.diag : 0.f);
            }
          }
        }
        if (nkt == 0 && gi < nk)
          for (int gc = pj * 256; gc < min(pj * 256 + 256, nk); ++gc)
            crow[gc] = gc == gi ? a.diag : 0.f;
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
  if (tid == 0 && bars.abort && a.err) atomicOr(a.err, 1);
}

}  // namespace

template <int TN>
int launch_tn(const GemmMaps &m, const GemmArgs3 &a, int tiles, int B, cudaStream_t st) {
  KVS_CUDA_TRY(set_smem_once(k_gemm3<TN>, G3<TN>::SMEM));
  if (tiles <= 0) return KVS_OK;
  k_gemm3<TN><<<dim3(tiles, B), 192, G3<TN>::SMEM, st>>>(m.ah, m.al, m.bh, m.bl, a);
  KVS_LAUNCH_CHECK("k_gemm3");
  return KVS_OK;
}

int launch_gram2_tc(const GemmMaps &m, const GemmArgs3 &a, int tiles_m, int B, cudaStream_t st) {
  KVS_CUDA_TRY(set_smem_once(k_gram2, GSMEM));
  const int P = (tiles_m + 1) / 2;
  const int tiles = P * (P + 1) / 2;
  if (tiles <= 0) return KVS_OK;
  k_gram2<<<dim3(tiles, B), 192, GSMEM, st>>>(m.ah, m.al, a);
  KVS_LAUNCH_CHECK("k_gram2");
  return KVS_OK;
}

int launch_gemm3_tc(const GemmMaps &m, const GemmArgs3 &a, int tiles_m, int B, cudaStream_t st) {
  if (a.n_fixed == 128) return launch_tn<128>(m, a, tiles_m, B, st);
  if (a.n_fixed == 64) return launch_tn<64>(m, a, tiles_m, B, st);
  return KVS_ENOTSUP;
}

}  // namespace kvs
