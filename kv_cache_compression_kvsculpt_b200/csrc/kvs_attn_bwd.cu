// Key-tile attention kernel on tcgen05 tensor cores: the key gradient of the
// distillation loss and the attention importance of each key.
//
// "KVSculpt: KV Cache Compression as Distillation", section 2 "Loss
// Function" (gradient of output MSE + LSE matching with respect to the keys,
// for L-BFGS in "Key Optimization") and "Initialization" (keys ranked by
// attention importance).
//
// One CTA owns 128 keys of one problem and streams its training queries in
// tiles of 128.  Per tile, with A = exp(S - l_row):
//   S^T  = K Q^T                    K_hi Q_hi + K_lo Q_hi + K_hi Q_lo  (K in smem, N = 128)
//   DK:     dP^T = V Go^T           V_hi Go + V_lo Go  (V in TMEM, Go bf16; delta was
//                                   formed from the same rounded Go; N = 128)
//           dS = A (dP - delta_row) written as bf16 hi/lo over the S buffer in TMEM
//           dK += dS Q              dS_hi Q_hi + dS_hi Q_lo + dS_lo Q_hi
//   COLSUM: importance += sum over the tile's queries of A
// Near an optimum the key gradient is a small sum of large terms, so every
// product keeps about 16 significant bits.  A tcgen05.mma instruction costs
// about the same for any N up to 256, so the query tile is 128 wide.
// Tensor memory (512 columns): S at 0, dP at 128, dK at 256, V hi/lo after dK.
// The two row warpgroups split every tile: warpgroup g takes queries
// 64g .. 64g+63, and the dK product of its half starts as soon as it is done.
// Warp roles: warps 0-7 one thread per key row (warp w <-> TMEM lanes
// 32 (w % 4) ..), warp 8 TMA producer (also stages l and delta of the tile),
// warp 9 MMA issuer.  Shared memory: K hi/lo resident, two Q hi/lo stages, one
// Go stage, then the barriers (all dynamic, 1024-byte aligned).
#include <math.h>

#include "kvs_attn_tc.cuh"

namespace kvs {
namespace {

using namespace tc;

constexpr int BK = 128;      // keys per CTA
constexpr int BQ = BWD_BQ;   // queries per tile
constexpr int HQ = BQ / 2;   // queries per warpgroup
constexpr int NTHREADS = 320;
constexpr int NSQ = 2;       // query stages
constexpr float L2E = 1.4426950408889634f;
static_assert(BQ == 128, "tensor-memory layout assumes 128-query tiles");

template <int D, int MODE>
struct Bwd {
  static constexpr int KD = D / 64;
  static constexpr bool DK = (MODE == BWD_DK);
  static constexpr int K_BYTES = BK * D * 2;   // one copy of the key tile
  static constexpr int Q_BYTES = BQ * D * 2;   // one copy of a query tile
  static constexpr int OFF_Q = 2 * K_BYTES;    // K hi, K lo resident
  static constexpr int QSTAGE = 2 * Q_BYTES;   // Q hi, Q lo
  static constexpr int OFF_G = OFF_Q + NSQ * QSTAGE;
  static constexpr int OFF_BARS = OFF_G + (DK ? Q_BYTES : 0);
  static constexpr uint32_t TMEM_COLS = DK ? 512 : 128;
  static constexpr uint32_t COL_DP = 128;
  static constexpr uint32_t COL_DK = 256;
  static constexpr uint32_t COL_V = 256 + D;
};

struct BwdBars {
  uint64_t k_full, v_full;
  uint64_t q_full[NSQ], q_empty[NSQ];
  uint64_t g_full, g_empty;
  uint64_t sd_full, s_free;
  uint64_t ds_full[2];
  uint64_t done;
  uint32_t tmem;
  int abort;
  float lse2[NSQ][BQ];  // row lse in log2 units (+inf for rows outside the problem)
  union {
    float del[NSQ][BQ];  // DK
    float imp[BK];       // COLSUM: warpgroup 1's partial importance
  };
};

template <int D, int MODE>
constexpr int bwd_smem() {
  return Bwd<D, MODE>::OFF_BARS + (int)sizeof(BwdBars);
}

__device__ __forceinline__ void rows_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

template <int D, int MODE>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_attn_bwd(const __grid_constant__ CUtensorMap mKh, const __grid_constant__ CUtensorMap mKl,
               const __grid_constant__ CUtensorMap mQh, const __grid_constant__ CUtensorMap mQl,
               const __grid_constant__ CUtensorMap mG, BwdArgs a) {
  using C = Bwd<D, MODE>;
  extern __shared__ __align__(1024) unsigned char sm[];
  BwdBars &bars = *reinterpret_cast<BwdBars *>(sm + C::OFF_BARS);
  const int b = blockIdx.y;
  if (a.flt.skip(b)) return;
  const int64_t k_begin = a.k_off[b];
  const int nk = (int)(a.k_off[b + 1] - k_begin);
  const int k0 = blockIdx.x * BK;
  if (k0 >= nk) return;
  if (smem_u32(sm) & 1023) {  // the swizzled operand tiles need 1024-byte alignment
    if (threadIdx.x == 0 && a.err) atomicOr(a.err, 1);
    return;
  }
  const int64_t q_begin = a.q_off[b];
  const int nq = (int)(a.q_off[b + 1] - q_begin);
  const int nqt = (nq + BQ - 1) / BQ;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(&bars.k_full, 1);
    mbar_init(&bars.v_full, 2 * BK);
    for (int i = 0; i < NSQ; ++i) {
      mbar_init(&bars.q_full[i], 1);
      mbar_init(&bars.q_empty[i], 1 + 2 * BK);
    }
    mbar_init(&bars.g_full, 1);
    mbar_init(&bars.g_empty, 1);
    mbar_init(&bars.sd_full, 1);
    mbar_init(&bars.s_free, C::DK ? 1 : 2 * BK);
    mbar_init(&bars.ds_full[0], BK);
    mbar_init(&bars.ds_full[1], BK);
    mbar_init(&bars.done, 1);
    bars.abort = 0;
    fence_barrier_init();
  }
  if (warp == 9) tmem_alloc(&bars.tmem, C::TMEM_COLS);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = bars.tmem;
  volatile int *abort = &bars.abort;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int krow = (int)(k_begin + k0);
      mbar_arrive_expect_tx(&bars.k_full, 2 * C::K_BYTES);
      for (int r = 0; r < C::KD; ++r) {
        tma_load_2d(sm + r * BK * 128, &mKh, &bars.k_full, 64 * r, krow);
        tma_load_2d(sm + C::K_BYTES + r * BK * 128, &mKl, &bars.k_full, 64 * r, krow);
      }
    }
    int q_issued = 0, g_issued = 0;
    bool ok = true;
    for (int i = 0; ok && i < nqt; ++i) {
      const int st = i % NSQ;
      if (i >= NSQ)
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&bars.q_empty[st], ((i / NSQ) - 1) & 1, abort));
      if (!ok) break;
      for (int e = lane; e < BQ; e += 32) {
        const int q = i * BQ + e;
        const bool v = q < nq;
        bars.lse2[st][e] = v ? a.lse[q_begin + q] * L2E : INFINITY;
        if (C::DK) bars.del[st][e] = v ? a.delta[q_begin + q] : 0.f;
      }
      __syncwarp();
      const int qrow = (int)(q_begin + i * BQ);
      if (lane == 0) {
        q_issued = i + 1;
        unsigned char *base = sm + C::OFF_Q + st * C::QSTAGE;
        mbar_arrive_expect_tx(&bars.q_full[st], C::QSTAGE);
        for (int r = 0; r < C::KD; ++r) {
          tma_load_2d(base + r * BQ * 128, &mQh, &bars.q_full[st], 64 * r, qrow);
          tma_load_2d(base + C::Q_BYTES + r * BQ * 128, &mQl, &bars.q_full[st], 64 * r, qrow);
        }
      }
      if (C::DK) {
        // Go of tile i once dP of tile i-1 has read the previous one
        if (lane == 0) {
          if (i >= 1 && !mbar_wait(&bars.g_empty, (i - 1) & 1, abort)) {
            ok = false;
          } else {
            g_issued = i + 1;
            mbar_arrive_expect_tx(&bars.g_full, C::Q_BYTES);
            for (int r = 0; r < C::KD; ++r)
              tma_load_2d(sm + C::OFF_G + r * BQ * 128, &mG, &bars.g_full, 64 * r, qrow);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
    }
    if (!ok) *abort = 1;
    if (lane == 0 && *abort) {  // let issued copies land before shared memory is released
      mbar_wait(&bars.k_full, 0);
      for (int i = (q_issued > NSQ ? q_issued - NSQ : 0); i < q_issued; ++i)
        mbar_wait(&bars.q_full[i % NSQ], (i / NSQ) & 1);
      if (g_issued > 0) mbar_wait(&bars.g_full, (g_issued - 1) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(BK, BQ, false, false);
      const uint32_t id_dk = idesc_bf16(BK, D, false, true);
      bool ok = mbar_wait(&bars.k_full, 0, abort);
      if (C::DK) ok = ok && mbar_wait(&bars.v_full, 0, abort);
      fence_after_sync();
      const uint64_t kh0 = sdesc(smem_u32(sm), 16, 1024), kl0 = sdesc_add(kh0, C::K_BYTES);
      const uint64_t gd0 = sdesc(smem_u32(sm + C::OFF_G), 16, 1024);
      const uint32_t tv_hi = tmem + C::COL_V, tv_lo = tmem + C::COL_V + D / 2;
      for (int i = 0; ok && i < nqt; ++i) {
        const int st = i % NSQ;
        if (!mbar_wait(&bars.q_full[st], (i / NSQ) & 1, abort)) { ok = false; break; }
        if (C::DK && !mbar_wait(&bars.g_full, i & 1, abort)) { ok = false; break; }
        // the S and dP buffers are free once dK (or the importance rows) of tile i-1 is done
        if (i >= 1 && !mbar_wait(&bars.s_free, (i - 1) & 1, abort)) { ok = false; break; }
        fence_after_sync();
        const uint64_t qh0 = sdesc(smem_u32(sm + C::OFF_Q + st * C::QSTAGE), 16, 1024);
        const uint64_t ql0 = sdesc_add(qh0, C::Q_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ok_ = (kk >> 2) * (BK * 128) + (kk & 3) * 32;
          const uint32_t oq = (kk >> 2) * (BQ * 128) + (kk & 3) * 32;
          const uint64_t kh = sdesc_add(kh0, ok_), kl = sdesc_add(kl0, ok_);
          const uint64_t qh = sdesc_add(qh0, oq), ql = sdesc_add(ql0, oq);
          mma_bf16(tmem, kh, qh, id_s, kk > 0 ? 1u : 0u);
          mma_bf16(tmem, kl, qh, id_s, 1u);
          mma_bf16(tmem, kh, ql, id_s, 1u);
          if (C::DK) {
            const uint64_t gd = sdesc_add(gd0, oq);
            mma_bf16_ts(tmem + C::COL_DP, tv_hi + kk * 8, gd, id_s, kk > 0 ? 1u : 0u);
            mma_bf16_ts(tmem + C::COL_DP, tv_lo + kk * 8, gd, id_s, 1u);
          }
        }
        mma_commit(&bars.sd_full);
        if (!C::DK) {
          mma_commit(&bars.q_empty[st]);
          continue;
        }
        mma_commit(&bars.g_empty);
        // dK += dS Q, one half of the tile's queries per warpgroup as it finishes
        const uint64_t qm0 = sdesc(smem_u32(sm + C::OFF_Q + st * C::QSTAGE), BQ * 128, 1024);
        const uint64_t qml0 = sdesc_add(qm0, C::Q_BYTES);
        for (int g = 0; g < 2; ++g) {
          if (!mbar_wait(&bars.ds_full[g], i & 1, abort)) { ok = false; break; }
          fence_after_sync();
          const uint32_t tds = tmem + g * HQ;  // dS hi at +0, lo at +HQ/2 columns
#pragma unroll
          for (int kk = 0; kk < HQ / 16; ++kk) {
            const uint32_t off = (uint32_t)(g * (HQ / 16) + kk) * 2048;  // 16 query rows
            const uint64_t qh = sdesc_add(qm0, off), ql = sdesc_add(qml0, off);
            const uint32_t acc = (i > 0 || g > 0 || kk > 0) ? 1u : 0u;
            mma_bf16_ts(tmem + C::COL_DK, tds + kk * 8, qh, id_dk, acc);
            mma_bf16_ts(tmem + C::COL_DK, tds + kk * 8, ql, id_dk, 1u);
            mma_bf16_ts(tmem + C::COL_DK, tds + HQ / 2 + kk * 8, qh, id_dk, 1u);
          }
        }
        if (!ok) break;
        mma_commit(&bars.q_empty[st]);
        mma_commit(&bars.s_free);
      }
      mma_commit(&bars.done);
      if (!ok) *abort = 1;
      mbar_wait(&bars.done, 0);  // every MMA of this CTA has completed
    }
  } else {
    // --------------------------------------------------------- key rows
    const int wg = warp >> 2;  // warpgroup: queries 64 wg .. 64 wg + 63 of every tile
    const int row = tid & (BK - 1);
    const int kr = k0 + row;
    const bool kvalid = kr < nk;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    if (C::DK) {
      // this warpgroup's half of the value row (hi, lo) into tensor memory: the A
      // operand of dP^T = V Go^T
      const uint4 *vh = reinterpret_cast<const uint4 *>(a.v_hi + (k_begin + kr) * D);
      const uint4 *vl = reinterpret_cast<const uint4 *>(a.v_lo + (k_begin + kr) * D);
#pragma unroll 1
      for (int c0 = wg * 32; c0 < D / 2; c0 += 64) {
        uint32_t wh[32], wl[32];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint4 h = kvalid ? vh[c0 / 4 + e] : make_uint4(0, 0, 0, 0);
          const uint4 l = kvalid ? vl[c0 / 4 + e] : make_uint4(0, 0, 0, 0);
          wh[4 * e] = h.x; wh[4 * e + 1] = h.y; wh[4 * e + 2] = h.z; wh[4 * e + 3] = h.w;
          wl[4 * e] = l.x; wl[4 * e + 1] = l.y; wl[4 * e + 2] = l.z; wl[4 * e + 3] = l.w;
        }
        tmem_st32u(tmem + lane_base + C::COL_V + c0, wh);
        tmem_st32u(tmem + lane_base + C::COL_V + D / 2 + c0, wl);
      }
      tmem_wait_st();
      fence_before_sync();
      mbar_arrive(&bars.v_full);
    }
    const float sl2 = a.scale * L2E;
    const int cbase = wg * HQ;  // this warpgroup's first column of the tile
    float imp = 0.f;
    bool ok = true;
    for (int i = 0; i < nqt; ++i) {
      const int st = i % NSQ;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars.sd_full, i & 1, abort));
      // the tile's l and delta were staged by the producer lanes: acquire them directly
      ok = ok && __all_sync(0xffffffffu, mbar_wait(&bars.q_full[st], (i / NSQ) & 1, abort));
      if (!ok) break;
      fence_after_sync();
      float s[HQ];
      tmem_ld32(tmem + lane_base + cbase, s);
      tmem_ld32(tmem + lane_base + cbase + 32, s + 32);
      const int qvalid = nq - i * BQ - cbase;  // valid columns of this half
      if (!C::DK) {
#pragma unroll
        for (int c = 0; c < HQ; ++c)
          imp += (c < qvalid) ? exp2f(fmaf(s[c], sl2, -bars.lse2[st][cbase + c])) : 0.f;
        fence_before_sync();
        mbar_arrive(&bars.s_free);
      } else {
        float dp[HQ];
        tmem_ld32(tmem + lane_base + C::COL_DP + cbase, dp);
        tmem_ld32(tmem + lane_base + C::COL_DP + cbase + 32, dp + 32);
        uint32_t hh[HQ / 2], ll[HQ / 2];
#pragma unroll
        for (int c2 = 0; c2 < HQ / 2; ++c2) {
          float v[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int c = 2 * c2 + u;
            const float p = exp2f(fmaf(s[c], sl2, -bars.lse2[st][cbase + c]));
            v[u] = (kvalid && c < qvalid) ? p * (dp[c] - bars.del[st][cbase + c]) : 0.f;
          }
          split_pack(v[0], v[1], hh[c2], ll[c2]);
        }
        // dS (hi, lo) over this half of the S buffer: the A operand of dK += dS Q
        tmem_st32u(tmem + lane_base + cbase, hh);
        tmem_st32u(tmem + lane_base + cbase + HQ / 2, ll);
        tmem_wait_st();
        fence_before_sync();
        mbar_arrive(&bars.ds_full[wg]);
      }
      mbar_arrive(&bars.q_empty[st]);
    }
    if (!ok) *abort = 1;
    if (C::DK) {
      if (!mbar_wait(&bars.done, 0, abort)) *abort = 1;
      fence_after_sync();
#pragma unroll 1
      for (int c0 = wg * (D / 2); c0 < (wg + 1) * (D / 2); c0 += 32) {
        float o[32];
        tmem_ld32(tmem + lane_base + C::COL_DK + c0, o);
        if (kvalid) {
          float4 *dst = reinterpret_cast<float4 *>(a.dk + (k_begin + kr) * D + c0);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(o[4 * e] * a.scale, o[4 * e + 1] * a.scale,
                                 o[4 * e + 2] * a.scale, o[4 * e + 3] * a.scale);
        }
      }
    } else {
      if (!mbar_wait(&bars.done, 0, abort)) *abort = 1;
      if (wg == 1) bars.imp[row] = imp;
      rows_sync();
      if (wg == 0 && kvalid) a.imp[k_begin + kr] = imp + bars.imp[row];
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 9) {
    fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (tid == 0 && bars.abort && a.err) atomicOr(a.err, 1);
}

}  // namespace

template <int D, int MODE>
int launch_bwd_tc(const BwdMaps &m, const BwdArgs &a, int max_tiles, int B, cudaStream_t st) {
  constexpr int smem = bwd_smem<D, MODE>();
  static_assert(smem <= 232448, "shared memory");
  auto kern = k_attn_bwd<D, MODE>;
  KVS_CUDA_TRY(set_smem_once(kern, smem));
  kern<<<dim3(max_tiles, B), NTHREADS, smem, st>>>(m.kh, m.kl, m.qh, m.ql, m.g, a);
  KVS_LAUNCH_CHECK("k_attn_bwd");
  return KVS_OK;
}

template int launch_bwd_tc<64, BWD_DK>(const BwdMaps &, const BwdArgs &, int, int, cudaStream_t);
template int launch_bwd_tc<128, BWD_DK>(const BwdMaps &, const BwdArgs &, int, int, cudaStream_t);
template int launch_bwd_tc<64, BWD_COLSUM>(const BwdMaps &, const BwdArgs &, int, int, cudaStream_t);
template int launch_bwd_tc<128, BWD_COLSUM>(const BwdMaps &, const BwdArgs &, int, int, cudaStream_t);

}  // namespace kvs
