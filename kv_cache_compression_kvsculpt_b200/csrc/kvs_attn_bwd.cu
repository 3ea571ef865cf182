// Key-tile attention kernel on tcgen05 tensor cores: the key gradient of the
// distillation loss and the attention importance of each key.
//
// "KVSculpt: KV Cache Compression as Distillation", section 2 "Loss
// Function" (gradient of output MSE + LSE matching with respect to the keys,
// for L-BFGS in "Key Optimization") and "Initialization" (keys ranked by
// attention importance).
//
// One CTA owns 128 keys of one problem and streams its training queries in
// tiles of 64.  Per tile, with A = exp(S - l_row):
//   S^T  = K Q^T      K_hi [Q_hi | Q_lo] (one N = 128 product into two column
//                     halves) + K_lo Q_hi (into the first half); S = sum of the
//                     halves, i.e. K_hi Q_hi + K_hi Q_lo + K_lo Q_hi  (K in smem)
//   DK:  dP^T = V Go^T  V_hi Go + V_lo Go  (fp16: V split by the row threads into
//                       TMEM, Go written by the loss forward, scaled into fp16's
//                       range; delta was formed from the same rounded Go)
//        dS = A (dP - delta_row), written as bf16 hi/lo over the tile's dP buffer
//        dK += dS Q     dS_hi Q_hi + dS_hi Q_lo + dS_lo Q_hi  (Q as the N-major operand)
//   COLSUM: importance += sum over the tile's queries of A
// Near an optimum the key gradient is a small sum of large terms, so every
// product keeps about 16 significant bits.  Each tcgen05.mma instruction costs
// about the same for any N up to 128, so the score product takes Q_hi and Q_lo
// side by side: two instructions per 16-deep step instead of three.
// Tensor memory (512 columns, DK): one S buffer (two 64-column halves) at 0,
// dP / dS buffers at 128 and 192 (one per tile parity), dK at 256, V hi at 384,
// V lo at 384 + D/2.  COLSUM: two S buffers at 0 and 128.
// DK issue order: S(i), dP(i), dK(i-1): the next tile's scores run while the
// row threads form dS of the last tile, and dP(i + 2) reuses the buffer of dS(i)
// once dK(i) has drained it, behind S(i + 2) in the tensor pipe.
// Two row warpgroups take alternate query tiles.  Warp roles: warps 0-7 one
// thread per key row (warp w <-> TMEM lanes 32 (w % 4) ..), warp 8 TMA
// producer (also stages l and delta of the tile), warp 9 MMA issuer.
#include <math.h>

#include "kvs_attn_tc.cuh"

namespace kvs {
namespace {

using namespace tc;

constexpr int BK = 128;  // keys per CTA
constexpr int BQ = BWD_BQ;  // queries per tile
constexpr int NTHREADS = 320;
constexpr int NSTAGE = 3;  // query-tile stages in flight
constexpr float L2E = 1.4426950408889634f;

template <int D, int MODE>
struct Bwd {
  static constexpr int KD = D / 64;
  static constexpr bool DK = (MODE == BWD_DK);
  static constexpr int NS = NSTAGE;
  static constexpr int K_BYTES = BK * D * 2;   // one copy of the key tile
  static constexpr int QB = BQ * 128;          // one 64-column box of a query tile
  static constexpr int Q_BYTES = KD * QB;      // one copy of a query tile
  // stage: per 64-column box r, Q_hi then Q_lo (the score product reads them as one
  // N = 2 BQ operand); then the Go boxes
  static constexpr int STAGE = (DK ? 3 : 2) * Q_BYTES;
  static constexpr int OFF_GO = 2 * Q_BYTES;
  static constexpr int OFF_ST = 2 * K_BYTES;
  static constexpr int BYTES = OFF_ST + NS * STAGE;
  static constexpr int SMEM = BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = DK ? 512 : 256;
  static constexpr uint32_t COL_DP = 128;      // DK: dP / dS buffers, 64 columns each
  static constexpr uint32_t COL_DK = 256;
  static constexpr uint32_t COL_V = 384;
};

struct BwdBars {
  uint64_t k_full, v_full;
  uint64_t q_full[NSTAGE], q_empty[NSTAGE];
  uint64_t s_full[2];               // S of tile i done: [i & 1]
  uint64_t s_free[2];               // S read by the rows: DK [0] (one buffer), COLSUM [i & 1]
  uint64_t dp_full[2], ds_full[2];  // DK, per tile parity
  uint64_t dk_done[NSTAGE];         // DK: dK of tile i done, [i % NSTAGE]; frees the stage
  uint64_t done;                    // the work item's products are done (once per item)
  uint64_t dk_free;                 // DK: the rows have read the item's dK (once per item)
  uint64_t all_done;                // every MMA of the CTA has completed
  uint32_t tmem;
  int abort;
  __align__(16) float lse2[NSTAGE][BQ];  // row lse in log2 units (+inf past the problem)
  __align__(16) float del[NSTAGE][BQ];
  float imp[BK];       // COLSUM: warpgroup 1's partial importance
};

__device__ __forceinline__ void rows_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

template <int D, int MODE>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_attn_bwd(const __grid_constant__ CUtensorMap mKh, const __grid_constant__ CUtensorMap mKl,
               const __grid_constant__ CUtensorMap mQh, const __grid_constant__ CUtensorMap mQl,
               const __grid_constant__ CUtensorMap mG, BwdArgs a) {
  using C = Bwd<D, MODE>;
  extern __shared__ unsigned char smraw[];
  unsigned char *sm = (unsigned char *)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
  __shared__ BwdBars bars;
  const int b = blockIdx.y;
  if (a.flt.skip(b)) return;
  const int64_t k_begin = a.k_off[b];
  const int nk = (int)(a.k_off[b + 1] - k_begin);
  // work items: key tiles blockIdx.x, blockIdx.x + gridDim.x, ... of problem b, one
  // after another (each over the same query range); the next item's key tile loads
  // while the current item's last products and epilogue run
  const int nkt = (nk + BK - 1) / BK;
  const int n_items = (int)blockIdx.x < nkt ? (nkt - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  if (n_items == 0) return;
  const int64_t q_begin = a.q_off[b];
  const int nq = (int)(a.q_off[b + 1] - q_begin);
  // split z of the problem's query tiles: tiles t0 .. t0 + nqt - 1 (DK partial sums)
  const int nqt_all = (nq + BQ - 1) / BQ;
  const int per = (nqt_all + a.nsplit - 1) / a.nsplit;
  const int t0 = blockIdx.z * per;
  const int nqt = max(0, min(nqt_all, t0 + per) - t0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(&bars.k_full, 1);
    mbar_init(&bars.v_full, 2 * BK);
    for (int i = 0; i < NSTAGE; ++i) {
      mbar_init(&bars.q_full[i], 2);  // the copies' arrival and the staged l / delta
      mbar_init(&bars.q_empty[i], BK);  // COLSUM: the rows are done with the stage
      mbar_init(&bars.dk_done[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.s_free[i], BK);
      mbar_init(&bars.dp_full[i], 1);
      mbar_init(&bars.ds_full[i], BK);
    }
    mbar_init(&bars.done, 1);
    mbar_init(&bars.dk_free, 2 * BK);
    mbar_init(&bars.all_done, 1);
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
    int issued = 0, k_issued = 0;
    bool pok = true;
    for (int m = 0; pok && m < n_items; ++m) {
      const int k0 = ((int)blockIdx.x + m * (int)gridDim.x) * BK, I0 = m * nqt;
      // the item's key tile, once the previous item's last score product has read
      // the buffer
      if (lane == 0) {
        if (m > 0 && nqt > 0 &&
            !mbar_wait(&bars.s_full[(I0 - 1) & 1], ((I0 - 1) >> 1) & 1, abort, a.wait))
          *abort = 1;
        if (!*abort) {
          k_issued = m + 1;
          const int krow = (int)(a.k_pad[b] + k0);
          mbar_arrive_expect_tx(&bars.k_full, 2 * C::K_BYTES);
          for (int r = 0; r < C::KD; ++r) {
            tma_load_2d(sm + r * BK * 128, &mKh, &bars.k_full, 64 * r, krow);
            tma_load_2d(sm + C::K_BYTES + r * BK * 128, &mKl, &bars.k_full, 64 * r, krow);
          }
        }
      }
      if (__any_sync(0xffffffffu, *abort)) {
        pok = false;
        break;
      }
      for (int i = 0; i < nqt; ++i) {
        const int I = I0 + i, st = I % C::NS;  // I counts query tiles over the CTA's items
        if (I >= C::NS) {
          // DK: the last product that reads the stage is dK of tile I - NS, which starts
          // after the rows are done with its l and delta; COLSUM: only S reads it, and
          // the rows arrive after S has completed
          uint64_t *fr = C::DK ? &bars.dk_done[st] : &bars.q_empty[st];
          const bool w = __all_sync(0xffffffffu, mbar_wait(fr, ((I / C::NS) - 1) & 1, abort, a.wait));
          if (!w) {
            *abort = 1;
            pok = false;
            break;
          }
        }
        // the tile's copies first, then its l and delta (their loads overlap the copies)
        if (lane == 0) {
          issued = I + 1;
          unsigned char *base = sm + C::OFF_ST + st * C::STAGE;
          const int qrow = (int)(a.q_pad[b] + (t0 + i) * BQ);
          mbar_arrive_expect_tx(&bars.q_full[st], C::STAGE);
          for (int r = 0; r < C::KD; ++r) {
            tma_load_2d(base + 2 * r * C::QB, &mQh, &bars.q_full[st], 64 * r, qrow);
            tma_load_2d(base + (2 * r + 1) * C::QB, &mQl, &bars.q_full[st], 64 * r, qrow);
            if (C::DK)
              tma_load_2d(base + C::OFF_GO + r * C::QB, &mG, &bars.q_full[st], 64 * r, qrow);
          }
        }
        for (int e = lane; e < BQ; e += 32) {
          const int q = (t0 + i) * BQ + e;
          const bool v = q < nq;
          bars.lse2[st][e] = v ? a.lse[q_begin + q] * L2E : INFINITY;
          bars.del[st][e] = (v && C::DK) ? a.delta[q_begin + q] : 0.f;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.q_full[st]);
      }
    }
    if (lane == 0 && *abort) {  // let issued copies land before shared memory is released
      if (k_issued) mbar_wait(&bars.k_full, (k_issued - 1) & 1);
      for (int I = (issued > C::NS ? issued - C::NS : 0); I < issued; ++I)
        mbar_wait(&bars.q_full[I % C::NS], (I / C::NS) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s2 = idesc_bf16(BK, 2 * BQ, false, false);  // K_hi [Q_hi | Q_lo]
      const uint32_t id_s1 = idesc_bf16(BK, BQ, false, false);      // K_lo Q_hi
      const uint32_t id_dp = idesc_f16(BK, BQ, false, false);       // V Go (fp16)
      const uint32_t id_dk = idesc_bf16(BK, D, false, true);
      const uint64_t kh0 = sdesc(smem_u32(sm), 16, 1024), kl0 = sdesc_add(kh0, C::K_BYTES);
      const uint32_t tv_hi = tmem + C::COL_V, tv_lo = tmem + C::COL_V + D / 2;
      // S^T of tile I into the S buffer at column col
      auto issue_s = [&](int I, uint32_t col) {
        const uint32_t base = smem_u32(sm + C::OFF_ST + (I % C::NS) * C::STAGE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int r = kk >> 2;
          const uint32_t in = (kk & 3) * 32;
          const uint64_t kh = sdesc_add(kh0, r * (BK * 128) + in), kl = sdesc_add(kl0, r * (BK * 128) + in);
          const uint64_t qcat = sdesc(base + 2 * r * C::QB + in, 16, 1024);  // Q_hi box r, Q_lo box r
          mma_bf16(tmem + col, kh, qcat, id_s2, kk > 0 ? 1u : 0u);
          mma_bf16(tmem + col, kl, qcat, id_s1, 1u);  // first N = BQ rows: Q_hi
        }
      };
      // dP^T of tile I into dP buffer I & 1
      auto issue_dp = [&](int I) {
        const uint32_t base = smem_u32(sm + C::OFF_ST + (I % C::NS) * C::STAGE + C::OFF_GO);
        const uint32_t col = C::COL_DP + (I & 1) * BQ;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t gd = sdesc(base + (kk >> 2) * C::QB + (kk & 3) * 32, 16, 1024);
          mma_bf16_ts(tmem + col, tv_hi + kk * 8, gd, id_dp, kk > 0 ? 1u : 0u);
          mma_bf16_ts(tmem + col, tv_lo + kk * 8, gd, id_dp, 1u);
        }
      };
      // dK += dS(I) Q(I): dS hi / lo over dP buffer I & 1, Q as the N-major operand
      // (64-wide d blocks of Q_hi 2 QB apart, Q_lo one box further); `first`: the
      // item's first tile, whose product overwrites dK once the rows have read the
      // previous item's dK
      auto issue_dk = [&](int I, bool first, int m) -> bool {
        const int db = I & 1;
        if (!mbar_wait(&bars.ds_full[db], (I >> 1) & 1, abort, a.wait)) return false;
        if (first && m > 0 && !mbar_wait(&bars.dk_free, (m - 1) & 1, abort, a.wait)) return false;
        fence_after_sync();
        const uint32_t base = smem_u32(sm + C::OFF_ST + (I % C::NS) * C::STAGE);
        const uint64_t qh0 = sdesc(base, 2 * C::QB, 1024), ql0 = sdesc(base + C::QB, 2 * C::QB, 1024);
        const uint32_t tds = tmem + C::COL_DP + db * BQ;  // dS hi at +0, lo at +BQ/2 columns
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk) {
          const uint64_t qh = sdesc_add(qh0, kk * 2048), ql = sdesc_add(ql0, kk * 2048);
          mma_bf16_ts(tmem + C::COL_DK, tds + kk * 8, qh, id_dk, (!first || kk > 0) ? 1u : 0u);
          mma_bf16_ts(tmem + C::COL_DK, tds + kk * 8, ql, id_dk, 1u);
          mma_bf16_ts(tmem + C::COL_DK, tds + BQ / 2 + kk * 8, qh, id_dk, 1u);
        }
        mma_commit(&bars.dk_done[I % C::NS]);  // frees dP buffer I & 1 and stage I % NS
        return true;
      };
      bool ok = true;
      for (int m = 0; ok && m < n_items; ++m) {
        const int I0 = m * nqt;
        if (!mbar_wait(&bars.k_full, m & 1, abort, a.wait)) { ok = false; break; }
        for (int i = 0; ok && i < nqt; ++i) {
          const int I = I0 + i, st = I % C::NS;
          if (!mbar_wait(&bars.q_full[st], (I / C::NS) & 1, abort, a.wait)) { ok = false; break; }
          if (C::DK) {
            // one S buffer: the rows of tile I - 1 have read it
            if (I >= 1 && !mbar_wait(&bars.s_free[0], (I - 1) & 1, abort, a.wait)) { ok = false; break; }
            fence_after_sync();
            issue_s(I, 0);
            mma_commit(&bars.s_full[I & 1]);  // per tile parity: each warpgroup waits its own
            // V reaches tensor memory through the row threads (the item's first S runs
            // meanwhile); dP buffer I & 1 held dS(I - 2) until dK(I - 2) drained it
            if (i == 0 && !mbar_wait(&bars.v_full, m & 1, abort, a.wait)) { ok = false; break; }
            if (I >= 2 && !mbar_wait(&bars.dk_done[(I - 2) % C::NS], ((I - 2) / C::NS) & 1, abort,
                                     a.wait)) {
              ok = false;
              break;
            }
            fence_after_sync();
            issue_dp(I);
            mma_commit(&bars.dp_full[I & 1]);
            if (i >= 1 && !issue_dk(I - 1, i == 1, m)) { ok = false; break; }
          } else {
            const int sb = I & 1;
            if (I >= 2 && !mbar_wait(&bars.s_free[sb], ((I >> 1) - 1) & 1, abort, a.wait)) {
              ok = false;
              break;
            }
            fence_after_sync();
            issue_s(I, sb * 128);
            mma_commit(&bars.s_full[sb]);
          }
        }
        if (ok && C::DK && nqt > 0) ok = issue_dk(I0 + nqt - 1, nqt == 1, m);
        mma_commit(&bars.done);  // this item's products (also when the loop stopped early)
      }
      mma_commit(&bars.all_done);
      if (!ok) *abort = 1;
      mbar_wait(&bars.all_done, 0);  // every MMA of this CTA has completed
    }
  } else {
    // --------------------------------------------------------- key rows
    const int wg = warp >> 2;  // warpgroup: query tiles I with I % 2 == wg
    const int row = tid & (BK - 1);
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const float sl2 = a.scale * L2E;
    bool ok = true;
    for (int m = 0; ok && m < n_items; ++m) {
      const int k0 = ((int)blockIdx.x + m * (int)gridDim.x) * BK, I0 = m * nqt;
      const int kr = k0 + row;
      const bool kvalid = kr < nk;
      if (C::DK) {
        // the previous item's last dP product has read V from tensor memory
        if (m > 0 && nqt > 0)
          ok = __all_sync(0xffffffffu, mbar_wait(&bars.dp_full[(I0 - 1) & 1], ((I0 - 1) >> 1) & 1,
                                                 abort, a.wait));
        if (!ok) break;
        fence_after_sync();
        // this warpgroup's half of the value row, split into fp16 hi / lo, into tensor
        // memory: the A operand of dP^T = V Go^T (rows past the problem are zero)
        const float4 *v4 = reinterpret_cast<const float4 *>(a.v32 + (k_begin + kr) * D);
#pragma unroll 1
        for (int c0 = wg * 32; c0 < D / 2; c0 += 64) {  // packed columns c0 .. c0 + 31
          uint32_t wh[32], wl[32];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float4 v = kvalid ? v4[c0 / 2 + e] : make_float4(0.f, 0.f, 0.f, 0.f);
            split_pack_f16(v.x, v.y, wh[2 * e], wl[2 * e]);
            split_pack_f16(v.z, v.w, wh[2 * e + 1], wl[2 * e + 1]);
          }
          tmem_st32u(tmem + lane_base + C::COL_V + c0, wh);
          tmem_st32u(tmem + lane_base + C::COL_V + D / 2 + c0, wl);
        }
        tmem_wait_st();
        fence_before_sync();
        mbar_arrive(&bars.v_full);
      }
      float imp = 0.f;
      // this warpgroup's tiles: I % 2 == wg (I counts query tiles over the CTA's items)
      for (int I = I0 + ((I0 ^ wg) & 1); I < I0 + nqt; I += 2) {
        const int sb = I & 1, st = I % C::NS;
        // S of tile I is signalled on s_full[I & 1] (phase I / 2) in both modes
        ok = __all_sync(0xffffffffu, mbar_wait(&bars.s_full[sb], (I >> 1) & 1, abort, a.wait));
        // the tile's l and delta were staged by the producer lanes: acquire them directly
        ok = ok && __all_sync(0xffffffffu, mbar_wait(&bars.q_full[st], (I / C::NS) & 1, abort, a.wait));
        if (!ok) break;
        fence_after_sync();
        float s[BQ];
        {
          float t[BQ];  // the two halves of the score product
          const uint32_t col = C::DK ? 0u : (uint32_t)sb * 128u;
          tmem_ld64x2(tmem + lane_base + col, s, tmem + lane_base + col + BQ, t);
#pragma unroll
          for (int c = 0; c < BQ; ++c) s[c] += t[c];
        }
        fence_before_sync();
        mbar_arrive(&bars.s_free[C::DK ? 0 : sb]);
        const float4 *l4 = reinterpret_cast<const float4 *>(bars.lse2[st]);
        if (!C::DK) {
#pragma unroll
          for (int c4 = 0; c4 < BQ / 4; ++c4) {  // l = +inf past the problem
            const float4 l = l4[c4];
            imp += ex2(fmaf(s[4 * c4], sl2, -l.x)) + ex2(fmaf(s[4 * c4 + 1], sl2, -l.y)) +
                   ex2(fmaf(s[4 * c4 + 2], sl2, -l.z)) + ex2(fmaf(s[4 * c4 + 3], sl2, -l.w));
          }
        } else {
          ok = __all_sync(0xffffffffu, mbar_wait(&bars.dp_full[sb], (I >> 1) & 1, abort, a.wait));
          if (!ok) break;
          fence_after_sync();
          const uint32_t tdp = tmem + lane_base + C::COL_DP + sb * BQ;
          float dp[BQ];
          tmem_ld64(tdp, dp);
          uint32_t hh[BQ / 2], ll[BQ / 2];
          const float4 *d4 = reinterpret_cast<const float4 *>(bars.del[st]);
#pragma unroll
          for (int c4 = 0; c4 < BQ / 4; ++c4) {
            // queries past the problem have l = +inf (p = 0), delta = 0 and zero Q and
            // Go rows; rows of keys past it only feed their own dK rows, which are not
            // stored
            const float4 l = l4[c4], dl = d4[c4];
            const int c = 4 * c4;
            const float v0 = ex2(fmaf(s[c], sl2, -l.x)) * (dp[c] - dl.x);
            const float v1 = ex2(fmaf(s[c + 1], sl2, -l.y)) * (dp[c + 1] - dl.y);
            const float v2 = ex2(fmaf(s[c + 2], sl2, -l.z)) * (dp[c + 2] - dl.z);
            const float v3 = ex2(fmaf(s[c + 3], sl2, -l.w)) * (dp[c + 3] - dl.w);
            split_pack(v0, v1, hh[2 * c4], ll[2 * c4]);
            split_pack(v2, v3, hh[2 * c4 + 1], ll[2 * c4 + 1]);
          }
          // dS (hi, lo) over this tile's dP buffer: the A operand of dK += dS Q
          tmem_st32u(tdp, hh);
          tmem_st32u(tdp + BQ / 2, ll);
          tmem_wait_st();
          fence_before_sync();
          mbar_arrive(&bars.ds_full[sb]);
        }
        if (!C::DK) mbar_arrive(&bars.q_empty[st]);
      }
      if (!ok) *abort = 1;
      if (C::DK) {
        if (!mbar_wait(&bars.done, m & 1, abort, a.wait)) *abort = 1;
        fence_after_sync();
        const float dks = a.scale / go_scale(nq, D, a.w_out);  // score scale, Go's scale undone
#pragma unroll 1
        for (int c0 = wg * (D / 2); c0 < (wg + 1) * (D / 2); c0 += 32) {
          float o[32];
          tmem_ld32(tmem + lane_base + C::COL_DK + c0, o);
          if (nqt == 0) {  // a split without query tiles contributes zero
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0.f;
          }
          if (kvalid) {
            float4 *dst = reinterpret_cast<float4 *>(a.dk + blockIdx.z * a.dk_stride +
                                                     (k_begin + kr) * D + c0);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(o[4 * e] * dks, o[4 * e + 1] * dks, o[4 * e + 2] * dks,
                                   o[4 * e + 3] * dks);
          }
        }
        // dK is read: the next item's first dK product may overwrite it
        fence_before_sync();
        mbar_arrive(&bars.dk_free);
      } else {
        if (wg == 1) bars.imp[row] = imp;
        rows_sync();
        if (wg == 0 && kvalid) a.imp[k_begin + kr] = imp + bars.imp[row];
        rows_sync();  // the next item writes bars.imp again
      }
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
int launch_bwd_tc(const BwdMaps &m, const BwdArgs &a, int max_tiles, int items, int B,
                  cudaStream_t st) {
  using C = Bwd<D, MODE>;
  static_assert(C::SMEM + sizeof(BwdBars) <= 232448, "shared memory");
  auto kern = k_attn_bwd<D, MODE>;
  KVS_CUDA_TRY(set_smem_once(kern, C::SMEM));
  // each CTA takes up to `items` key tiles of its problem, one after another
  const int gx = (max_tiles + items - 1) / items;
  kern<<<dim3(gx, B, a.nsplit), NTHREADS, C::SMEM, st>>>(m.kh, m.kl, m.qh, m.ql, m.g, a);
  KVS_LAUNCH_CHECK("k_attn_bwd");
  return KVS_OK;
}

template int launch_bwd_tc<64, BWD_DK>(const BwdMaps &, const BwdArgs &, int, int, int, cudaStream_t);
template int launch_bwd_tc<128, BWD_DK>(const BwdMaps &, const BwdArgs &, int, int, int, cudaStream_t);
template int launch_bwd_tc<64, BWD_COLSUM>(const BwdMaps &, const BwdArgs &, int, int, int, cudaStream_t);
template int launch_bwd_tc<128, BWD_COLSUM>(const BwdMaps &, const BwdArgs &, int, int, int, cudaStream_t);

}  // namespace kvs
