// Query-tile attention kernel on tcgen05 tensor cores.
//
// "KVSculpt: KV Cache Compression as Distillation", section 2 "Loss
// Function": the compressed cache's attention output Y_hat and log-sum-exp
// l_hat are matched to the full cache's (Y, l) over the training queries.
//
// One CTA owns 128 training queries of one head-problem and streams the
// problem's keys in tiles of 128.  Every product keeps about 16 significant
// bits through a bf16 hi/lo split, with fp32 accumulation in tensor memory:
//   S = Q K^T     Q_hi K_hi + Q_hi K_lo + Q_lo K_hi   (Q and K in smem; N = 128)
//   online softmax, one thread per query row, lazy rescaling of O
//   O += P V      P_hi [V_hi | V_lo] (N = 2d) + P_lo V_hi (N = d)  (P in TMEM over S)
// An instruction of N = 128 costs half as much as one of N = 256, so the value
// product takes V_hi and V_lo side by side for P_hi: two instructions per 16
// keys instead of three, into two output halves O_a = P_hi V_hi + P_lo V_hi and
// O_b = P_hi V_lo, summed at the end.
// Keys and values have separate shared-memory rings: the next key tile loads
// while P V of the previous tile runs, the value tile while S of the next runs.
// Tensor memory (512 columns): S/P buffers at 0 and 128, O_a | O_b at 256.
// Modes:
//   LOSS     keys K_c, values V_c: writes l_hat, Go = dL/dY_hat (fp16, scaled by
//            go_scale), delta = Go . Y_hat - dL/dl_hat (same scale, with the
//            rounded Go), loss partials
//   TARGETS  keys K_z, values V_z: writes Y (fp32 and bf16 hi/lo) and l
//   STATS    row log-sum-exp only
//   WRITE_A  given l_hat: writes A = exp(S - l_hat) as bf16 hi/lo
// Two row warpgroups split every key tile: warpgroup g takes keys 64g .. 64g+63
// of each tile for all 128 query rows (the row maximum is exchanged through
// shared memory once per tile), and output columns g*d/2 .. in the epilogue.
// Warp roles: warps 0-7 softmax/epilogue (warp w <-> TMEM lanes 32 (w % 4) ..,
// thread t <-> query row t % 128), warp 8 TMA producer (Q once, then keys and
// values), warp 9 TMEM allocator and MMA issuer.
#include <math.h>

#include "kvs_attn_tc.cuh"

namespace kvs {
namespace {

using namespace tc;

constexpr int BM = 128;          // queries per CTA
constexpr int BN = FWD_BN;       // keys per tile
constexpr int HB = BN / 2;       // keys of a tile per row warpgroup
constexpr int NTHREADS = 320;
constexpr float kRescale = 8.f;  // lazy rescale threshold (log2 units)
constexpr float L2E = 1.4426950408889634f;
static_assert(BN == 128, "tensor-memory layout assumes 128-key tiles");

template <int D, int MODE>
struct Fwd {
  static constexpr int KD = D / 64;
  static constexpr bool PV = (MODE == FWD_LOSS || MODE == FWD_TARGETS);
  static constexpr int T_BYTES = BN * D * 2;   // one 128-row bf16 tile (hi or lo)
  static constexpr bool WA = MODE == FWD_WRITE_A;
  static constexpr int NSK = (PV || WA) ? 1 : 2;  // key stages (K hi + K lo each)
  static constexpr int NSV = PV ? 1 : 0;       // value stages (V hi + V lo each)
  static constexpr int NSVI = PV ? NSV : 1;     // ring index modulus (unused without values)
  static constexpr int OFF_K = 2 * T_BYTES;    // after Q hi, Q lo (BM = BN rows)
  static constexpr int OFF_V = OFF_K + NSK * 2 * T_BYTES;
  static constexpr int OFF_STG = OFF_V + NSV * 2 * T_BYTES;
  static constexpr int STG_WARP = 2 * 32 * HB * 2;  // WRITE_A: a row warp's 32 x 64 A hi and lo
  static constexpr int BYTES = OFF_STG + (WA ? 8 * STG_WARP : 0);
  static constexpr int SMEM = BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_O = 2 * BN;     // O_a at +0, O_b at +D
  // the single key / value stages are freed by the commits that signal S and P V
  static_assert(!PV || (NSK == 1 && NSVI == 1), "stage release through s_full / s_free");
  static_assert(!WA || NSK == 1, "stage release through s_full");
  // LOSS: the fp32 target tile (BM x D) takes the key stage after the last S
  static_assert(MODE != FWD_LOSS || NSK * 2 * T_BYTES >= BM * D * 4, "target tile");
};
static_assert(BM == BN, "the Q tile shares the key tile's layout");

struct FwdBars {
  uint64_t q_full;
  uint64_t k_full[3], k_empty[3];
  uint64_t v_full[1];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2];
  uint64_t o_done;       // P V of the work item's last tile done (once per item)
  uint64_t o_free;       // the rows have read the item's O (once per item)
  uint64_t y_full;       // LOSS: the item's target rows landed in the key stage
  uint64_t y_free;       // LOSS: the rows have read them (the key stage is free again)
  uint64_t all_done;     // every MMA of the CTA has completed
  uint32_t tmem;
  int abort;
  float red[8];
  float mx[2][BM];       // per warpgroup row maximum of the current tile (raw scores)
  float ls[2][BM];       // per warpgroup running sums
  float part[2][BM][2];  // per warpgroup half-row sums: |Yh - Y|^2, Go . Yh
};

__device__ __forceinline__ void rows_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Barrier of the 256 row threads that also ANDs a predicate over them: every
// row thread leaves the tile loop at the same tile.
__device__ __forceinline__ bool rows_all(bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)p)
      : "memory");
  return r != 0;
}

template <int D, int MODE>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_attn_fwd(const __grid_constant__ CUtensorMap mKh, const __grid_constant__ CUtensorMap mKl,
               const __grid_constant__ CUtensorMap mVh, const __grid_constant__ CUtensorMap mVl,
               const __grid_constant__ CUtensorMap mQh, const __grid_constant__ CUtensorMap mQl,
               const __grid_constant__ CUtensorMap mY, FwdArgs a) {
  using C = Fwd<D, MODE>;
  extern __shared__ unsigned char smraw[];
  unsigned char *sm = (unsigned char *)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
  __shared__ FwdBars bars;
  const int b = blockIdx.y;
  if (a.flt.skip(b)) return;
  const int64_t q_begin = a.q_off[b];
  const int nq = (int)(a.q_off[b + 1] - q_begin);
  // work items: query tiles blockIdx.x, blockIdx.x + gridDim.x, ... of problem b,
  // processed one after another; the next item's query copy and first score
  // product overlap the current item's last P V and epilogue
  const int nqt = (nq + BM - 1) / BM;
  const int n_items = (int)blockIdx.x < nqt ? (nqt - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  if (n_items == 0) return;
  const int64_t k_begin = a.k_off[b];
  const int nk = (int)(a.k_off[b + 1] - k_begin);
  const int ntiles = (nk + BN - 1) / BN;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(&bars.q_full, 1);
    for (int i = 0; i < C::NSK; ++i) {
      mbar_init(&bars.k_full[i], 1);
      mbar_init(&bars.k_empty[i], 1);
    }
    for (int i = 0; i < C::NSV; ++i) mbar_init(&bars.v_full[i], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.s_free[i], C::PV ? 1 : 2 * BM);
      mbar_init(&bars.p_full[i], 2 * BM);
    }
    mbar_init(&bars.o_done, 1);
    mbar_init(&bars.o_free, 2 * BM);
    mbar_init(&bars.y_full, 1);
    mbar_init(&bars.y_free, 2 * BM);
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
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_map(&mKh);
      int q_issued = 0, k_issued = 0, v_issued = 0, y_issued = 0;
      // tile J (counted over the CTA's items; j within its item)
      auto load_k = [&](int J, int j) -> bool {
        const int st = J % C::NSK;
        if (J >= C::NSK) {
          // one stage: free once S(J - 1) has completed, which its commit on s_full
          // signals (a separate commit per tile would cost the tensor pipe a slot)
          const bool w = C::NSK == 1
                             ? mbar_wait(&bars.s_full[(J - 1) & 1], ((J - 1) >> 1) & 1, abort, a.wait)
                             : mbar_wait(&bars.k_empty[st], ((J / C::NSK) - 1) & 1, abort, a.wait);
          if (!w) return false;
        }
        k_issued = J + 1;
        unsigned char *base = sm + C::OFF_K + st * 2 * C::T_BYTES;
        const int krow = (int)(a.k_pad[b] + j * BN);
        mbar_arrive_expect_tx(&bars.k_full[st], 2 * C::T_BYTES);
        for (int r = 0; r < C::KD; ++r) {
          tma_load_2d(base + r * BN * 128, &mKh, &bars.k_full[st], 64 * r, krow);
          tma_load_2d(base + C::T_BYTES + r * BN * 128, &mKl, &bars.k_full[st], 64 * r, krow);
        }
        return true;
      };
      auto load_v = [&](int J, int j) -> bool {
        const int st = J % C::NSVI;
        // one stage: free once P V of tile J - 1 has completed (its commit on s_free)
        if (J >= 1 && !mbar_wait(&bars.s_free[(J - 1) & 1], ((J - 1) >> 1) & 1, abort, a.wait))
          return false;
        v_issued = J + 1;
        unsigned char *base = sm + C::OFF_V + st * 2 * C::T_BYTES;
        const int krow = (int)(a.k_pad[b] + j * BN);
        mbar_arrive_expect_tx(&bars.v_full[st], 2 * C::T_BYTES);
        for (int r = 0; r < C::KD; ++r) {
          tma_load_2d(base + r * BN * 128, &mVh, &bars.v_full[st], 64 * r, krow);
          tma_load_2d(base + C::T_BYTES + r * BN * 128, &mVl, &bars.v_full[st], 64 * r, krow);
        }
        return true;
      };
      bool ok = true;
      for (int m = 0; ok && m < n_items; ++m) {
        const int q0 = ((int)blockIdx.x + m * (int)gridDim.x) * BM;
        const int J0 = m * ntiles;
        // the item's query tile, hi and lo (padded rows: zeros past the problem), once
        // the previous item's last score product no longer reads the buffer
        if (m > 0 && ntiles > 0 &&
            !mbar_wait(&bars.s_full[(J0 - 1) & 1], ((J0 - 1) >> 1) & 1, abort, a.wait)) {
          ok = false;
          break;
        }
        q_issued = m + 1;
        const int qrow = (int)(a.a_pad_off[b] + q0);
        mbar_arrive_expect_tx(&bars.q_full, 2 * C::T_BYTES);
        for (int r = 0; r < C::KD; ++r) {
          tma_load_2d(sm + r * BM * 128, &mQh, &bars.q_full, 64 * r, qrow);
          tma_load_2d(sm + C::T_BYTES + r * BM * 128, &mQl, &bars.q_full, 64 * r, qrow);
        }
        if (C::PV) {
          // LOSS: the key stage holds the previous item's targets until the rows have read them
          if (MODE == FWD_LOSS && m > 0 && !mbar_wait(&bars.y_free, (m - 1) & 1, abort, a.wait)) {
            ok = false;
            break;
          }
          // key tile j+1 goes ahead of value tile j: S of the next tile never waits
          // behind the value ring
          if (ntiles > 0) ok = load_k(J0, 0);
          for (int j = 0; ok && j < ntiles; ++j) {
            if (j + 1 < ntiles) ok = load_k(J0 + j + 1, j + 1);
            ok = ok && load_v(J0 + j, j);
          }
          if (MODE == FWD_LOSS && ok) {
            // the item's target rows (fp32) into the key stage once its last S is done:
            // the epilogue reads them from shared memory instead of waiting on global
            // loads after the last P V
            if (ntiles > 0)
              ok = mbar_wait(&bars.s_full[(J0 + ntiles - 1) & 1], ((J0 + ntiles - 1) >> 1) & 1,
                             abort, a.wait);
            if (ok) {
              y_issued = m + 1;
              mbar_arrive_expect_tx(&bars.y_full, BM * D * 4);
              for (int r = 0; r < D / 32; ++r)
                tma_load_2d(sm + C::OFF_K + r * BM * 128, &mY, &bars.y_full, 32 * r,
                            (int)(q_begin + q0));
            }
          }
        } else {
          for (int j = 0; ok && j < ntiles; ++j) ok = load_k(J0 + j, j);
        }
      }
      if (!ok) *abort = 1;
      if (*abort) {  // let issued copies land before shared memory is released
        if (q_issued) mbar_wait(&bars.q_full, (q_issued - 1) & 1);
        for (int J = (k_issued > C::NSK ? k_issued - C::NSK : 0); J < k_issued; ++J)
          mbar_wait(&bars.k_full[J % C::NSK], (J / C::NSK) & 1);
        for (int J = (v_issued > C::NSVI ? v_issued - C::NSVI : 0); J < v_issued; ++J)
          mbar_wait(&bars.v_full[J % C::NSVI], (J / C::NSVI) & 1);
        if (y_issued) mbar_wait(&bars.y_full, (y_issued - 1) & 1);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s128 = idesc_bf16(BM, BN, false, false);
      const uint32_t id_s64 = idesc_bf16(BM, 64, false, false);
      const uint32_t id_pv = idesc_bf16(BM, 2 * D, false, true);  // N = [V_hi | V_lo]
      const uint32_t id_pvh = idesc_bf16(BM, D, false, true);     // N = V_hi
      const uint64_t qh0 = sdesc(smem_u32(sm), 16, 1024), ql0 = sdesc_add(qh0, C::T_BYTES);
      // P V of tile I (over the CTA's items); `first`: the item's first tile, whose
      // product overwrites O once the rows have read the previous item's O
      auto issue_pv = [&](int I, int i, bool first, int m) -> bool {
        const int pb = I & 1;
        if (!mbar_wait(&bars.p_full[pb], (I >> 1) & 1, abort, a.wait)) return false;
        if (!mbar_wait(&bars.v_full[I % C::NSVI], (I / C::NSVI) & 1, abort, a.wait)) return false;
        if (first && m > 0 && !mbar_wait(&bars.o_free, (m - 1) & 1, abort, a.wait)) return false;
        fence_after_sync();
        // V_hi and V_lo boxes sit back to back with one stride: one N = 2d operand
        const uint64_t v0 = sdesc(smem_u32(sm + C::OFF_V + (I % C::NSVI) * 2 * C::T_BYTES),
                                  BN * 128, 1024);
        const uint32_t tp = tmem + pb * BN;  // P hi at +0, P lo at +BN/2 columns
        const int kv = min(nk - i * BN, BN);
        const int nks = (kv + 15) / 16;      // key steps that hold valid keys
        for (int kk = 0; kk < nks; ++kk) {
          const uint64_t v = sdesc_add(v0, kk * 2048);
          // P_hi [V_hi | V_lo] into both halves, P_lo V_hi into the first
          mma_bf16_ts(tmem + C::COL_O, tp + kk * 8, v, id_pv, (!first || kk > 0) ? 1u : 0u);
          mma_bf16_ts(tmem + C::COL_O, tp + BN / 2 + kk * 8, v, id_pvh, 1u);
        }
        mma_commit(&bars.s_free[pb]);  // also frees the value stage
        return true;
      };
      bool ok = true;
      for (int m = 0; ok && m < n_items; ++m) {
        const int J0 = m * ntiles;
        if (!mbar_wait(&bars.q_full, m & 1, abort, a.wait)) { ok = false; break; }
        for (int j = 0; ok && j < ntiles; ++j) {
          const int J = J0 + j, st = J % C::NSK, sb = J & 1;
          if (!mbar_wait(&bars.k_full[st], (J / C::NSK) & 1, abort, a.wait)) { ok = false; break; }
          if (J >= 2 && !mbar_wait(&bars.s_free[sb], ((J >> 1) - 1) & 1, abort, a.wait)) { ok = false; break; }
          fence_after_sync();
          // a last tile with at most 64 keys takes the narrower product
          const uint32_t id_s = (nk - j * BN) > 64 ? id_s128 : id_s64;
          const uint64_t kh0 = sdesc(smem_u32(sm + C::OFF_K + st * 2 * C::T_BYTES), 16, 1024);
          const uint64_t kl0 = sdesc_add(kh0, C::T_BYTES);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * (BN * 128) + (kk & 3) * 32;  // same for Q and K
            const uint64_t kh = sdesc_add(kh0, off), kl = sdesc_add(kl0, off);
            const uint64_t qh = sdesc_add(qh0, off), ql = sdesc_add(ql0, off);
            mma_bf16(tmem + sb * BN, qh, kh, id_s, kk > 0 ? 1u : 0u);
            mma_bf16(tmem + sb * BN, qh, kl, id_s, 1u);
            mma_bf16(tmem + sb * BN, ql, kh, id_s, 1u);
          }
          mma_commit(&bars.s_full[sb]);
          if (C::NSK > 1) mma_commit(&bars.k_empty[st]);  // one stage: freed through s_full
          if (C::PV && j >= 1 && !issue_pv(J - 1, j - 1, j == 1, m)) { ok = false; break; }
        }
        if (ok && C::PV && ntiles > 0) ok = issue_pv(J0 + ntiles - 1, ntiles - 1, ntiles == 1, m);
        mma_commit(&bars.o_done);  // this item's products (also when the loop stopped early)
      }
      mma_commit(&bars.all_done);
      if (!ok) *abort = 1;
      mbar_wait(&bars.all_done, 0);  // every MMA of this CTA has completed
    }
  } else {
    // ------------------------------------------------- softmax / epilogue rows
    const int wg = warp >> 2;          // keys 64 wg .. of every tile
    const int row = tid & (BM - 1);    // query row
    const int cb = wg * HB;            // first key (S column) of this warpgroup
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const float sl2 = a.scale * L2E;  // score scale in log2 units
    bool ok = true;
    for (int m = 0; ok && m < n_items; ++m) {
      const int qt = (int)blockIdx.x + m * (int)gridDim.x;  // the item's query tile
      const int q0 = qt * BM, J0 = m * ntiles;
      const int q = q0 + row;
      const bool valid = q < nq;
      float lrow2 = 0.f;                // WRITE_A: the given lse in log2 units
      if (MODE == FWD_WRITE_A && valid) lrow2 = a.lse_in[q_begin + q] * L2E;
      float mref = -INFINITY, lsum = 0.f;  // mref is the same in both warpgroups
      for (int j = 0; j < ntiles; ++j) {
        const int J = J0 + j, sb = J & 1;  // J counts tiles over the CTA's items
        ok = ok && __all_sync(0xffffffffu, mbar_wait(&bars.s_full[sb], (J >> 1) & 1, abort, a.wait));
        if (MODE == FWD_WRITE_A && !ok) break;  // no barrier below in this mode
        float s[HB];
        if (ok) {
          fence_after_sync();
          tmem_ld64(tmem + lane_base + sb * BN + cb, s);
        } else {
#pragma unroll
          for (int c = 0; c < HB; ++c) s[c] = -INFINITY;
        }
        const int kvalid = nk - j * BN - cb;  // raw scores; keys past the problem get -inf
        if (kvalid < HB) {
#pragma unroll
          for (int c = 0; c < HB; ++c) s[c] = (c < kvalid) ? s[c] : -INFINITY;
        }
        if (!C::PV) {
          fence_before_sync();
          mbar_arrive(&bars.s_free[sb]);
        }
        if (MODE == FWD_WRITE_A) {
          // A = exp2(t - lse2), split into bf16 hi / lo.  The warp stages its 32 rows
          // x 64 keys in shared memory (16-byte chunks XOR-swizzled by row), then
          // writes them out as whole 128-byte row segments of the padded A buffer.
          uint4 *stg = reinterpret_cast<uint4 *>(sm + C::OFF_STG + warp * C::STG_WARP);
#pragma unroll
          for (int ch = 0; ch < HB / 8; ++ch) {
            uint32_t h[4], l[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float p0 = valid ? ex2(fmaf(s[ch * 8 + 2 * e], sl2, -lrow2)) : 0.f;
              const float p1 = valid ? ex2(fmaf(s[ch * 8 + 2 * e + 1], sl2, -lrow2)) : 0.f;
              split_pack(p0, p1, h[e], l[e]);
            }
            const int slot = lane * 8 + (ch ^ (lane & 7));
            stg[slot] = make_uint4(h[0], h[1], h[2], h[3]);
            stg[256 + slot] = make_uint4(l[0], l[1], l[2], l[3]);
          }
          __syncwarp();
          const int64_t arow0 = a.a_pad_off[b] + q0 + (warp & 3) * 32;
          const int cc = lane & 7;
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            const int rr = it * 4 + (lane >> 3);
            const int slot = rr * 8 + (cc ^ (rr & 7));
            const int64_t off = (arow0 + rr) * a.ld_a + j * BN + cb + cc * 8;
            *reinterpret_cast<uint4 *>(a.a_hi + off) = stg[slot];
            *reinterpret_cast<uint4 *>(a.a_lo + off) = stg[256 + slot];
          }
          __syncwarp();  // the staging is reused by the next tile
          continue;
        }
        float mt = -INFINITY;
#pragma unroll
        for (int c = 0; c < HB; ++c) mt = fmaxf(mt, s[c]);
        // the tile's row maximum over both halves; the barrier also orders both
        // warpgroups' S loads before either writes P over the buffer
        bars.mx[wg][row] = mt;
        ok = rows_all(ok);  // a wait that gave up anywhere ends the loop for every row
        if (!ok) break;
        mt = fmaxf(bars.mx[0][row], bars.mx[1][row]) * sl2;  // the scale is positive
        float alpha = 1.f;
        bool rescale = false;
        if (mt > mref + kRescale || mref == -INFINITY) {
          const float mnew = fmaxf(mt, mref);
          if (mref != -INFINITY) {
            alpha = ex2(mref - mnew);
            rescale = true;
          }
          mref = mnew;
        }
        float ts = 0.f;
#pragma unroll
        for (int c = 0; c < HB; ++c) {
          s[c] = ex2(fmaf(s[c], sl2, -mref));
          ts += s[c];
        }
        lsum = lsum * alpha + ts;
        if (C::PV) {
          // P (hi, lo) of this warpgroup's keys over the S buffer: the A operand of O += P V
          {
            uint32_t ph[32], pl[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) split_pack(s[2 * c], s[2 * c + 1], ph[c], pl[c]);
            tmem_st32u(tmem + lane_base + sb * BN + cb / 2, ph);
            tmem_st32u(tmem + lane_base + sb * BN + BN / 2 + cb / 2, pl);
          }
          if (__any_sync(0xffffffffu, rescale)) {
            // O *= alpha once PV of tile j-1 has landed (PV of tile j waits for p_full);
            // the TMEM access is warp-wide, rows without a new max use alpha = 1.  The
            // rows' rescale decisions are the same in both warpgroups; each scales
            // one output half.
            const int pj = J - 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&bars.s_free[pj & 1], (pj >> 1) & 1, abort, a.wait));
            if (ok) {  // a failed wait ends the loop at the next tile's row barrier
              fence_after_sync();
#pragma unroll 1
              for (int c0 = wg * D; c0 < (wg + 1) * D; c0 += 32) {
                float o[32];
                tmem_ld32(tmem + lane_base + C::COL_O + c0, o);
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] *= alpha;
                tmem_st32(tmem + lane_base + C::COL_O + c0, o);
              }
            }
          }
          tmem_wait_st();
          fence_before_sync();
          mbar_arrive(&bars.p_full[sb]);
        }
      }
      if (!ok) *abort = 1;
      // ------------------------------------------------------------ epilogue
      if (MODE != FWD_WRITE_A) {
        bars.ls[wg][row] = lsum;
        rows_sync();
        lsum = bars.ls[0][row] + bars.ls[1][row];
        const float lse = (mref + log2f(lsum)) * 0.6931471805599453f;
        if (C::PV) {
          if (!mbar_wait(&bars.o_done, m & 1, abort, a.wait)) *abort = 1;
          if (MODE == FWD_LOSS && !mbar_wait(&bars.y_full, m & 1, abort, a.wait)) *abort = 1;
          fence_after_sync();
        }
        const float inv = 1.f / lsum;
        const float sig = go_scale(nq, D, a.w_out);
        const float c_out = 2.f * a.w_out / ((float)nq * (float)D) * sig;  // scaled
        const float c_lse = 2.f * a.w_lse / (float)nq * sig;
        const int64_t grow = q_begin + q;
        const int64_t prow = a.a_pad_off[b] + q;  // row of the padded bf16 buffers
        float se = 0.f, ls = 0.f, gy = 0.f;
        if (C::PV) {
          // this warpgroup's half of the row's output columns
#pragma unroll 1
          for (int c0 = wg * (D / 2); c0 < (wg + 1) * (D / 2); c0 += 32) {
            float o[32], ob[32];
            tmem_ld32(tmem + lane_base + C::COL_O + c0, o);
            tmem_ld32(tmem + lane_base + C::COL_O + D + c0, ob);
            if (!valid) {
              // rows past the problem: zero padding of the bf16 operand buffers (this
              // CTA's tile ends within the problem's padded rows)
              const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
              if (MODE == FWD_TARGETS) {
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                  reinterpret_cast<uint4 *>(a.y_hi + prow * D + c0)[ch] = z4;
                  reinterpret_cast<uint4 *>(a.y_lo + prow * D + c0)[ch] = z4;
                }
              } else {
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) reinterpret_cast<uint4 *>(a.go + prow * D + c0)[ch] = z4;
              }
              continue;
            }
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = (o[e] + ob[e]) * inv;  // O = O_a + O_b
            if (MODE == FWD_TARGETS) {
              float4 *y4 = reinterpret_cast<float4 *>(a.y_out + grow * D + c0);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                y4[e] = make_float4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
              uint4 *yh = reinterpret_cast<uint4 *>(a.y_hi + prow * D + c0);
              uint4 *yl = reinterpret_cast<uint4 *>(a.y_lo + prow * D + c0);
#pragma unroll
              for (int ch = 0; ch < 4; ++ch) {
                uint32_t h[4], l[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  split_pack(o[ch * 8 + 2 * e], o[ch * 8 + 2 * e + 1], h[e], l[e]);
                yh[ch] = make_uint4(h[0], h[1], h[2], h[3]);
                yl[ch] = make_uint4(l[0], l[1], l[2], l[3]);
              }
            } else {
              // Y[row][c0 .. c0 + 31]: one 128-byte swizzled row of box c0 / 32
              const unsigned char *yrow = sm + C::OFF_K + (c0 >> 5) * (BM * 128) + row * 128;
              float ev[32];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float4 v = *reinterpret_cast<const float4 *>(yrow + ((e ^ (row & 7)) << 4));
                ev[4 * e] = o[4 * e] - v.x;
                ev[4 * e + 1] = o[4 * e + 1] - v.y;
                ev[4 * e + 2] = o[4 * e + 2] - v.z;
                ev[4 * e + 3] = o[4 * e + 3] - v.w;
              }
              uint4 *g4 = reinterpret_cast<uint4 *>(a.go + prow * D + c0);
#pragma unroll
              for (int ch = 0; ch < 4; ++ch) {
                uint32_t h[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int i0 = ch * 8 + 2 * e;
                  // delta uses the fp16-rounded Go that the backward's dP product sees,
                  // so the rounding of Go cancels exactly in dP - delta.
                  h[e] = pack_f16(c_out * ev[i0], c_out * ev[i0 + 1]);
                  const float2 gg = unpack_f16(h[e]);
                  const float g0 = gg.x, g1 = gg.y;
                  se = fmaf(ev[i0], ev[i0], se);
                  se = fmaf(ev[i0 + 1], ev[i0 + 1], se);
                  gy = fmaf(g0, o[i0], gy);
                  gy = fmaf(g1, o[i0 + 1], gy);
                }
                g4[ch] = make_uint4(h[0], h[1], h[2], h[3]);
              }
            }
          }
          // O (and the targets in the key stage) are read: the next item's first P V may
          // overwrite O, and its first key tile may take the key stage
          fence_before_sync();
          mbar_arrive(&bars.o_free);
          if (MODE == FWD_LOSS) mbar_arrive(&bars.y_free);
        }
        if (MODE == FWD_LOSS) {
          bars.part[wg][row][0] = se;
          bars.part[wg][row][1] = gy;
          rows_sync();
          if (wg == 0) {
            se = bars.part[0][row][0] + bars.part[1][row][0];
            gy = bars.part[0][row][1] + bars.part[1][row][1];
            if (valid) {
              const float el = lse - a.lse_in[grow];
              ls = el * el;
              a.lse_out[grow] = lse;
              a.delta[grow] = gy - c_lse * el;
            } else {
              se = 0.f;
            }
            // deterministic per-CTA partial sums of the two loss terms
            se = warp_sum(se);
            ls = warp_sum(ls);
            if (lane == 0) {
              bars.red[warp] = se;
              bars.red[4 + warp] = ls;
            }
          }
          rows_sync();
          if (tid == 0) {
            float *part = a.partials + ((int64_t)b * a.tiles_per_problem + qt) * 2;
            part[0] = (bars.red[0] + bars.red[1]) + (bars.red[2] + bars.red[3]);
            part[1] = (bars.red[4] + bars.red[5]) + (bars.red[6] + bars.red[7]);
          }
        } else if (wg == 0 && valid) {  // TARGETS, STATS
          a.lse_out[grow] = lse;
        }
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
int launch_fwd_tc(const FwdMaps &m, const FwdArgs &a, int max_tiles, int items, int B,
                  cudaStream_t st) {
  using C = Fwd<D, MODE>;
  static_assert(C::SMEM + sizeof(FwdBars) <= 232448, "shared memory");
  auto kern = k_attn_fwd<D, MODE>;
  KVS_CUDA_TRY(set_smem_once(kern, C::SMEM));
  // each CTA takes up to `items` query tiles of its problem, one after another
  const int gx = (max_tiles + items - 1) / items;
  kern<<<dim3(gx, B), NTHREADS, C::SMEM, st>>>(m.kh, m.kl, m.vh, m.vl, m.qh, m.ql,
                                               MODE == FWD_LOSS ? m.y : m.kh, a);
  KVS_LAUNCH_CHECK("k_attn_fwd");
  return KVS_OK;
}

template int launch_fwd_tc<64, FWD_LOSS>(const FwdMaps &, const FwdArgs &, int, int, int, cudaStream_t);
template int launch_fwd_tc<128, FWD_LOSS>(const FwdMaps &, const FwdArgs &, int, int, int, cudaStream_t);
template int launch_fwd_tc<64, FWD_TARGETS>(const FwdMaps &, const FwdArgs &, int, int, int, cudaStream_t);
template int launch_fwd_tc<128, FWD_TARGETS>(const FwdMaps &, const FwdArgs &, int, int, int, cudaStream_t);
template int launch_fwd_tc<64, FWD_STATS>(const FwdMaps &, const FwdArgs &, int, int, int, cudaStream_t);
template int launch_fwd_tc<128, FWD_STATS>(const FwdMaps &, const FwdArgs &, int, int, int, cudaStream_t);
template int launch_fwd_tc<64, FWD_WRITE_A>(const FwdMaps &, const FwdArgs &, int, int, int, cudaStream_t);
template int launch_fwd_tc<128, FWD_WRITE_A>(const FwdMaps &, const FwdArgs &, int, int, int, cudaStream_t);

}  // namespace kvs
